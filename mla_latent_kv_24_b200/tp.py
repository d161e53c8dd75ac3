"""Group-sharded GQA-path decode over tensor-parallel ranks.

"GQLA: Group-Query Latent Attention ..." (abstract): the GQA path supports up to 8-way
zero-redundancy tensor parallelism, since its expanded cache splits by KV group, while the
MQA-absorb path replicates the latent on every rank.  Rank r of tp owns KV groups
[r G/tp, (r+1) G/tp) and their heads.  It expands only those groups (the shared RoPE keys stay in
the latent cache, which every rank keeps) and decodes them with the ordinary C-ABI calls, given
dims of H/tp heads.  One all-gather over the head axis then assembles the output.  That
all-gather is the path's only exchange.

This module is plumbing around the library (torch.distributed for the collective); every step
of the decode itself runs in libmla's kernels.
"""
from dataclasses import dataclass

from . import gqla_decode_grouped, make_dims


@dataclass(frozen=True)
class Shard:
    """The heads [head0, head1) and KV groups [group0, group1) that rank `rank` of `tp` owns."""
    rank: int
    tp: int
    head0: int
    head1: int
    group0: int
    group1: int


def shard(dims, tp: int, rank: int) -> Shard:
    """Contiguous, equal shares of the KV groups; tp must divide the group count."""
    H, hpw = dims.n_heads, dims.heads_per_group
    G = H // hpw
    if tp < 1 or G % tp or not 0 <= rank < tp:
        raise ValueError(f"tp = {tp} must divide the {G} KV groups and 0 <= rank < tp (rank = {rank})")
    gl = G // tp
    return Shard(rank, tp, rank * gl * hpw, (rank + 1) * gl * hpw, rank * gl, (rank + 1) * gl)


def local_dims(dims, tp: int):
    """dims of one rank's share: H / tp heads, everything else unchanged."""
    shard(dims, tp, 0)   # validates tp
    return make_dims(n_heads=dims.n_heads // tp, heads_per_group=dims.heads_per_group, d_c=dims.d_c,
                     d_rope=dims.d_rope, d_nope=dims.d_nope, d_v=dims.d_v, page_size=dims.page_size,
                     softmax_scale=dims.softmax_scale, rope_base=dims.rope_base,
                     dtype="bf16" if dims.dtype == 0 else "fp32")


def gather_heads(out_local, group=None):
    """All-gather [B, s_q, H/tp, d_v] from every rank into [B, s_q, H, d_v] (rank order = head order)."""
    import torch
    import torch.distributed as dist
    tp = dist.get_world_size(group)
    parts = [torch.empty_like(out_local) for _ in range(tp)]
    dist.all_gather(parts, out_local.contiguous(), group=group)
    return torch.cat(parts, dim=2)


def decode_grouped_tp(dims, q_local, expanded_local, latent_cache, page_table, seq_lens, seq_lens_host, batch, s_q,
                      max_pages, n_pages_total, out_local, workspace, group=None, stream=None):
    """This rank's grouped decode (its heads, its groups' expanded cache), then the head all-gather.

    q_local [B, s_q, H/tp, d_nope + d_rope] and expanded_local [n_pages, G/tp, page, d_nope + d_v]
    hold this rank's share; the workspace is sized by gqla_decode_workspace_size(local_dims(dims, tp), ...).
    Returns the full [B, s_q, H, d_v] output on every rank."""
    import torch.distributed as dist
    tp = dist.get_world_size(group)
    gqla_decode_grouped(local_dims(dims, tp), q_local, expanded_local, latent_cache, page_table, seq_lens,
                        seq_lens_host, batch, s_q, max_pages, n_pages_total, out_local, workspace, stream=stream)
    return gather_heads(out_local, group)
