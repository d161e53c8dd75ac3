"""mla_select_path: the roofline choice between the MQA-absorb and GQA paths of GQLA weights
("GQLA: Group-Query Latent Attention ..." abstract: the runtime picks the hardware-matched path;
the absorb path trades traffic for computation and replicates the latent on every rank, the GQA
path shards KV groups over up to 8 ranks).  Host arithmetic only: runs without a GPU."""
import pytest

import mla_latent_kv_24_b200 as mla

GQLA = dict(n_heads=128, heads_per_group=8)      # 16 groups of 8 heads, d_c 512, d_rope 64
MLA = dict(n_heads=128, heads_per_group=1)
B, L = 32, 8192
INF = 1e30                                        # a peak so large that its term never binds

# Vendor datasheet figures (dense bf16 tensor throughput, HBM bandwidth) of the two GPUs the page
# names, used only as inputs; the expected choices are the page's claims.
H100 = (3.35e12, 989e12)
H20 = (4.0e12, 148e12)


def select(dims_kw, s_q, bw, fl, tp=1, lens=None):
    return mla.mla_select_path(mla.make_dims(**dims_kw), B, s_q, lens or [L] * B, bw, fl, tp)


def test_h100_mqa_absorb_at_sq1_and_h20_gqa_at_sq2():
    # the page: one set of weights pins the H100 roofline on the MQA-absorb path (s_q = 1) and
    # the H20 roofline on the GQA path with MTP (s_q = 2)
    assert select(GQLA, 1, *H100)[0] == "absorbed"
    assert select(GQLA, 2, *H20)[0] == "grouped"


def test_single_gpu_grouped_path_moves_8320_over_1152_the_bytes():
    # memory only, one rank: per token 16 groups x (128 + 128) x 2 B + 64 x 2 B = 8320 B against the
    # latent's 1152 B (plus the absorbed path's W_UK + W_UV read once)
    _, ta, tg = select(GQLA, 1, 1.0, INF)
    weights = 16 * (128 + 128) * 512 * 2
    assert tg / (ta - weights) == pytest.approx(8320 / 1152, rel=1e-12)


def test_tp8_grouped_bytes_per_rank_equal_the_latent():
    # 8-way group sharding: 2 groups x 512 B + 128 B of shared RoPE key = 1152 B per token, the
    # replicated latent's size; the absorbed rank still reads its 2 groups' weights
    _, ta, tg = select(GQLA, 1, 1.0, INF, tp=8)
    weights = 2 * (128 + 128) * 512 * 2
    assert ta - tg == pytest.approx(weights, rel=1e-12)
    assert tg == pytest.approx(B * L * 1152, rel=1e-12)


def test_flop_ratio_of_the_two_paths():
    # compute only: per visible (query, token) pair and head, 2 x (512 + 64 + 512) flops absorbed
    # against 2 x (128 + 64 + 128) grouped; the absorbed path adds q absorption and W_UV per query
    s_q = 2
    _, ta, tg = select(GQLA, s_q, INF, 1.0)
    visible = B * sum(L - s_q + j + 1 for j in range(s_q))
    per_query = B * s_q * 128 * 2 * 512 * (128 + 128)
    assert (ta - per_query) / tg == pytest.approx(1088 / 320, rel=1e-12)
    assert tg == pytest.approx(visible * 2 * 128 * 320, rel=1e-12)


def test_mla_weights_never_pick_the_grouped_path():
    # hpw = 1: a "group" per head, 128 x 256 x 2 B = 64 KiB per token on the grouped path
    for bw, fl in (H100, H20, (6535.7e9, 1638e12)):
        for s_q in (1, 2, 4):
            assert select(MLA, s_q, bw, fl)[0] == "absorbed"


def test_b200_measured_peaks_prefer_absorb_for_gqla_weights():
    # this GPU's measured copy bandwidth and bf16 GEMM throughput: ridge ~250 flop/B, high enough
    # that the latent's 7.2x smaller traffic wins at s_q = 1 and 2
    for s_q in (1, 2):
        assert select(GQLA, s_q, 6535.7e9, 1638e12)[0] == "absorbed"


def test_ragged_lengths_count_visible_pairs():
    lens = [5, 64, 1000]
    dims = mla.make_dims(**GQLA)
    _, _, tg = mla.mla_select_path(dims, 3, 2, lens, INF, 1.0, 1)
    visible = sum(2 * n - 1 for n in lens)                 # (n - 1) + n for s_q = 2
    assert tg == pytest.approx(visible * 2 * 128 * 320, rel=1e-12)


@pytest.mark.parametrize("kw", [dict(tp=3), dict(s_q=5), dict(s_q=0), dict(tp=0), dict(bw=0.0)])
def test_invalid_arguments_are_rejected(kw):
    args = dict(s_q=1, bw=1e12, fl=1e15, tp=1)
    args.update(kw)
    with pytest.raises(mla.MlaError) as e:
        select(GQLA, args["s_q"], args["bw"], args["fl"], tp=args["tp"])
    assert e.value.status == 1


def test_length_shorter_than_sq_is_rejected():
    with pytest.raises(mla.MlaError):
        mla.mla_select_path(mla.make_dims(**GQLA), 2, 2, [1, 10], 1e12, 1e15, 1)
