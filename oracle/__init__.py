"""CPU oracle for MLA latent-KV decode and the GQLA grouped path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (the C-ABI library and its Python binding) never imports, links or runs it,
and this package imports nothing from the product path.

Sources (the pages this oracle follows, cited by title and section):
  [MLA-GRPO]  "MLA and GRPO architecture" (kushumpoudel.com.np blog), section 2
              "Multi-Head Latent Attention (MLA): Low-Rank Compression": "The Mathematics
              of MLA" (c_t^KV = W_DKV h_t; k_t^C = W_UK c_t^KV, v_t^C = W_UV c_t^KV),
              "Decoupled Rotary Position Embeddings (RoPE)" (cached state [c_t^KV, k_t^R]),
              "Memory Footprint Comparison" table; section 1 (MHA cache-size formula).
  [UPGRADE]   "How to upgrade GQA models to MLA for massive KV Cache Savings" (drivenets),
              "Under the hood: how offline conversion works", stage "Decompression
              Multiplex" (W_UK folded into the query by associativity); "Real-world results"
              (2K -> 768 bytes per token).
  [CLARITY]   "MLA's 512-Scalar KV Latent Cuts Cache 98%, Enabling 512 Concurrent 128k
              Streams" (theclarity.today): 128 heads x 128, latent 512, 32,768-scalar MHA
              baseline, 1.56 %, 64-fold, RoPE / up-projection non-commutation.
  [GQLA-ABS]  "GQLA: Group-Query Latent Attention for Hardware-Adaptive Large Language Model
              Decoding" (arXiv 2605.15250 abstract page): two algebraically equivalent decoding
              paths (MQA-absorb and GQA with a per-group expanded cache); 28.125 %.
  [GQLA-RADIO] "GQLA: Group-Query Latent Attention for Hardware-Adaptive Decoding" (AI Radio
              episode): "Key concepts" (MQA-absorb path, GQA path); the paper's abstract
              ("absorbed and head-expanded forms", group-shared up-projections); transcript
              "The paper's summary" (absorb path caches latent + shared RoPE key; GQA path
              caches per-group K and V + the shared RoPE key).

Readings where the pages are silent (each is a parameter or stated in the docstring where
it is used): softmax scale 1/sqrt(d_nope + d_rope); RoPE on interleaved pairs (2i, 2i+1)
with theta_i = base^(-2i/d_rope); the cache holds the s_q current tokens and query j sits at
position L - s_q + j with keys t <= that position; k_rope = RoPE(W_KR h); head h uses weight
group h // heads_per_group; W_UV stored [d_v, d_c].

Pins: every function here is checked in ``tests/test_oracle.py`` against something other
than itself (pure-Python brute force, closed forms, the equivalence of the absorbed,
expanded and grouped forms, RoPE identities, and the pages' cache-size arithmetic in
``tests/golden/``).  The attention values themselves have no worked example on the pages.
"""
from .mla import (  # noqa: F401
    rope_frequencies, rope, down_project, slot_of, request_rows,
    attention_weights, decode_request_expanded, decode_expanded,
    decode_request_absorbed, expand_group_cache, decode_request_grouped,
    partial_attention, combine_partials, cache_append,
    mha_scalars_per_token, mla_scalars_per_token, gqa_scalars_per_token,
    gqa_path_bytes_per_token, absorbed_path_bytes_per_token,
)
