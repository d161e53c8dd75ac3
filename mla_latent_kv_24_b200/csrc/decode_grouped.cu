// GQA-path split decode over the per-group expanded cache ("GQLA: Group-Query Latent Attention
// ..." abstract: the GQA path with a per-group expanded cache; AI Radio episode transcript:
// per-group K and V plus the shared RoPE key).  For query j of request b (position p_j) and
// head h of group g = h / 8:
//     s_t = scale * ([q_nope | RoPE(q_rope, p_j)] . [K_g,t | k^R_t]),  t <= p_j
//     o   = sum_t softmax(s)_t V_g,t
//
// The queries arrive rotated (the q RoPE kernel runs once per call).  The path is bound by HBM
// (8320 bytes per token for 16 groups, ~10 flop per byte per query), so the kernel streams the
// expanded cache through a two-stage pipeline of tensor copies (TMA: one 32 KiB box of K_g|V_g
// and one 8 KiB box of k^R per page, 128-byte swizzled, completion on an mbarrier), two CTAs
// per SM, and uses warp-level mma.sync (m16n8k16, fp32 accumulators), whose throughput is far
// above what the bytes need.  Two tensor copies per page instead of 2,560 16-byte copies leave
// the issue slots to the MMAs and the softmax, which matters when the SM clock drops under the
// power limit.
// One CTA takes one chunk of one request and one group: the group's 8 heads of every query of
// the request form the 16 rows of the MMA tile (both MTP queries share each K/V tile), so each
// page of K_g|V_g (32 KiB, contiguous) and of k^R (8 KiB) is read once per chunk.  Four warps
// each take 16 tokens of every 64-token page and keep their own online softmax; the CTA merges
// the four (m, l, O) at the end and writes one partial result per query for the combine.
//
// Deeper multi-token prediction (s_q = 3 or 4) uses two 16-row tiles (queries 0-1 and 2-3 of
// the group's 8 heads): every K/V fragment a warp loads from shared memory feeds both tiles, so
// the four queries still share each page read from HBM.
//
// The head-expanded prefill ("GQLA ..." abstract: MLA's absorbed and head-expanded forms) is
// compute-dense and runs on the 5th-generation tensor cores (prefill_tc.cu); only its launcher
// lives here, beside the grouped decode whose cache it reads.
#include <math.h>

#include <cudaTypedefs.h>
#include <mutex>

#include "tc_decode.h"
#include "tc_ptx.cuh"
#include "warp_mma.cuh"

namespace mla {
namespace {

constexpr int GH = 8;                 // heads per group
constexpr int D_N = 128, D_V = 128, D_R = 64, D_QK = 192, D_LAT = 512, D_ROW = 576, PAGE = 64;
constexpr int Q_LD = D_QK + 8;        // padded query row
constexpr int STAGES = 2;
constexpr int WARPS = 4;
// A stage holds one page: [4 blocks of 64 columns][64 rows][128 B] of K_g|V_g, then the k^R block,
// each block 128-byte swizzled as the tensor copy writes it (16-byte chunk c of row r sits at
// chunk c ^ (r % 8)), so the ldmatrix rows below are free of bank conflicts without padding.
constexpr uint32_t BLK = PAGE * 128;                  // one 64-column block of a page: 8 KiB
constexpr uint32_t KV_BYTES = 4 * BLK, KR_BYTES = BLK;
constexpr uint32_t STAGE = KV_BYTES + KR_BYTES;       // 40 KiB
constexpr uint32_t STAGE_BYTES = STAGES * STAGE;
// The final cross-warp reduction reuses the stage buffers (all copies have landed by then).
constexpr size_t red_bytes(int rt) { return sizeof(float) * WARPS * 16 * rt * (2 + D_V); }
static_assert(red_bytes(2) <= STAGE_BYTES, "reduction buffer must fit in the stage buffers");
constexpr size_t q_bytes(int rt) { return sizeof(__nv_bfloat16) * 16 * rt * Q_LD; }
constexpr size_t bar_off(int rt) { return STAGE_BYTES + ((q_bytes(rt) + 15) & ~(size_t)15); }
// + barriers (full and empty per stage) + room to align the window to 1024 bytes: 89 KiB with one
// row tile, 95 KiB with two, so two CTAs per SM either way.
constexpr size_t smem_bytes(int rt) { return 1024 + bar_off(rt) + 2 * STAGES * 8; }
constexpr uint64_t WAIT_NS = 2000000000ull;   // 2 s: no legitimate wait comes near this

// Byte offset of 16-byte chunk (row r, column c, c % 8 == 0) in a 128-byte-swizzled tile of
// 64-column blocks of PAGE rows.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
    return (uint32_t)((c >> 6) * BLK + r * 128 + ((((c >> 3) & 7) ^ (r & 7)) << 4));
}
__device__ __forceinline__ void tma_load_3d_own(uint32_t dst, const CUtensorMap *m, int x, int y, int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_own(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

struct GParams {
    const __nv_bfloat16 *q, *expanded, *latent;   // q: rotated queries [rows, H, 192]
    const int *page_table, *seq_lens;
    Plan plan;
    int max_pages, n_pages, s_q, H, hpw;          // s_q: queries per request (prefill: n_q)
    float scale_log2;
    float *part_o, *part_ml;   // [n_work * s_q, H, 128], [n_work * s_q, H, 2]
    int *err;
};

// Rows of the MMA tiles: CTA = (group g, item), row m = query m / 8 of head g*8 + m % 8; RT row
// tiles of 16 (RT = 1 for s_q <= 2, 2 for s_q = 3, 4).
//
// Tensor maps (bf16, 128-byte swizzle, 64-column inner blocks):
//   tm_kv  3-D over the expanded cache [n_pages G 64, 256]: (64, rows, 4), box (64, 64, 4): a page of K_g|V_g
//   tm_kr  3-D over the latent cache [n_pages 64, 576]: (64, rows, 9), box (64, 64, 1) at block 8: k^R
template <int RT>
__global__ void __launch_bounds__(WARPS * 32, 2)
    grouped_decode_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_kr, GParams p) {
    constexpr int ROWS = 16 * RT;
    step_begin();
    extern __shared__ __align__(16) uint8_t gsm_raw[];
    const uint32_t raw = smem_u32(gsm_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;                        // stages need 1024-byte alignment
    uint8_t *gsm = gsm_raw + (sbase - raw);
    __nv_bfloat16 *qs = reinterpret_cast<__nv_bfloat16 *>(gsm + STAGE_BYTES);   // [ROWS][Q_LD]
    const uint32_t bars = sbase + (uint32_t)bar_off(RT);                  // full[STAGES], empty[STAGES]
    float *red_ml = reinterpret_cast<float *>(gsm);                       // [WARPS][ROWS][2], after the loop
    float *red_o = red_ml + WARPS * ROWS * 2;                             // [WARPS][ROWS][128], after the loop

    // blockIdx.x = group (fastest), so the 16 groups of a chunk run together and the chunk's RoPE
    // keys, which every group reads, come from L2 after the first group's read.
    const int item = (int)(blockIdx.z * 65535 + blockIdx.y);   // grid.y <= 65535
    if (item >= p.plan.n_work) return;
    const WorkItem it = p.plan.items[item];
    const int g = (int)blockIdx.x;
    const int G = p.H / GH;
    auto row_query = [&](int m) { return m / GH; };
    auto row_head = [&](int m) { return g * GH + m % GH; };
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int b = it.row;                   // the plan of this path has one row per request
    const int L = p.seq_lens[b];
    // Every chunk ends at or before L, which the last query sees, so all its pages count.
    const int n_pg = ceil_div(it.t1 - it.t0, PAGE);
    const size_t part_base = (size_t)item * p.s_q;

    if (tid == 0) {
        for (int i = 0; i < 2 * STAGES; ++i) tc::mbar_init(bars + 8 * i, i < STAGES ? 1 : WARPS);
        tc::fence_mbar_init();
    }
    if (it.t1 <= it.t0) {   // only in a rejected plan
        for (int m = tid; m < ROWS; m += blockDim.x) {
            if (row_query(m) >= p.s_q) continue;
            const size_t r = part_base + row_query(m);
            p.part_ml[(r * p.H + row_head(m)) * 2] = -INFINITY;
            p.part_ml[(r * p.H + row_head(m)) * 2 + 1] = 0.f;
        }
        return;
    }
    // Queries, already rotated (q_rot = [q_nope | RoPE(q_rope, p_j)], one pass per call): s_q = 2
    // fills the 16 rows of one tile, s_q = 1 the first 8; rows past the last query are zero.
    for (int i = tid; i < ROWS * (D_QK / 8); i += blockDim.x) {   // 16-byte chunks
        const int m = i / (D_QK / 8), c = 8 * (i % (D_QK / 8));
        const int j = row_query(m), h = row_head(m);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (j < p.s_q) v = *reinterpret_cast<const uint4 *>(p.q + (((size_t)b * p.s_q + j) * p.H + h) * D_QK + c);
        *reinterpret_cast<uint4 *>(qs + m * Q_LD + c) = v;
    }
    __syncthreads();

    // Page i of the chunk into stage i % STAGES (thread 0).  An out-of-range page id reads as zeros
    // (a row coordinate past the end).  Rows past the chunk's end on its ragged last page hold
    // whatever the slots hold, NaN included; each warp zeroes its own rows of them before use.
    auto issue_page = [&](int i) {
        int pid = p.page_table[(size_t)b * p.max_pages + it.t0 / PAGE + i];
        if (pid < 0 || pid >= p.n_pages) {
            report(p.err, MLA_ERR_DEVICE_BOUNDS);
            pid = p.n_pages;
        }
        const int st = i % STAGES;
        const uint32_t full = bars + 8 * st, dst = sbase + STAGE * st;
        tc::mbar_arrive_expect_tx(full, STAGE);
        tma_load_3d_own(dst, &tm_kv, 0, (pid * G + g) * PAGE, 0, full);
        tma_load_3d_own(dst + KV_BYTES, &tm_kr, 0, pid * PAGE, 8, full);
    };

    // One tile's query A fragments stay in registers for the whole chunk (12 k-steps of 16 dims);
    // with two tiles they are reloaded from shared memory per k-step (registers hold O instead).
    uint32_t qa[RT == 1 ? 12 : 1][4];
    if constexpr (RT == 1) {
#pragma unroll
        for (int ks = 0; ks < 12; ++ks)
            ldmatrix_x4(qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3],
                        qs + ((lane % 8) + 8 * ((lane / 8) % 2)) * Q_LD + 16 * ks + 8 * (lane / 16));
    }
    auto q_frag = [&](int t, int ks, uint32_t *f) {
        ldmatrix_x4(f[0], f[1], f[2], f[3], qs + (16 * t + (lane % 8) + 8 * ((lane / 8) % 2)) * Q_LD + 16 * ks + 8 * (lane / 16));
    };

    const int gid = lane / 4, t4 = lane % 4;
    // Rows gid and gid + 8 of each tile's fragments: query index and last visible position.
    int lim[RT][2];
    float mrow[RT][2], lrow[RT][2];
    float o[RT][16][4];
#pragma unroll
    for (int t = 0; t < RT; ++t) {
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int j = row_query(16 * t + gid + 8 * h2);
            lim[t][h2] = j < p.s_q ? L - p.s_q + j : -1;
            mrow[t][h2] = -INFINITY;
            lrow[t][h2] = 0.f;
        }
#pragma unroll
        for (int n = 0; n < 16; ++n) o[t][n][0] = o[t][n][1] = o[t][n][2] = o[t][n][3] = 0.f;
    }

    if (tid == 0)
        for (int i = 0; i < STAGES && i < n_pg; ++i) issue_page(i);
    bool ok = true;
    for (int i = 0; i < n_pg; ++i) {
        const int st = i % STAGES;
        const uint32_t full = bars + 8 * st, empty = bars + 8 * (STAGES + st);
        ok = __all_sync(0xffffffffu, tc::mbar_wait(full, (uint32_t)(i / STAGES) & 1u, WAIT_NS));
        if (!ok) break;
        const uint8_t *tkv = gsm + STAGE * st, *tkr = tkv + KV_BYTES;
        const int valid = it.t1 - (it.t0 + PAGE * i);
        if (valid < 16 * warp + 16) {   // this warp's rows past the chunk's end: zero them
            for (int e = lane; e < 16 * 5 * 8; e += 32) {
                const int r = 16 * warp + e / 40, q = e % 40;   // 40 chunks of 16 B per row (4 KV blocks + k^R)
                if (r < valid) continue;
                uint8_t *d = const_cast<uint8_t *>(q < 32 ? tkv + (q / 8) * BLK : tkr) + r * 128 + 16 * (q % 8);
                *reinterpret_cast<uint4 *>(d) = make_uint4(0u, 0u, 0u, 0u);
            }
            __syncwarp();
        }
        // S [16 rows x 16 tokens] per tile = Q~ K~^T over 192 dims.
        float s[RT][2][4];
#pragma unroll
        for (int t = 0; t < RT; ++t)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) s[t][nt][0] = s[t][nt][1] = s[t][nt][2] = s[t][nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 12; ks += 2) {
            uint32_t qf[RT][2][4];
            if constexpr (RT > 1) {
#pragma unroll
                for (int t = 0; t < RT; ++t) {
                    q_frag(t, ks, qf[t][0]);
                    q_frag(t, ks + 1, qf[t][1]);
                }
            }
            // B fragments: rows = tokens, dims contiguous; x4 covers 2 k-steps of one n8 tile.
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t bf[4];
                const int tok = 16 * warp + 8 * nt + (lane % 8);
                const uint8_t *src = ks < 8 ? tkv + sw_off(tok, 16 * ks + 8 * (lane / 8))
                                            : tkr + sw_off(tok, 16 * (ks - 8) + 8 * (lane / 8));
                ldmatrix_x4(bf[0], bf[1], bf[2], bf[3], src);
#pragma unroll
                for (int t = 0; t < RT; ++t) {
                    const uint32_t *a0 = RT == 1 ? qa[RT == 1 ? ks : 0] : qf[t][0];
                    const uint32_t *a1 = RT == 1 ? qa[RT == 1 ? ks + 1 : 0] : qf[t][1];
                    mma_bf16(s[t][nt], a0, bf[0], bf[1]);
                    mma_bf16(s[t][nt], a1, bf[2], bf[3]);
                }
            }
        }
        // Mask, scale, online softmax per row (rows gid and gid + 8 of each tile; 4 tokens per row here).
        const int tok_base = it.t0 + PAGE * i + 16 * warp;
#pragma unroll
        for (int t = 0; t < RT; ++t) {
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tk = tok_base + 8 * nt + 2 * t4 + e;
                    const bool in = tk < it.t1;
                    s[t][nt][e] = (in && tk <= lim[t][0]) ? s[t][nt][e] * p.scale_log2 : -INFINITY;
                    s[t][nt][2 + e] = (in && tk <= lim[t][1]) ? s[t][nt][2 + e] * p.scale_log2 : -INFINITY;
                    mx0 = fmaxf(mx0, s[t][nt][e]);
                    mx1 = fmaxf(mx1, s[t][nt][2 + e]);
                }
#pragma unroll
            for (int off = 1; off <= 2; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float n0 = fmaxf(mrow[t][0], mx0), n1 = fmaxf(mrow[t][1], mx1);
            const float a0 = n0 == -INFINITY ? 1.f : exp2f(mrow[t][0] - n0);
            const float a1 = n1 == -INFINITY ? 1.f : exp2f(mrow[t][1] - n1);
            float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    s[t][nt][e] = n0 == -INFINITY ? 0.f : exp2f(s[t][nt][e] - n0);
                    s[t][nt][2 + e] = n1 == -INFINITY ? 0.f : exp2f(s[t][nt][2 + e] - n1);
                    sum0 += s[t][nt][e];
                    sum1 += s[t][nt][2 + e];
                }
            lrow[t][0] = lrow[t][0] * a0 + sum0;
            lrow[t][1] = lrow[t][1] * a1 + sum1;
            mrow[t][0] = n0;
            mrow[t][1] = n1;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                o[t][n][0] *= a0;
                o[t][n][1] *= a0;
                o[t][n][2] *= a1;
                o[t][n][3] *= a1;
            }
        }
        // P (accumulator layout of S) is the A fragment of P.V (rows x 16 tokens).
        uint32_t pa[RT][4];
#pragma unroll
        for (int t = 0; t < RT; ++t) {
            pa[t][0] = pack_bf16(s[t][0][0], s[t][0][1]);
            pa[t][1] = pack_bf16(s[t][0][2], s[t][0][3]);
            pa[t][2] = pack_bf16(s[t][1][0], s[t][1][1]);
            pa[t][3] = pack_bf16(s[t][1][2], s[t][1][3]);
        }
        // O [16 x 128] += P V per tile: V rows = tokens with v contiguous; .trans gives B fragments,
        // each shared by the tiles.
#pragma unroll
        for (int n = 0; n < 16; n += 2) {
            uint32_t vb[4];
            const uint8_t *src = tkv + sw_off(16 * warp + (lane % 8) + 8 * ((lane / 8) % 2), D_N + 8 * n + 8 * (lane / 16));
            ldmatrix_x4_trans(vb[0], vb[1], vb[2], vb[3], src);
#pragma unroll
            for (int t = 0; t < RT; ++t) {
                mma_bf16(o[t][n], pa[t], vb[0], vb[1]);
                mma_bf16(o[t][n + 1], pa[t], vb[2], vb[3]);
            }
        }
        // This warp is done with the stage; thread 0 refills it once all four are.  If that wait
        // runs out, warp 0 leaves the loop as a whole (the other warps' next waits then run out).
        __syncwarp();
        if (lane == 0) mbar_arrive_own(empty);
        bool refilled = true;
        if (tid == 0 && i + STAGES < n_pg) {
            refilled = tc::mbar_wait(empty, (uint32_t)(i / STAGES) & 1u, WAIT_NS);
            if (refilled) issue_page(i + STAGES);
        }
        if (warp == 0 && !__all_sync(0xffffffffu, refilled)) {
            ok = false;
            break;
        }
    }
    if (!ok) {   // a wait ran out: let copies in flight land before the memory is released
        if (lane == 0) report(p.err, MLA_ERR_TIMEOUT);
        const uint64_t t0 = tc::globaltimer();
        while (tc::globaltimer() - t0 < 200000ull) {
        }
    }
    __syncthreads();   // the stage buffers become the reduction buffer

    // Merge the four warps' partial softmaxes: row sums over the 4 threads of each row first.
#pragma unroll
    for (int t = 0; t < RT; ++t)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            float l = lrow[t][h2];
#pragma unroll
            for (int off = 1; off <= 2; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
            const int m = 16 * t + gid + 8 * h2;
            if (t4 == 0) {
                red_ml[(warp * ROWS + m) * 2] = mrow[t][h2];
                red_ml[(warp * ROWS + m) * 2 + 1] = l;
            }
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                red_o[(warp * ROWS + m) * D_V + 8 * n + 2 * t4] = o[t][n][2 * h2];
                red_o[(warp * ROWS + m) * D_V + 8 * n + 2 * t4 + 1] = o[t][n][2 * h2 + 1];
            }
        }
    __syncthreads();
    // ROWS rows x 128 columns; rows past the last query are padding.
    for (int i = tid; i < ROWS * D_V; i += blockDim.x) {
        const int m = i / D_V, c = i % D_V, j = row_query(m);
        if (j >= p.s_q) continue;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) M = fmaxf(M, red_ml[(w * ROWS + m) * 2]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            const float mw = red_ml[(w * ROWS + m) * 2];
            const float wt = mw == -INFINITY ? 0.f : exp2f(mw - M);
            num += wt * red_o[(w * ROWS + m) * D_V + c];
            den += wt * red_ml[(w * ROWS + m) * 2 + 1];
        }
        const size_t r = part_base + j;
        const int h = row_head(m);
        p.part_o[(r * p.H + h) * D_V + c] = num;   // relative to max M (log2 units)
        if (c == 0) {
            p.part_ml[(r * p.H + h) * 2] = M * 0.69314718055994531f;
            p.part_ml[(r * p.H + h) * 2 + 1] = den;
        }
    }
}


}  // namespace

bool grouped_tc_ok(const Dims &d, int s_q) {
    return s_q <= 4 && d.bf16 && d.hpw == GH && d.d_n == D_N && d.d_v == D_V && d.d_r == D_R && d.d_c == D_LAT && d.page == PAGE &&
           d.H % GH == 0;
}
int grouped_units(const Dims &d, int sms) { return std::max(1, 8 * 2 * sms / std::max(1, d.H / GH)); }
int grouped_token_granule() { return PAGE; }

static GParams grouped_params(const Dims &d, const void *q, const void *expanded, const void *latent,
                              const int *seq_lens, const int *page_table, const Plan &plan, int max_pages, int n_pages,
                              int s_q, float *part_o, float *part_ml, int *err) {
    GParams p;
    p.q = (const __nv_bfloat16 *)q;
    p.expanded = (const __nv_bfloat16 *)expanded;
    p.latent = (const __nv_bfloat16 *)latent;
    p.page_table = page_table;
    p.seq_lens = seq_lens;
    p.plan = plan;
    p.max_pages = max_pages;
    p.n_pages = n_pages;
    p.s_q = s_q;
    p.H = d.H;
    p.hpw = d.hpw;
    p.scale_log2 = d.scale * 1.4426950408889634f;
    p.part_o = part_o;
    p.part_ml = part_ml;
    p.err = err;
    return p;
}

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled g_encode_fn() {
    static const EncodeTiled fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiled>(ptr);
        return (EncodeTiled) nullptr;
    }();
    return fn;
}

// The two maps of a (expanded cache, latent cache) pair; a decode loop passes the same buffers
// every step, so recent encodings are reused (an encoding costs about a microsecond on the host).
static bool grouped_maps(const void *expanded, const void *latent, int n_pages, int G, CUtensorMap *tm_kv,
                         CUtensorMap *tm_kr) {
    struct Entry {
        const void *expanded, *latent;
        int n_pages, G, device;
        CUtensorMap kv, kr;
    };
    static std::mutex mu;
    static Entry cache[8];
    static int used = 0, next = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (cache[i].expanded == expanded && cache[i].latent == latent && cache[i].n_pages == n_pages &&
                cache[i].G == G && cache[i].device == dev) {
                *tm_kv = cache[i].kv;
                *tm_kr = cache[i].kr;
                return true;
            }
    }
    EncodeTiled fn = g_encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[3] = {1, 1, 1};
    const cuuint64_t dkv[3] = {64, (cuuint64_t)n_pages * G * PAGE, 4}, skv[2] = {256 * 2, 128};
    const cuuint32_t bkv[3] = {64, PAGE, 4};
    const cuuint64_t dkr[3] = {64, (cuuint64_t)n_pages * PAGE, 9}, skr[2] = {D_ROW * 2, 128};
    const cuuint32_t bkr[3] = {64, PAGE, 1};
    if (fn(tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(expanded), dkv, skv, bkv, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        fn(tm_kr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(latent), dkr, skr, bkr, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> lock(mu);
    cache[next] = Entry{expanded, latent, n_pages, G, dev, *tm_kv, *tm_kr};
    next = (next + 1) % 8;
    used = used < 8 ? used + 1 : 8;
    return true;
}

cudaError_t launch_grouped_decode(const Dims &d, const void *q, const void *expanded, const void *latent,
                                  const int *seq_lens, const int *page_table, const Plan &plan, int max_pages,
                                  int n_pages, int s_q, float *part_o, float *part_ml, int *err, cudaStream_t st) {
    if (plan.n_work == 0) return cudaSuccess;
    const GParams p = grouped_params(d, q, expanded, latent, seq_lens, page_table, plan, max_pages, n_pages, s_q,
                                     part_o, part_ml, err);
    CUtensorMap tm_kv, tm_kr;
    if (!grouped_maps(expanded, latent, n_pages, d.H / GH, &tm_kv, &tm_kr)) return cudaErrorInvalidValue;
    dim3 grid(d.H / GH, std::min(plan.n_work, 65535), ceil_div(plan.n_work, 65535));
    if (s_q <= 2) {
        cudaError_t e = raise_smem_limit((const void *)grouped_decode_kernel<1>, smem_bytes(1));
        if (e != cudaSuccess) return e;
        MLA_STEP_LAUNCH(grouped_decode_kernel<1>, dim3(grid), dim3(WARPS * 32), smem_bytes(1), st, tm_kv, tm_kr, p);
    } else {
        cudaError_t e = raise_smem_limit((const void *)grouped_decode_kernel<2>, smem_bytes(2));
        if (e != cudaSuccess) return e;
        MLA_STEP_LAUNCH(grouped_decode_kernel<2>, dim3(grid), dim3(WARPS * 32), smem_bytes(2), st, tm_kv, tm_kr, p);
    }
    return cudaGetLastError();
}

bool prefill_ok(const Dims &d) {
    return d.bf16 && d.d_n == D_N && d.d_v == D_V && d.d_r == D_R && d.d_c == D_LAT && d.page == PAGE;
}

cudaError_t launch_prefill_expanded(const Dims &d, const void *q_rot, const void *expanded, const void *latent,
                                    const int *seq_lens, const int *page_table, const Plan &plan, int max_pages,
                                    int n_pages, int n_q, float *part_o, float *part_ml, int *err, cudaStream_t st) {
    return launch_prefill_tc(d, q_rot, expanded, latent, seq_lens, page_table, plan, max_pages, n_pages, n_q, part_o,
                             part_ml, err, st);
}

}  // namespace mla
