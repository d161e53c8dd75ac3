// Head-expanded prefill on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "GQLA: Group-Query Latent Attention ..." abstract: MLA's head-expanded form attends with K and V
// up-projected per head (or per group of heads for GQLA weights); the prefill of a request's last
// n_q tokens is causal.  For query q of request b (position p_q = L_b - n_q + q) and head h of
// group g = h / heads_per_group:
//     s_t = scale * ([q_nope | RoPE(q_rope, p_q)] . [K_g,t | k^R_t]),  t <= p_q
//     o   = sum_t softmax(s)_t V_g,t
// Unlike decode this is compute-dense (one K/V tile serves 256 queries), so the kernel is laid
// out for the tensor pipe: a cluster of two CTAs runs every MMA as one cta_group::2 instruction
// with M = 256 queries (128 per CTA, one TMEM lane each), per 128-token step:
//   S  = Q K^T   M=256, N=128 tokens, K=192: CTA r supplies page r of the step as its half of B
//                (K_g from the expanded cache, k^R from the latent cache).
//   O += P V     M=256, N=128 (d_v), K=128 tokens: P is read from TMEM (each CTA's 128 rows, one
//                lane per query), CTA r supplies d_v columns [64 r, +64) of both pages.
// TMEM per CTA: two S buffers (128 columns each), O (128) and two P buffers (64 columns of bf16
// pairs each), so the softmax of step i waits for PV(i-2) before writing P, and for PV(i-1) only
// when it rescales O.
// Shared memory: Q (128 queries x 192, 48 KiB), a K ring (one page per slot: 16 KiB of K_g and
// 8 KiB of k^R) and a V ring (one step per slot: 2 pages x 64 d_v columns, 16 KiB).
// Warp roles (384 threads): warps 0-7 softmax and epilogue (two warps per TMEM lane quadrant: a
// query row's 128 scores of a step are split between the threads of lane L in warps w and w + 4),
// warp 8 K/Q producer, warp 9 QK^T issuer (leader CTA) and TMEM allocator, warp 10 V producer,
// warp 11 PV issuer (leader CTA).  Every wait is bounded; a timeout records MLA_ERR_TIMEOUT and the kernel
// still frees its tensor memory.
#include <cudaTypedefs.h>
#include <math.h>

#include "tc_decode.h"
#include "tc_ptx.cuh"

namespace mla {
namespace {

constexpr int PAGE = 64, STEP = 128, QT = 128;        // tokens per page / step, queries per CTA
constexpr int D_QK = 192, D_V = 128;
constexpr int NK = 4;                                 // K ring slots (one page each)
constexpr int NV = 2;                                 // V ring slots (one step each)
constexpr uint32_t QBLK = QT * 128;                   // one 64-column block of the 128 queries
constexpr uint32_t KBLK = PAGE * 128;                 // one 64-column block of a page
constexpr uint32_t Q_BYTES = 3 * QBLK;                // 48 KiB
constexpr uint32_t KSLOT = 3 * KBLK;                  // K_g (2 blocks) + k^R (1 block): 24 KiB
constexpr uint32_t VSLOT = 2 * KBLK;                  // 2 pages x 64 d_v columns: 16 KiB
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_V = OFF_K + NK * KSLOT;
constexpr uint32_t OFF_BAR = OFF_V + NV * VSLOT;
enum {
    B_KFULL = 0,
    B_KEMPTY = B_KFULL + NK,
    B_VFULL = B_KEMPTY + NK,
    B_VEMPTY = B_VFULL + NV,
    B_QFULL = B_VEMPTY + NV,
    B_SFULL,
    B_SFREE = B_SFULL + 2,
    B_PFULL = B_SFREE + 2,
    B_PVDONE = B_PFULL + 2,
    B_COUNT = B_PVDONE + 2
};
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + B_COUNT * 8;
constexpr uint32_t OFF_FLAG = OFF_TMEMPTR + 8;
constexpr uint32_t OFF_RED = (OFF_FLAG + 8 + 15) & ~15u;   // float[2 buffers][2 halves][128 rows]
constexpr uint32_t SMEM_USED = OFF_RED + 2 * 2 * 128 * 4;
constexpr uint32_t SMEM_ALLOC = SMEM_USED;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

constexpr uint32_t TM_S = 0;      // two S buffers of 128 columns
constexpr uint32_t TM_O = 256;    // O: 128 columns
constexpr uint32_t TM_P = 384;    // P: two buffers of 64 columns of bf16 pairs
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_QK = tc::idesc_bf16_f32(256, 128, false, false);
constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(256, 128, false, true);
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr int SM_WARPS = 8;
constexpr int W_KPROD = 8, W_QK = 9, W_VPROD = 10, W_PV = 11;
constexpr int THREADS = 384;
constexpr float RESCALE_LOG2 = 8.f;

struct PfParams {
    int n_q, H, hpw, G, max_pages, n_pages, n_items;
    const int *page_table, *seq_lens;
    const WorkItem *items;
    float scale_log2;
    float *part_o, *part_ml;   // [n_items * n_q, H, 128], [n_items * n_q, H, 2]
    int *err;
};

struct Ctx {
    uint32_t base;
    uint8_t *sbase;
    uint32_t rank;
    volatile int *abort_flag;
    __device__ uint32_t bar(int i) const { return base + OFF_BAR + 8u * i; }
    __device__ uint32_t lead_bar(int i) const { return tc::map_to_rank(bar(i), 0); }
    __device__ uint32_t kslot(int i) const { return base + OFF_K + KSLOT * i; }
    __device__ uint32_t vslot(int i) const { return base + OFF_V + VSLOT * i; }
};

__device__ __forceinline__ bool wait_or_abort(const Ctx &c, uint32_t bar, uint32_t parity, int *err) {
    if (*c.abort_flag) return false;
    if (tc::mbar_wait(bar, parity, WAIT_NS)) return true;
    report(err, MLA_ERR_TIMEOUT);
    *c.abort_flag = 1;
    return false;
}
__device__ __forceinline__ bool warp_wait(const Ctx &c, uint32_t bar, uint32_t parity, int *err) {
    const bool ok = wait_or_abort(c, bar, parity, err);
    return __all_sync(0xffffffffu, ok);
}

// The unit of a cluster: head, work item (one request, tokens [t0, t1)), 256-query tile.
struct Unit {
    int head, g, b, t0, t1, q0, L, n_steps;
};
__device__ __forceinline__ Unit unit_of(const PfParams &p) {
    Unit u;
    u.head = blockIdx.z % p.H;
    const int item = blockIdx.z / p.H;
    const WorkItem it = p.items[item];
    u.g = u.head / p.hpw;
    u.b = it.row;
    u.t0 = it.t0;
    u.L = p.seq_lens[u.b];
    u.q0 = 2 * QT * blockIdx.y;
    const int q_last = min(p.n_q, u.q0 + 2 * QT) - 1;
    u.t1 = min(it.t1, u.L - p.n_q + q_last + 1);     // tokens after the tile's last query are masked
    u.n_steps = u.t1 > u.t0 ? (u.t1 - u.t0 + STEP - 1) / STEP : 0;
    return u;
}

// Row of page index pi of request b in a page-granular view; past t_end or out of range:
// a row past the end (TMA fills zeros).
__device__ __forceinline__ int page_id(const PfParams &p, int b, int pi, int t_end, bool *ok) {
    *ok = false;
    if (pi * PAGE >= t_end) return -1;
    const int pid = p.page_table[(size_t)b * p.max_pages + pi];
    if (pid < 0 || pid >= p.n_pages) {
        report(p.err, MLA_ERR_DEVICE_BOUNDS);
        return -1;
    }
    *ok = true;
    return pid;
}

// --------------------------------------------------------------------------- producers
// Tensor maps (128-byte swizzle, 64-column inner blocks):
//   tm_q   4-D over q_rot [B n_q, H, 192]: (64, H, B n_q, 3), box (64, 1, 128, 3): 128 queries of one head
//   tm_ek  3-D over the expanded cache [n_pages G 64, 256]: (64, rows, 4), box (64, 64, 2): K_g of a page
//   tm_ev  same view, box (64, 64, 1): one 64-column block of V_g (block 2 + rank)
//   tm_kr  3-D over the latent cache [n_pages 64, 576]: (64, rows, 9), box (64, 64, 1) at block 8: k^R
__device__ void run_k_producer(const Ctx &c, const PfParams &p, const Unit &u, const CUtensorMap *tm_q,
                               const CUtensorMap *tm_ek, const CUtensorMap *tm_kr) {
    if (c.rank == 0) tc::mbar_arrive_expect_tx(c.bar(B_QFULL), 2u * Q_BYTES);
    tc::tma_load_4d_pair(c.base + OFF_Q, tm_q, 0, u.head, u.b * p.n_q + u.q0 + QT * (int)c.rank, 0,
                         c.lead_bar(B_QFULL));
    const int past_e = p.n_pages * p.G * PAGE, past_l = p.n_pages * PAGE;
    for (int i = 0; i < u.n_steps; ++i) {
        const int slot = i % NK;
        bool ok;
        const int pid = page_id(p, u.b, (u.t0 + STEP * i) / PAGE + (int)c.rank, u.t1, &ok);
        if (!wait_or_abort(c, c.bar(B_KEMPTY + slot), ((uint32_t)(i / NK) & 1u) ^ 1u, p.err)) return;
        if (c.rank == 0) tc::mbar_arrive_expect_tx(c.bar(B_KFULL + slot), 2u * KSLOT);
        tc::tma_load_3d_pair(c.kslot(slot), tm_ek, 0, ok ? (pid * p.G + u.g) * PAGE : past_e, 0,
                             c.lead_bar(B_KFULL + slot));
        tc::tma_load_3d_pair(c.kslot(slot) + 2 * KBLK, tm_kr, 0, ok ? pid * PAGE : past_l, 8,
                             c.lead_bar(B_KFULL + slot));
    }
}

// V producer: per step, d_v columns [64 rank, +64) of both pages of the step.
__device__ void run_v_producer(const Ctx &c, const PfParams &p, const Unit &u, const CUtensorMap *tm_ev) {
    const int past_e = p.n_pages * p.G * PAGE;
    for (int i = 0; i < u.n_steps; ++i) {
        const int slot = i % NV;
        if (!wait_or_abort(c, c.bar(B_VEMPTY + slot), ((uint32_t)(i / NV) & 1u) ^ 1u, p.err)) return;
        if (c.rank == 0) tc::mbar_arrive_expect_tx(c.bar(B_VFULL + slot), 2u * VSLOT);
        for (int pg = 0; pg < 2; ++pg) {
            bool ok;
            const int pid = page_id(p, u.b, (u.t0 + STEP * i) / PAGE + pg, u.t1, &ok);
            tc::tma_load_3d_pair(c.vslot(slot) + pg * KBLK, tm_ev, 0, ok ? (pid * p.G + u.g) * PAGE : past_e,
                                 2 + (int)c.rank, c.lead_bar(B_VFULL + slot));
        }
    }
}

// --------------------------------------------------------------------------- MMA issuers
__device__ void run_qk_issuer(const Ctx &c, const PfParams &p, const Unit &u, uint32_t tmem) {
    const uint64_t qdesc = tc::sdesc_sw128(c.base + OFF_Q, 16, 1024);
    const uint64_t kdesc = tc::sdesc_sw128(c.base + OFF_K, 16, 1024);
    if (!wait_or_abort(c, c.bar(B_QFULL), 0u, p.err)) return;
    tc::fence_after_sync();
    for (int i = 0; i < u.n_steps; ++i) {
        const int sb = i & 1, slot = i % NK;
        if (i >= 2 && !wait_or_abort(c, c.bar(B_SFREE + sb), (uint32_t)((i - 2) >> 1) & 1u, p.err)) return;
        if (!wait_or_abort(c, c.bar(B_KFULL + slot), (uint32_t)(i / NK) & 1u, p.err)) return;
        tc::fence_after_sync();
        const uint32_t d = tmem + TM_S + 128 * sb;
#pragma unroll
        for (int kb = 0; kb < 3; ++kb)
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) {
                const uint64_t a = tc::sdesc_add(qdesc, kb * QBLK + 32 * w4);
                const uint64_t b = tc::sdesc_add(kdesc, slot * KSLOT + kb * KBLK + 32 * w4);
                if (kb == 0 && w4 == 0)
                    tc::mma_pair_bf16_k<false>(d, a, b, IDESC_QK);
                else
                    tc::mma_pair_bf16_k<true>(d, a, b, IDESC_QK);
            }
        tc::commit_pair(c.bar(B_KEMPTY + slot), 0x3);
        tc::commit_pair(c.bar(B_SFULL + sb), 0x3);
    }
}

__device__ void run_pv_issuer(const Ctx &c, const PfParams &p, const Unit &u, uint32_t tmem) {
    const uint64_t vdesc = tc::sdesc_sw128(c.base + OFF_V, KBLK, 1024);
    for (int i = 0; i < u.n_steps; ++i) {
        const int slot = i % NV;
        if (!wait_or_abort(c, c.bar(B_PFULL + (i & 1)), (uint32_t)(i >> 1) & 1u, p.err)) return;
        if (!wait_or_abort(c, c.bar(B_VFULL + slot), (uint32_t)(i / NV) & 1u, p.err)) return;
        tc::fence_after_sync();
#pragma unroll
        for (int k = 0; k < 8; ++k) {   // 16 tokens per instruction: page k / 4, rows 16 (k % 4)
            const uint32_t a = tmem + TM_P + 64 * (i & 1) + 8 * k;
            const uint64_t b = tc::sdesc_add(vdesc, slot * VSLOT + (k / 4) * KBLK + 2048 * (k % 4));
            if (i == 0 && k == 0)
                tc::mma_pair_ts_bf16_k<false>(tmem + TM_O, a, b, IDESC_PV);
            else
                tc::mma_pair_ts_bf16_k<true>(tmem + TM_O, a, b, IDESC_PV);
        }
        tc::commit_pair(c.bar(B_VEMPTY + slot), 0x3);
        tc::commit_pair(c.bar(B_PVDONE + (i & 1)), 0x3);
    }
}

// --------------------------------------------------------------------------- softmax + epilogue
// Warps w and w + 4 read TMEM lane quadrant w % 4: thread L = 32 (w % 4) + lane of warp w owns
// query q0 + 128 rank + L and tokens [64 (w / 4), +64) of each step.  The two threads of a row swap
// their maxima through shared memory (one 64-thread named barrier per warp pair) and keep their
// own sums, added at the end.  O is rescaled lazily, only when a row max grows by more than 2^8
// (exact after the final division by l); both warps of a pair see the same rows and maxima, so
// their warp-uniform rescale decisions agree.
__device__ void run_softmax(const Ctx &c, const PfParams &p, const Unit &u, uint32_t tmem) {
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int quad = warp & 3, half = warp >> 2;
    const int L = 32 * quad + lane;
    const int q = u.q0 + QT * (int)c.rank + L;
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    const int p_q = min(u.L - p.n_q + q, u.L - 1);   // last visible token (padding rows: the last token)
    float *red = reinterpret_cast<float *>(c.sbase + OFF_RED);   // [2][2][128]
    auto partner = [&](int buf, float v) {
        red[256 * buf + 128 * half + L] = v;
        tc::named_sync(1 + quad, 64);
        return red[256 * buf + 128 * (half ^ 1) + L];
    };
    float m_run = -INFINITY, l_run = 0.f;
    for (int i = 0; i < u.n_steps; ++i) {
        const int sb = i & 1;
        warp_wait(c, c.bar(B_SFULL + sb), (uint32_t)(i >> 1) & 1u, p.err);
        tc::fence_after_sync();
        float s[64];
        tc::tmem_ld64(tmem + TM_S + 128 * sb + 64 * half + lane_addr, s);
        tc::tmem_wait_ld();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_cluster(c.lead_bar(B_SFREE + sb));
        const int nvis = min(STEP, max(0, p_q - (u.t0 + STEP * i) + 1)) - 64 * half;   // visible prefix of my tokens
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
            s[j] = j < nvis ? s[j] * p.scale_log2 : -INFINITY;
            mx = fmaxf(mx, s[j]);
        }
        mx = fmaxf(mx, partner(i & 1, mx));
        const bool any = __any_sync(0xffffffffu, i > 0 && mx > m_run + RESCALE_LOG2);
        // PV(i-1) must be complete before O is rescaled and before P is overwritten.
        // P is double-buffered: P(i) needs PV(i-2) complete; a rescale of O needs PV(i-1).
        if (any && i >= 1)
            warp_wait(c, c.bar(B_PVDONE + ((i - 1) & 1)), (uint32_t)((i - 1) >> 1) & 1u, p.err);
        else if (i >= 2)
            warp_wait(c, c.bar(B_PVDONE + (i & 1)), (uint32_t)((i - 2) >> 1) & 1u, p.err);
        tc::fence_after_sync();
        if (i == 0) {
            m_run = mx;
        } else if (any) {
            const float m_new = fmaxf(m_run, mx);
            const float alpha = m_new == -INFINITY ? 1.f : tc::ex2(m_run - m_new);
            float v[64];
            tc::tmem_ld64(tmem + TM_O + 64 * half + lane_addr, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] *= alpha;
            tc::tmem_st64(tmem + TM_O + 64 * half + lane_addr, v);
            tc::tmem_wait_st();
            l_run *= alpha;
            m_run = m_new;
        }
        uint32_t pk[32];
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const float a = 2 * j < nvis ? tc::ex2(s[2 * j] - m_run) : 0.f;
            const float b2 = 2 * j + 1 < nvis ? tc::ex2(s[2 * j + 1] - m_run) : 0.f;
            sum += a + b2;
            __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b2);
            pk[j] = *reinterpret_cast<uint32_t *>(&h2);
        }
        l_run += sum;
        const uint32_t pcol = tmem + TM_P + 64 * (i & 1) + 32 * half + lane_addr;
        tc::tmem_st16(pcol, pk);
        tc::tmem_st16(pcol + 16, pk + 16);
        tc::tmem_wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_cluster(c.lead_bar(B_PFULL + (i & 1)));
    }
    // Epilogue: the unnormalised O (relative to m, log2 units), m in natural-log units, and l.
    if (u.n_steps > 0) {
        warp_wait(c, c.bar(B_PVDONE + ((u.n_steps - 1) & 1)), (uint32_t)((u.n_steps - 1) >> 1) & 1u, p.err);
        tc::fence_after_sync();
    }
    const float l_tot = l_run + partner(u.n_steps & 1, l_run);
    const bool real = q < p.n_q;
    const size_t r = ((size_t)(blockIdx.z / p.H) * p.n_q + q) * p.H + u.head;
    float v[64];
    if (u.n_steps > 0) {
        tc::tmem_ld64(tmem + TM_O + 64 * half + lane_addr, v);
        tc::tmem_wait_ld();
    } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = 0.f;
    }
    if (real) {
        float *dst = p.part_o + r * D_V + 64 * half;
#pragma unroll
        for (int j = 0; j < 8; ++j) tc::st_global_v8(dst + 8 * j, v + 8 * j);
        if (half == 0) {
            p.part_ml[r * 2] = m_run * 0.69314718055994531f;
            p.part_ml[r * 2 + 1] = l_tot;
        }
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ek,
                      const __grid_constant__ CUtensorMap tm_ev, const __grid_constant__ CUtensorMap tm_kr,
                      PfParams p) {
    step_begin();
    extern __shared__ uint8_t smem_raw[];
    Ctx c;
    const uint32_t raw = tc::smem_addr(smem_raw);
    c.base = (raw + 1023u) & ~1023u;
    c.sbase = smem_raw + (c.base - raw);
    c.rank = tc::cluster_rank();
    c.abort_flag = reinterpret_cast<volatile int *>(c.sbase + OFF_FLAG);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    uint32_t dyn_bytes;
    asm("mov.u32 %0, %dynamic_smem_size;" : "=r"(dyn_bytes));
    if (c.base - raw + SMEM_USED > dyn_bytes) {   // uniform for the whole cluster: nothing ran yet
        if (threadIdx.x == 0) report(p.err, MLA_ERR_UNSUPPORTED);
        return;
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < NK; ++i) {
            tc::mbar_init(c.bar(B_KFULL + i), 1);
            tc::mbar_init(c.bar(B_KEMPTY + i), 1);
        }
        for (int i = 0; i < NV; ++i) {
            tc::mbar_init(c.bar(B_VFULL + i), 1);
            tc::mbar_init(c.bar(B_VEMPTY + i), 1);
        }
        tc::mbar_init(c.bar(B_QFULL), 1);
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(c.bar(B_SFULL + i), 1);
            tc::mbar_init(c.bar(B_SFREE + i), 2 * SM_WARPS);
            tc::mbar_init(c.bar(B_PVDONE + i), 1);
        }
        tc::mbar_init(c.bar(B_PFULL), 2 * SM_WARPS);
        tc::mbar_init(c.bar(B_PFULL + 1), 2 * SM_WARPS);
        *c.abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == W_KPROD && lane == 0) {
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_ek);
        tc::prefetch_tmap(&tm_kr);
    }
    if (warp == W_VPROD && lane == 0) tc::prefetch_tmap(&tm_ev);
    if (warp == W_QK) tc::tmem_alloc_pair(c.base + OFF_TMEMPTR, TM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::cluster_sync();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(c.sbase + OFF_TMEMPTR);

    const Unit u = unit_of(p);   // the same for both CTAs of the pair
    if (warp < SM_WARPS) {
        run_softmax(c, p, u, tmem);
    } else if (warp == W_KPROD) {
        if (lane == 0) run_k_producer(c, p, u, &tm_q, &tm_ek, &tm_kr);
    } else if (warp == W_VPROD) {
        if (lane == 0) run_v_producer(c, p, u, &tm_ev);
    } else if (warp == W_QK) {
        if (c.rank == 0 && lane == 0) run_qk_issuer(c, p, u, tmem);
    } else if (warp == W_PV) {
        if (c.rank == 0 && lane == 0) run_pv_issuer(c, p, u, tmem);
    }
    if (*c.abort_flag) {   // a wait ran out: let copies in flight land before the memory is released
        const uint64_t t0 = tc::globaltimer();
        while (tc::globaltimer() - t0 < 200000ull) {
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::cluster_sync();
    if (warp == W_QK) {
        tc::fence_after_sync();
        tc::tmem_dealloc_pair(tmem, TM_COLS);
        tc::tmem_relinquish_pair();
    }
}

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once; the initialisation of a function-local static is thread-safe.
EncodeTiled pf_encode_fn() {
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

// bf16 map with 128-byte swizzle; dims[0] = 64 columns (one block), strides in bytes for dims 1..rank-1.
bool pf_encode(CUtensorMap *m, const void *ptr, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
               const cuuint32_t *box) {
    EncodeTiled fn = pf_encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_prefill_tc(const Dims &d, const void *q_rot, const void *expanded, const void *latent,
                              const int *seq_lens, const int *page_table, const Plan &plan, int max_pages,
                              int n_pages, int n_q, float *part_o, float *part_ml, int *err, cudaStream_t st) {
    if (plan.n_work == 0) return cudaSuccess;
    const int G = d.H / d.hpw;
    const int n_tiles = (n_q + 2 * QT - 1) / (2 * QT);
    if ((long long)d.H * plan.n_work > 65535 || n_tiles > 65535) return cudaErrorInvalidValue;
    CUtensorMap tm_q, tm_ek, tm_ev, tm_kr;
    {
        const cuuint64_t dims[4] = {64, (cuuint64_t)d.H, (cuuint64_t)plan.rows * n_q, 3};
        const cuuint64_t strides[3] = {D_QK * 2, (cuuint64_t)d.H * D_QK * 2, 128};
        const cuuint32_t box[4] = {64, 1, QT, 3};
        if (!pf_encode(&tm_q, q_rot, 4, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[3] = {64, (cuuint64_t)n_pages * G * PAGE, 4};
        const cuuint64_t strides[2] = {256 * 2, 128};
        const cuuint32_t box_k[3] = {64, PAGE, 2}, box_v[3] = {64, PAGE, 1};
        if (!pf_encode(&tm_ek, expanded, 3, dims, strides, box_k) || !pf_encode(&tm_ev, expanded, 3, dims, strides, box_v))
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[3] = {64, (cuuint64_t)n_pages * PAGE, 9};
        const cuuint64_t strides[2] = {576 * 2, 128};
        const cuuint32_t box[3] = {64, PAGE, 1};
        if (!pf_encode(&tm_kr, latent, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    PfParams p;
    p.n_q = n_q;
    p.H = d.H;
    p.hpw = d.hpw;
    p.G = G;
    p.max_pages = max_pages;
    p.n_pages = n_pages;
    p.n_items = plan.n_work;
    p.page_table = page_table;
    p.seq_lens = seq_lens;
    p.items = plan.items;
    p.scale_log2 = d.scale * 1.4426950408889634f;
    p.part_o = part_o;
    p.part_ml = part_ml;
    p.err = err;
    constexpr uint32_t ALLOC = SMEM_ALLOC + 1024;   // room to align the window to 1024 bytes
    cudaError_t e = raise_smem_limit((const void *)prefill_tc_kernel, ALLOC);
    if (e != cudaSuccess) return e;
    MLA_STEP_LAUNCH(prefill_tc_kernel, dim3(2, n_tiles, d.H * plan.n_work), dim3(THREADS), ALLOC, st, tm_q, tm_ek,
                    tm_ev, tm_kr, p);
    return cudaGetLastError();
}

}  // namespace mla
