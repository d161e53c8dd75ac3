// Absorbed MLA split decode on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// The MQA-absorb path ("GQLA: Group-Query Latent Attention ..." abstract; "How to upgrade GQA
// models to MLA ...", stage "Decompression Multiplex"): every head's absorbed query q_abs =
// [W_UK^T q_nope | RoPE(q_rope)] (576 wide) scores the cached rows [c | k^R] of its request,
// and the probabilities weight the latents c (512 wide).  Per work item (one query row and a
// chunk of its tokens) this kernel produces the unnormalised partial O = sum_t e^{s_t - m} c_t
// with its running max m and sum l; combine.cu merges chunks and applies W_UV.
//
// Shape of the computation: all 128 heads of a row share each latent tile, so heads are the
// MMA M dimension.  O (128 heads x 512 fp32) alone would fill one SM's whole tensor memory, so
// a cluster of two CTAs runs every MMA as one cta_group::2 instruction with M = 128: CTA r owns
// heads [64r, 64r+64), whose accumulators the hardware folds into 128 TMEM lanes x N/2 columns.
// Per 128-token step:
//   S  = Q K^T   M=128 heads, N=128 tokens, K=576: CTA r supplies the 64 tokens of page r of
//                the step (B is split along N between the pair); S lands in 64 TMEM columns.
//   O += P C     M=128 heads, N=256 latent columns (two instructions), K=128 tokens: CTA r
//                supplies latent columns [256c + 128r, +128) of both pages.
// Every CTA loads only its own tiles, from its own GPU's HBM, with plain (non-multicast) TMA.
//
// Warp roles (192 threads per CTA): warps 0-3 softmax + epilogue (thread i owns TMEM lane i:
// head i % 64, token half i / 64), warp 4 TMA producer, warp 5 MMA issuer (leader CTA only) and
// TMEM allocator.  Pipelines: a 7-slot ring of 16 KiB shared-memory slots for K and V tiles,
// two S buffers in TMEM and two P buffers in shared memory, so QK^T of step g+1 runs while the
// softmax of step g works.  The softmax rescales O only when a row max grows by more than 2^8
// (exact after the final division by l).  Every wait is bounded: on timeout the kernel records
// MLA_ERR_TIMEOUT, stops issuing work, and still frees its tensor memory before returning.
#include <cudaTypedefs.h>
#include <math.h>

#include "tc_decode.h"
#include "tc_ptx.cuh"

namespace mla {
namespace {

constexpr int H = 128, DROW = 576, PAGE = 64, STEP = 128;
constexpr int NSLOT = 7;
constexpr uint32_t BOX = 8192;                 // 64 rows x 128 bytes
constexpr uint32_t SLOT = 2 * BOX;
constexpr uint32_t Q_BYTES = 9 * BOX;          // 64 heads x 576 bf16
constexpr uint32_t P_BYTES = 2 * BOX;          // 64 heads x 128 tokens bf16
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_P = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_SLOT = OFF_P + 2 * P_BYTES;
constexpr uint32_t OFF_BAR = OFF_SLOT + NSLOT * SLOT;
enum {
    B_FULL = 0,
    B_EMPTY = B_FULL + NSLOT,
    B_QFULL = B_EMPTY + NSLOT,
    B_QEMPTY,
    B_SFULL,
    B_SFREE = B_SFULL + 2,
    B_PFULL = B_SFREE + 2,
    B_PVDONE = B_PFULL + 2,
    B_OFREE = B_PVDONE + 2,
    B_RED,                       // two barriers for the cross-warp exchange of row max / sum
    B_COUNT = B_RED + 2
};
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + B_COUNT * 8;
constexpr uint32_t OFF_FLAG = OFF_TMEMPTR + 8;
constexpr uint32_t OFF_RED = (OFF_FLAG + 8 + 15) & ~15u;   // float[2][128]
constexpr uint32_t SMEM_USED = OFF_RED + 2 * 128 * 4;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;            // slack for 1024-byte alignment

constexpr uint32_t TM_S = 0;      // two S buffers of 64 columns
constexpr uint32_t TM_O = 128;    // O: 256 columns
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_QK = tc::idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(128, 256, false, true);
constexpr uint64_t WAIT_NS = 2000000000ull;   // 2 s: no legitimate wait comes near this
constexpr int SOFTMAX_WARPS = 4;
constexpr float RESCALE_LOG2 = 8.f;           // rescale O when a row max grows by more than 2^8

struct TcParams {
    Plan plan;
    const int *page_table;
    int max_pages, n_pages, s_q;
    float scale_log2;  // softmax scale * log2(e)
    float *part_o;     // [n_work, H, 512]
    float *part_ml;    // [n_work, H, 2]: max (natural-log units), sum
    int *err;
};

struct Ctx {
    uint32_t base;      // 1024-aligned shared-memory base
    uint8_t *sbase;     // generic pointer to the same
    uint32_t rank;      // 0 = leader of the pair
    volatile int *abort_flag;
    __device__ uint32_t bar(int i) const { return base + OFF_BAR + 8u * i; }
    __device__ uint32_t lead_bar(int i) const { return tc::map_to_rank(bar(i), 0); }
    __device__ uint32_t slot(int s) const { return base + OFF_SLOT + SLOT * s; }
};

__device__ __forceinline__ bool wait_or_abort(const Ctx &c, uint32_t bar, uint32_t parity, int *err) {
    if (*c.abort_flag) return false;
    if (tc::mbar_wait(bar, parity, WAIT_NS)) return true;
    report(err, MLA_ERR_TIMEOUT);
    *c.abort_flag = 1;
    return false;
}

// Same, with one verdict for the whole warp (the tcgen05 loads that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(const Ctx &c, uint32_t bar, uint32_t parity, int *err) {
    const bool ok = wait_or_abort(c, bar, parity, err);
    return __all_sync(0xffffffffu, ok);
}

// Row coordinate (in the [n_pages*64, 576] view) of page index `pi` of request `b`; pages with
// no token before `t_end` and out-of-range page ids read as zeros (coordinate past the end).
__device__ __forceinline__ int page_row(const TcParams &p, int b, int pi, int t_end) {
    if (pi * PAGE >= t_end) return p.n_pages * PAGE;
    const int pid = p.page_table[(size_t)b * p.max_pages + pi];
    if (pid < 0 || pid >= p.n_pages) {
        report(p.err, MLA_ERR_DEVICE_BOUNDS);
        return p.n_pages * PAGE;
    }
    return pid * PAGE;
}

// --------------------------------------------------------------------------- producer
__device__ void run_producer(const Ctx &c, const TcParams &p, const CUtensorMap *tm_q, const CUtensorMap *tm_kv,
                             int pair, int n_pairs) {
    uint32_t u = 0;
    int item_n = 0;
    auto fill = [&](int nbox, int x0, int x1, int y) -> bool {
        const int s = (int)(u % NSLOT);
        const uint32_t use = u / NSLOT;
        if (!wait_or_abort(c, c.bar(B_EMPTY + s), (use & 1u) ^ 1u, p.err)) return false;
        const uint32_t full = c.lead_bar(B_FULL + s);
        if (c.rank == 0) tc::mbar_arrive_expect_tx(c.bar(B_FULL + s), 2u * nbox * BOX);
        tc::tma_load_2d_pair(c.slot(s), tm_kv, x0, y, full);
        if (nbox == 2) tc::tma_load_2d_pair(c.slot(s) + BOX, tm_kv, x1, y, full);
        ++u;
        return true;
    };
    auto fill_v = [&](int b, int t_step, int t_end) -> bool {
        for (int ch = 0; ch < 2; ++ch)
            for (int pg = 0; pg < 2; ++pg) {
                const int y = page_row(p, b, t_step / PAGE + pg, t_end);
                const int x = 256 * ch + 128 * (int)c.rank;
                if (!fill(2, x, x + 64, y)) return false;
            }
        return true;
    };
    for (int k = pair; k < p.plan.n_work; k += n_pairs) {
        const WorkItem it = p.plan.items[k];
        if (it.t1 <= it.t0) continue;   // only in a rejected plan, and then for every item
        const int b = it.row / p.s_q;
        const int n_steps = ceil_div(it.t1 - it.t0, STEP);
        if (item_n > 0 && !wait_or_abort(c, c.bar(B_QEMPTY), (uint32_t)(item_n - 1) & 1u, p.err)) return;
        ++item_n;
        if (c.rank == 0) tc::mbar_arrive_expect_tx(c.bar(B_QFULL), 2u * Q_BYTES);
        const uint32_t qfull = c.lead_bar(B_QFULL);
        const int qrow = it.row * H + 64 * (int)c.rank;
        for (int cb = 0; cb < 9; ++cb) tc::tma_load_2d_pair(c.base + OFF_Q + cb * BOX, tm_q, 64 * cb, qrow, qfull);
        for (int i = 0; i <= n_steps; ++i) {
            if (i < n_steps) {
                const int t_step = it.t0 + STEP * i;
                const int y = page_row(p, b, t_step / PAGE + (int)c.rank, it.t1);
                for (int j = 0; j < 4; ++j)
                    if (!fill(2, 128 * j, 128 * j + 64, y)) return;
                if (!fill(1, 512, 0, y)) return;
            }
            if (i >= 1 && !fill_v(b, it.t0 + STEP * (i - 1), it.t1)) return;
        }
    }
}

// --------------------------------------------------------------------------- MMA issuer
__device__ void run_mma(const Ctx &c, const TcParams &p, uint32_t tmem, int pair, int n_pairs) {
    uint32_t u = 0;
    int g = 0, item_n = 0;
    auto take = [&](int &s) -> bool {
        s = (int)(u % NSLOT);
        const uint32_t use = u / NSLOT;
        ++u;
        if (!wait_or_abort(c, c.bar(B_FULL + s), use & 1u, p.err)) return false;
        tc::fence_after_sync();
        return true;
    };
    auto pv = [&](int gj, bool first) -> bool {
        const int pb = gj & 1;
        if (!wait_or_abort(c, c.bar(B_PFULL + pb), (uint32_t)(gj >> 1) & 1u, p.err)) return false;
        if (first && item_n > 0 && !wait_or_abort(c, c.bar(B_OFREE), (uint32_t)(item_n - 1) & 1u, p.err))
            return false;
        tc::fence_after_sync();
        const uint32_t pbase = c.base + OFF_P + P_BYTES * pb;
        for (int ch = 0; ch < 2; ++ch)
            for (int pg = 0; pg < 2; ++pg) {
                int s;
                if (!take(s)) return false;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const uint64_t a = tc::sdesc_sw128(pbase + pg * BOX + 32 * k4, 16, 1024);
                    const uint64_t bd = tc::sdesc_sw128(c.slot(s) + 2048 * k4, BOX, 1024);
                    tc::mma_pair_bf16(tmem + TM_O + 128 * ch, a, bd, IDESC_PV, (first && pg == 0 && k4 == 0) ? 0u : 1u);
                }
                tc::commit_pair(c.bar(B_EMPTY + s), 0x3);
            }
        tc::commit_pair(c.bar(B_PVDONE + pb), 0x3);
        return true;
    };
    for (int k = pair; k < p.plan.n_work; k += n_pairs, ++item_n) {
        const WorkItem it = p.plan.items[k];
        if (it.t1 <= it.t0) {
            --item_n;   // only in a rejected plan, and then for every item
            continue;
        }
        const int n_steps = ceil_div(it.t1 - it.t0, STEP);
        if (!wait_or_abort(c, c.bar(B_QFULL), (uint32_t)item_n & 1u, p.err)) return;
        tc::fence_after_sync();
        for (int i = 0; i < n_steps; ++i, ++g) {
            const int sb = g & 1;
            if (g >= 2 && !wait_or_abort(c, c.bar(B_SFREE + sb), (uint32_t)((g - 2) >> 1) & 1u, p.err)) return;
            tc::fence_after_sync();
            const uint32_t d = tmem + TM_S + 64 * sb;
            for (int j = 0; j < 5; ++j) {
                int s;
                if (!take(s)) return;
                const int nk = j < 4 ? 8 : 4;
                for (int kk = 0; kk < nk; ++kk) {
                    const int cb = 2 * j + kk / 4, w4 = kk % 4;
                    const uint64_t a = tc::sdesc_sw128(c.base + OFF_Q + cb * BOX + 32 * w4, 16, 1024);
                    const uint64_t bd = tc::sdesc_sw128(c.slot(s) + (kk / 4) * BOX + 32 * w4, 16, 1024);
                    tc::mma_pair_bf16(d, a, bd, IDESC_QK, (j | kk) ? 1u : 0u);
                }
                tc::commit_pair(c.bar(B_EMPTY + s), 0x3);
            }
            if (i == n_steps - 1) tc::commit_pair(c.bar(B_QEMPTY), 0x3);
            tc::commit_pair(c.bar(B_SFULL + sb), 0x3);
            if (i >= 1 && !pv(g - 1, i == 1)) return;
        }
        if (!pv(g - 1, n_steps == 1)) return;
    }
}

// --------------------------------------------------------------------------- softmax + epilogue
__device__ void run_softmax(const Ctx &c, const TcParams &p, uint32_t tmem, int pair, int n_pairs) {
    const int L = threadIdx.x;  // TMEM lane, 0..127
    const int warp = L / 32, lane = L % 32;
    const int hl = L & 63, hsel = L >> 6;
    const int head = 64 * (int)c.rank + hl;
    const uint32_t lane_addr = (uint32_t)(32 * warp) << 16;
    float *red = reinterpret_cast<float *>(c.sbase + OFF_RED);
    int g = 0, item_n = 0;
    bool ok = true;
    // The two threads of a head (TMEM lanes L and L ^ 64) sit in different warps; they swap a
    // value through shared memory behind a 128-arrival mbarrier (bounded wait, no bar.sync that
    // could outlive an aborted warp).  Exchange x uses buffer x % 2.
    uint32_t xchg = 0;
    auto exchange = [&](float v, float &other) -> bool {
        const int bi = (int)(xchg & 1u);
        red[128 * bi + L] = v;
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(c.bar(B_RED + bi)) : "memory");
        const bool w = warp_wait(c, c.bar(B_RED + bi), (xchg >> 1) & 1u, p.err);
        if (w) other = red[128 * bi + (L ^ 64)];
        ++xchg;
        return w;
    };
    for (int k = pair; k < p.plan.n_work && ok; k += n_pairs, ++item_n) {
        const WorkItem it = p.plan.items[k];
        if (it.t1 <= it.t0) {
            if (hsel == 0) {
                p.part_ml[((size_t)k * H + head) * 2] = -INFINITY;
                p.part_ml[((size_t)k * H + head) * 2 + 1] = 0.f;
            }
            continue;
        }
        const int n_steps = ceil_div(it.t1 - it.t0, STEP);
        float m_run = -INFINITY, l_run = 0.f;
        for (int i = 0; i < n_steps; ++i, ++g) {
            const int sb = g & 1;
            if (!(ok = warp_wait(c, c.bar(B_SFULL + sb), (uint32_t)(g >> 1) & 1u, p.err))) break;
            tc::fence_after_sync();
            float s[64];
            tc::tmem_ld64(tmem + TM_S + 64 * sb + lane_addr, s);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive_cluster(c.lead_bar(B_SFREE + sb));

            const int tok0 = it.t0 + STEP * i + 64 * hsel;
            const int nvalid = min(64, max(0, it.t1 - tok0));
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                s[j] = j < nvalid ? s[j] * p.scale_log2 : -INFINITY;
                mx = fmaxf(mx, s[j]);
            }
            float mo = -INFINITY;
            if (!(ok = exchange(mx, mo))) break;
            const float mt = fmaxf(mx, mo);
            if (i == 0 || mt > m_run + RESCALE_LOG2) {
                if (i > 0) {
                    const float alpha = exp2f(m_run - mt);
                    // O holds steps < g: wait until PV(g-1) has landed, then rescale in place.
                    if (!(ok = warp_wait(c, c.bar(B_PVDONE + ((g - 1) & 1)), (uint32_t)((g - 1) >> 1) & 1u, p.err)))
                        break;
                    tc::fence_after_sync();
#pragma unroll 1
                    for (int q = 0; q < 4; ++q) {
                        float v[64];
                        tc::tmem_ld64(tmem + TM_O + 64 * q + lane_addr, v);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 64; ++j) v[j] *= alpha;
                        tc::tmem_st64(tmem + TM_O + 64 * q + lane_addr, v);
                    }
                    tc::tmem_wait_st();
                    l_run *= alpha;
                }
                m_run = mt;
            }
            float sum = 0.f;
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float a = exp2f(s[2 * j] - m_run), b2 = exp2f(s[2 * j + 1] - m_run);
                sum += a + b2;
                __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b2);
                pk[j] = *reinterpret_cast<uint32_t *>(&h2);
            }
            l_run += sum;
            // P buffer g%2 was read by PV(g-2).
            if (g >= 2 && !(ok = warp_wait(c, c.bar(B_PVDONE + sb), (uint32_t)((g - 2) >> 1) & 1u, p.err))) break;
            uint8_t *prow = c.sbase + OFF_P + P_BYTES * sb + BOX * hsel + 128 * hl;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 v = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
                *reinterpret_cast<uint4 *>(prow + ((ch ^ (hl & 7)) << 4)) = v;
            }
            tc::fence_proxy_async_smem();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive_cluster(c.lead_bar(B_PFULL + sb));
        }
        if (!ok) break;
        // Epilogue: the last PV of this item has landed; write the partial O, m, l.
        if (!(ok = warp_wait(c, c.bar(B_PVDONE + ((g - 1) & 1)), (uint32_t)((g - 1) >> 1) & 1u, p.err))) break;
        tc::fence_after_sync();
        float lo = 0.f;
        if (!(ok = exchange(l_run, lo))) break;
        const float l_tot = l_run + lo;
        float *dst = p.part_o + ((size_t)k * H + head) * 512;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
            float v[64];
            tc::tmem_ld64(tmem + TM_O + 64 * q + lane_addr, v);
            tc::tmem_wait_ld();
            const int d0 = 256 * (q / 2) + 128 * hsel + 64 * (q % 2);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                *reinterpret_cast<float4 *>(dst + d0 + 4 * j) = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_cluster(c.lead_bar(B_OFREE));
        if (hsel == 0) {
            p.part_ml[((size_t)k * H + head) * 2] = m_run * 0.69314718055994531f;
            p.part_ml[((size_t)k * H + head) * 2 + 1] = l_tot;
        }
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    tc_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv, TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    Ctx c;
    const uint32_t raw = tc::smem_addr(smem_raw);
    c.base = (raw + 1023u) & ~1023u;
    c.sbase = smem_raw + (c.base - raw);
    c.rank = tc::cluster_rank();
    c.abort_flag = reinterpret_cast<volatile int *>(c.sbase + OFF_FLAG);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSLOT; ++i) {
            tc::mbar_init(c.bar(B_FULL + i), 1);
            tc::mbar_init(c.bar(B_EMPTY + i), 1);
        }
        tc::mbar_init(c.bar(B_QFULL), 1);
        tc::mbar_init(c.bar(B_QEMPTY), 1);
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(c.bar(B_SFULL + i), 1);
            tc::mbar_init(c.bar(B_SFREE + i), 2 * SOFTMAX_WARPS);
            tc::mbar_init(c.bar(B_PFULL + i), 2 * SOFTMAX_WARPS);
            tc::mbar_init(c.bar(B_PVDONE + i), 1);
        }
        tc::mbar_init(c.bar(B_OFREE), 2 * SOFTMAX_WARPS);
        tc::mbar_init(c.bar(B_RED), 32 * SOFTMAX_WARPS);
        tc::mbar_init(c.bar(B_RED + 1), 32 * SOFTMAX_WARPS);
        *c.abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 4 && lane == 0) {
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_kv);
    }
    if (warp == 5) tc::tmem_alloc_pair(c.base + OFF_TMEMPTR, TM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::cluster_sync();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(c.sbase + OFF_TMEMPTR);

    const int pair = blockIdx.x / 2, n_pairs = gridDim.x / 2;
    if (warp == 4) {
        if (lane == 0) run_producer(c, p, &tm_q, &tm_kv, pair, n_pairs);
    } else if (warp == 5) {
        if (c.rank == 0 && lane == 0) run_mma(c, p, tmem, pair, n_pairs);
    } else {
        run_softmax(c, p, tmem, pair, n_pairs);
    }

    if (*c.abort_flag) {
        // A wait ran out: give any tile copies still in flight time to land before the
        // shared memory they target is released.
        const uint64_t t0 = tc::globaltimer();
        while (tc::globaltimer() - t0 < 200000ull) {
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::cluster_sync();
    if (warp == 5) {
        tc::fence_after_sync();
        tc::tmem_dealloc_pair(tmem, TM_COLS);
        tc::tmem_relinquish_pair();
    }
}

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(ptr);
    }
    return fn;
}

// [rows, 576] bf16 row-major, 64x64 boxes with 128-byte swizzle (zero fill past the end).
bool encode_rows576(CUtensorMap *m, const void *ptr, uint64_t rows) {
    EncodeTiled fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {DROW, rows};
    cuuint64_t strides[1] = {DROW * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_available() { return true; }
int tc_units(int sms) { return sms / 2; }
int tc_token_granule() { return STEP; }

cudaError_t launch_tc_decode(const Dims &d, const void *q_abs, const void *latent, const int *page_table,
                             const Plan &plan, int max_pages, int n_pages, int s_q, float *part_o, float *part_ml,
                             int *err, int sms, cudaStream_t st) {
    if (plan.n_work == 0) return cudaSuccess;
    CUtensorMap tm_q, tm_kv;
    if (!encode_rows576(&tm_q, q_abs, (uint64_t)plan.rows * H) ||
        !encode_rows576(&tm_kv, latent, (uint64_t)n_pages * PAGE))
        return cudaErrorInvalidValue;
    TcParams p;
    p.plan = plan;
    p.page_table = page_table;
    p.max_pages = max_pages;
    p.n_pages = n_pages;
    p.s_q = s_q;
    p.scale_log2 = d.scale * 1.4426950408889634f;
    p.part_o = part_o;
    p.part_ml = part_ml;
    p.err = err;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(tc_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int units = std::max(1, std::min(plan.n_work, std::max(1, sms / 2)));
    tc_decode_kernel<<<2 * units, 192, SMEM_ALLOC, st>>>(tm_q, tm_kv, p);
    return cudaGetLastError();
}

}  // namespace mla
