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
//                supplies latent columns [256c + 128r, +128) of both pages; P (the A operand)
//                comes from tensor memory.
// Every CTA loads only its own tiles, from its own GPU's HBM, with plain (non-multicast) TMA.
//
// Warp roles (416 threads per CTA): warps 0-7 softmax + epilogue (two warps per TMEM lane
// quadrant, each taking half of a lane's columns), warp 8 producer of K slots 0-1, warp 12
// producer of Q and of K slot 2, warp 10 producer of the V ring, warp 9 QK^T issuer (leader CTA
// only) and TMEM allocator, warp 11 PV issuer (leader CTA only).  The tensor copies one thread
// issues are processed one after another (measured: ~250 ns per copy from L2 and ~600 ns per
// 24 KiB box from HBM under full load, whatever the ring depth), so the K ring, which streams
// the cache from HBM, has two issuing threads.  Shared memory holds Q
// (72 KiB), a K ring of three 24 KiB slots (one step: the CTA's page x 576 columns as three
// groups of three 64-column blocks), a V ring of two 32 KiB slots (one per page of the step:
// this CTA's 256 latent columns) and a 16 KiB buffer through which the softmax threads of lanes
// L and L ^ 64 swap halves of P.  Tiles move as few, large TMA boxes (3-D and 4-D views of the
// [rows, 576] cache whose inner dimensions are 64-column blocks): a single thread issuing one
// small box at a time cannot reach HBM bandwidth, while one instruction per 24-32 KiB can.  K
// and V have separate rings and producers, so a V slot held until its PV never stalls the next
// step's K loads.  (An L2 prefetch of the pages ahead of their K loads was measured slower at
// every distance from one to five steps and is not used.)  Tensor memory holds two S buffers
// (QK^T of step g+1 runs while the softmax of step g works), O, and two P buffers (the softmax
// of step g+1 writes P while PV of step g still reads the other one).  The softmax rescales O
// only when a row max grows by more than 2^8 (exact after the final division by l), and only
// then waits for the previous PV.  Every wait is bounded: on timeout the kernel records
// MLA_ERR_TIMEOUT, stops issuing work, and still frees its tensor memory before returning.
#include <cudaTypedefs.h>
#include <math.h>

#include "tc_decode.h"
#include "tc_ptx.cuh"

namespace mla {
namespace {

constexpr int H = 128, DROW = 576, PAGE = 64, STEP = 128;
constexpr int NK = 3;                          // K ring: three slots of three 64-column blocks
constexpr int NV = 2;                          // V ring: one slot per page of the step
constexpr uint32_t BOX = 8192;                 // one 64-column block of 64 rows: 64 x 128 bytes
constexpr uint32_t KSLOT = 3 * BOX;
constexpr uint32_t VSLOT = 4 * BOX;            // [chunk 0..1][block pair][64 rows][64 cols]
constexpr uint32_t Q_BYTES = 9 * BOX;          // 64 heads x 576 bf16
constexpr uint32_t X_BYTES = 2 * BOX;          // P exchange: [2 column halves][128 lanes][64 B]
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_X = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_K = OFF_X + X_BYTES;
constexpr uint32_t OFF_V = OFF_K + NK * KSLOT;
constexpr uint32_t OFF_BAR = OFF_V + NV * VSLOT;
enum {
    B_KFULL = 0,
    B_KEMPTY = B_KFULL + NK,
    B_VFULL = B_KEMPTY + NK,
    B_VEMPTY = B_VFULL + NV,
    B_QFULL = B_VEMPTY + NV,
    B_QEMPTY,
    B_SFULL,
    B_SFREE = B_SFULL + 2,
    B_PFULL = B_SFREE + 2,
    B_PVDONE = B_PFULL + 2,
    B_OFREE = B_PVDONE + 2,
    B_VLOCAL,   // this CTA's own copy of a ragged page's V tile (count 1, local)
    B_VTAIL,    // both CTAs zeroed the stale rows of a ragged page's V tiles (count 2, leader)
    B_COUNT
};
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + B_COUNT * 8;
constexpr uint32_t OFF_FLAG = OFF_TMEMPTR + 8;
constexpr uint32_t OFF_RED = (OFF_FLAG + 8 + 15) & ~15u;   // float[2][2][128]
constexpr uint32_t SMEM_USED = OFF_RED + 2 * 256 * 4;
// The dynamic shared memory window starts 1024-byte aligned on sm_100 (the kernel checks this
// and reports MLA_ERR_UNSUPPORTED instead of running if it ever does not).
constexpr uint32_t SMEM_ALLOC = SMEM_USED;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

constexpr uint32_t TM_S = 0;      // two S buffers of 64 columns
constexpr uint32_t TM_O = 128;    // O: 256 columns
constexpr uint32_t TM_P = 384;    // two P buffers of 64 columns (bf16 pairs, duplicated lane halves)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_QK = tc::idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(128, 256, false, true);
constexpr uint64_t WAIT_NS = 2000000000ull;   // 2 s: no legitimate wait comes near this
constexpr int SOFTMAX_WARPS = 8;
constexpr int SM_THREADS = 32 * SOFTMAX_WARPS;
constexpr int W_KPROD = SOFTMAX_WARPS, W_MMA = SOFTMAX_WARPS + 1, W_VPROD = SOFTMAX_WARPS + 2,
              W_PV = SOFTMAX_WARPS + 3, W_KPROD2 = SOFTMAX_WARPS + 4;
constexpr int K_SPLIT = 2;   // K slots [0, K_SPLIT) come from W_KPROD, the rest from W_KPROD2
constexpr int THREADS = 32 * (SOFTMAX_WARPS + 5);
constexpr float RESCALE_LOG2 = 8.f;           // rescale O when a row max grows by more than 2^8

struct TcParams {
    Plan plan;
    const int *page_table;
    int max_pages, n_pages, s_q;
    float scale_log2;  // softmax scale * log2(e)
    float *part_o;     // [n_work, 64, H, 8]: column octet-major (see the epilogue)
    float *part_ml;    // [n_work, H, 2]: max (natural-log units), sum
    int *err;
    uint64_t wait_ns;  // limit of every barrier wait (WAIT_NS unless a test shortens it)
    int withhold;      // test hook: the PV issuer skips the completion signal of this step (-1: none)
};

struct Ctx {
    uint32_t base;      // 1024-aligned shared-memory base
    uint8_t *sbase;     // generic pointer to the same
    uint32_t rank;      // 0 = leader of the pair
    volatile int *abort_flag;
    uint64_t wait_ns;
    __device__ uint32_t bar(int i) const { return base + OFF_BAR + 8u * i; }
    __device__ uint32_t lead_bar(int i) const { return tc::map_to_rank(bar(i), 0); }
    __device__ uint32_t kslot(int i) const { return base + OFF_K + KSLOT * i; }
    __device__ uint32_t vslot(int i) const { return base + OFF_V + VSLOT * i; }
};

// `spin`: the MMA issuers wait without suspending, so they resume as soon as a phase completes.
template <bool spin = false>
__device__ __forceinline__ bool wait_or_abort(const Ctx &c, uint32_t bar, uint32_t parity, int *err) {
    if (*c.abort_flag) return false;
    if (spin ? tc::mbar_wait_spin(bar, parity, c.wait_ns) : tc::mbar_wait(bar, parity, c.wait_ns)) return true;
    report(err, MLA_ERR_TIMEOUT);
    *c.abort_flag = 1;
    return false;
}

// Same, with one answer for the whole warp (the tcgen05 loads that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(const Ctx &c, uint32_t bar, uint32_t parity, int *err) {
    const bool ok = wait_or_abort(c, bar, parity, err);
    return __all_sync(0xffffffffu, ok);
}

// Work item of round `rnd` of cluster pair `pair`: the plan's positions are dealt in snake order
// (pairs 0..U-1, then U-1..0, ...), and the plan lists full-length chunks first and the rows'
// shorter last chunks longest first, so every pair gets a similar number of steps even when the
// rows' lengths differ widely.  Every role of both CTAs walks the same sequence.  -1: no more.
__device__ __forceinline__ int item_of_round(const Plan &pl, int pair, int n_pairs, int rnd) {
    const int j = rnd * n_pairs + ((rnd & 1) ? n_pairs - 1 - pair : pair);
    if (j >= pl.n_work) return -1;
    return pl.order ? pl.order[j] : j;
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

// --------------------------------------------------------------------------- producers
// Tensor maps (all over row-major [rows, 576] bf16 with 128-byte swizzle; the inner dimension is
// one 64-column block, the row dimension has stride 1152 B, the block dimension stride 128 B):
//   tm_q    3-D (64, rows, 9),    box (64, 64, 9): 64 rows x 576 columns, block-major in smem
//   tm_k    3-D (64, rows, 9),    box (64, 64, 3): 64 rows x three blocks
//   tm_v    4-D (64, rows, 4, 2), strides (1152, 128, 512), box (64, 64, 2, 2): for chunk c in
//           {0, 1} the two blocks starting at 4c + 2 rank, i.e. columns [256c + 128 rank, +128)
// K producers: per work item the CTA's 64 query heads (Q, the producer of the last slot, so Q
// and slot 0 of an item's first step load in parallel), then per 128-token step K slots [j0, j1)
// of the CTA's own page of the step.  Steps are numbered across
// items (g), so every slot's phase is g's parity.
__device__ void run_k_producer(const Ctx &c, const TcParams &p, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                               int pair, int n_pairs, int j0, int j1) {
    int g = 0, item_n = 0;
    for (int rnd = 0, k; (k = item_of_round(p.plan, pair, n_pairs, rnd)) >= 0; ++rnd) {
        const WorkItem it = p.plan.items[k];
        if (it.t1 <= it.t0) continue;   // only in a rejected plan, and then for every item
        const int b = it.row / p.s_q;
        const int n_steps = ceil_div(it.t1 - it.t0, STEP);
        auto own_row = [&](int i) { return page_row(p, b, (it.t0 + STEP * i) / PAGE + (int)c.rank, it.t1); };
        if (j1 == NK) {
            if (item_n > 0 && !wait_or_abort(c, c.bar(B_QEMPTY), (uint32_t)(item_n - 1) & 1u, p.err)) return;
            if (c.rank == 0) tc::mbar_arrive_expect_tx(c.bar(B_QFULL), 2u * Q_BYTES);
            tc::tma_load_3d_pair(c.base + OFF_Q, tm_q, 0, it.row * H + 64 * (int)c.rank, 0, c.lead_bar(B_QFULL));
        }
        ++item_n;
        for (int i = 0; i < n_steps; ++i, ++g) {
            const int y = own_row(i);
            for (int j = j0; j < j1; ++j) {
                if (!wait_or_abort(c, c.bar(B_KEMPTY + j), ((uint32_t)g & 1u) ^ 1u, p.err)) return;
                if (c.rank == 0) tc::mbar_arrive_expect_tx(c.bar(B_KFULL + j), 2u * KSLOT);
                tc::tma_load_3d_pair(c.kslot(j), tm_k, 0, y, 3 * j, c.lead_bar(B_KFULL + j));
            }
        }
    }
}

// Rows of the page starting at token `row0` that lie inside the item, when that is a proper part
// of the page (the request's ragged last page): its other rows are slots past the request's length,
// which may hold anything, NaN included.  0 otherwise.
__device__ __forceinline__ int ragged_rows(const WorkItem &it, int row0) {
    const int valid = it.t1 - row0;
    return (valid > 0 && valid < PAGE) ? valid : 0;
}

// V producer (lane 0): per step and page pg of the step, this CTA's 256 latent columns of that
// page.  A ragged page is copied with this CTA's own barrier instead, and its stale rows are
// cleared by run_v_tail.
__device__ void run_v_producer(const Ctx &c, const TcParams &p, const CUtensorMap *tm_v, int pair, int n_pairs) {
    int g = 0;
    for (int rnd = 0, k; (k = item_of_round(p.plan, pair, n_pairs, rnd)) >= 0; ++rnd) {
        const WorkItem it = p.plan.items[k];
        if (it.t1 <= it.t0) continue;
        const int b = it.row / p.s_q;
        const int n_steps = ceil_div(it.t1 - it.t0, STEP);
        for (int i = 0; i < n_steps; ++i, ++g) {
            const int t_step = it.t0 + STEP * i;
            for (int pg = 0; pg < NV; ++pg) {
                const int y = page_row(p, b, t_step / PAGE + pg, it.t1);
                if (!wait_or_abort(c, c.bar(B_VEMPTY + pg), ((uint32_t)g & 1u) ^ 1u, p.err)) return;
                if (!ragged_rows(it, t_step + PAGE * pg)) {
                    if (c.rank == 0) tc::mbar_arrive_expect_tx(c.bar(B_VFULL + pg), 2u * VSLOT);
                    tc::tma_load_4d_pair(c.vslot(pg), tm_v, 0, y, 2 * (int)c.rank, 0, c.lead_bar(B_VFULL + pg));
                } else {
                    // This phase of VFULL carries no bytes; the PV issuer waits on the tail barrier.
                    if (c.rank == 0) tc::mbar_arrive_expect_tx(c.bar(B_VFULL + pg), 0u);
                    tc::mbar_arrive_expect_tx(c.bar(B_VLOCAL), VSLOT);
                    tc::tma_load_4d(c.vslot(pg), tm_v, 0, y, 2 * (int)c.rank, 0, c.bar(B_VLOCAL));
                }
            }
        }
    }
}

// Lanes 1-31 of the V producer's warp: for each ragged page, once its copy has landed, zero the
// rows past the item's end in this CTA's V tile (their probabilities are zero, but 0 x NaN is
// NaN in P.V), make the stores visible to the tensor core and report on the leader's tail
// barrier.  Zeroing whole 128-byte rows of each 64-column block needs no knowledge of the
// 128-byte swizzle.
__device__ void run_v_tail(const Ctx &c, const TcParams &p, int pair, int n_pairs) {
    const int lane = threadIdx.x % 32;   // 1..31
    int nt = 0;                          // ragged pages so far (phase of B_VLOCAL)
    for (int rnd = 0, k; (k = item_of_round(p.plan, pair, n_pairs, rnd)) >= 0; ++rnd) {
        const WorkItem it = p.plan.items[k];
        if (it.t1 <= it.t0) continue;
        const int n_steps = ceil_div(it.t1 - it.t0, STEP);
        for (int i = n_steps - 1; i < n_steps; ++i)   // only an item's last step can hold its end
            for (int pg = 0; pg < NV; ++pg) {
                const int valid = ragged_rows(it, it.t0 + STEP * i + PAGE * pg);
                if (!valid) continue;
                const bool ok = wait_or_abort(c, c.bar(B_VLOCAL), (uint32_t)(nt++) & 1u, p.err);
                if (!__all_sync(0xfffffffeu, ok)) return;
                uint8_t *tile = c.sbase + OFF_V + VSLOT * pg;      // four [64 rows][128 B] blocks
                const int n16 = (PAGE - valid) * 8;                // 16-byte pieces past the end, per block
                for (int e = lane - 1; e < 4 * n16; e += 31) {
                    const int blk = e / n16, r = e % n16;
                    *reinterpret_cast<uint4 *>(tile + BOX * blk + 128 * valid + 16 * r) = make_uint4(0u, 0u, 0u, 0u);
                }
                tc::fence_proxy_async_smem();
                __syncwarp(0xfffffffeu);
                if (lane == 1) tc::mbar_arrive_cluster(c.lead_bar(B_VTAIL));
            }
    }
}

// --------------------------------------------------------------------------- MMA issuers
// Two threads of the leader CTA issue the pair's MMAs, each waiting only on its own inputs, so
// the in-order tensor pipe always has whichever of QK^T(g + 1) and PV(g) is ready.  A
// tcgen05.commit tracks the MMAs of the thread that issues it, so each issuer's barriers
// report exactly its own work.
__device__ void run_qk_issuer(const Ctx &c, const TcParams &p, uint32_t tmem, int pair, int n_pairs) {
    int g = 0, item_n = 0;
    const uint64_t qdesc = tc::sdesc_sw128(c.base + OFF_Q, 16, 1024);
    const uint64_t kdesc = tc::sdesc_sw128(c.base + OFF_K, 16, 1024);
    for (int rnd = 0, k; (k = item_of_round(p.plan, pair, n_pairs, rnd)) >= 0; ++rnd) {
        const WorkItem it = p.plan.items[k];
        if (it.t1 <= it.t0) continue;   // only in a rejected plan, and then for every item
        const int n_steps = ceil_div(it.t1 - it.t0, STEP);
        if (!wait_or_abort<true>(c, c.bar(B_QFULL), (uint32_t)item_n & 1u, p.err)) return;
        tc::fence_after_sync();
        for (int i = 0; i < n_steps; ++i, ++g) {
            const int sb = g & 1;
            if (g >= 2 && !wait_or_abort<true>(c, c.bar(B_SFREE + sb), (uint32_t)((g - 2) >> 1) & 1u, p.err)) return;
            tc::fence_after_sync();
            const uint32_t d = tmem + TM_S + 64 * sb;
#pragma unroll
            for (int j = 0; j < NK; ++j) {
                if (!wait_or_abort<true>(c, c.bar(B_KFULL + j), (uint32_t)g & 1u, p.err)) return;
                tc::fence_after_sync();
#pragma unroll
                for (int q3 = 0; q3 < 3; ++q3)
#pragma unroll
                    for (int w4 = 0; w4 < 4; ++w4) {
                        const int cb = 3 * j + q3;
                        const uint64_t a = tc::sdesc_add(qdesc, cb * BOX + 32 * w4);
                        const uint64_t bd = tc::sdesc_add(kdesc, j * KSLOT + q3 * BOX + 32 * w4);
                        if (cb == 0 && w4 == 0)
                            tc::mma_pair_bf16_k<false>(d, a, bd, IDESC_QK);
                        else
                            tc::mma_pair_bf16_k<true>(d, a, bd, IDESC_QK);
                    }
                tc::commit_pair(c.bar(B_KEMPTY + j), 0x3);
            }
            if (i == n_steps - 1) tc::commit_pair(c.bar(B_QEMPTY), 0x3);
            tc::commit_pair(c.bar(B_SFULL + sb), 0x3);
        }
        ++item_n;
    }
}

__device__ void run_pv_issuer(const Ctx &c, const TcParams &p, uint32_t tmem, int pair, int n_pairs) {
    int g = 0, item_n = 0, nt = 0;   // nt: ragged pages so far (phase of B_VTAIL)
    const uint64_t vdesc = tc::sdesc_sw128(c.base + OFF_V, BOX, 1024);
    const uint32_t o_tmem = tmem + TM_O;
    for (int rnd = 0, k; (k = item_of_round(p.plan, pair, n_pairs, rnd)) >= 0; ++rnd) {
        const WorkItem it = p.plan.items[k];
        if (it.t1 <= it.t0) continue;
        const int n_steps = ceil_div(it.t1 - it.t0, STEP);
        for (int i = 0; i < n_steps; ++i, ++g) {
            if (!wait_or_abort<true>(c, c.bar(B_PFULL + (g & 1)), (uint32_t)(g >> 1) & 1u, p.err)) return;
            // The first PV of an item overwrites O: the previous item's epilogue must be done with it.
            if (i == 0 && item_n > 0 && !wait_or_abort<true>(c, c.bar(B_OFREE), (uint32_t)(item_n - 1) & 1u, p.err)) return;
            tc::fence_after_sync();
            const uint32_t p_tmem = tmem + TM_P + 64 * (g & 1);
#pragma unroll
            for (int pg = 0; pg < NV; ++pg) {
                if (!wait_or_abort<true>(c, c.bar(B_VFULL + pg), (uint32_t)g & 1u, p.err)) return;
                if (ragged_rows(it, it.t0 + STEP * i + PAGE * pg) &&
                    !wait_or_abort<true>(c, c.bar(B_VTAIL), (uint32_t)(nt++) & 1u, p.err))
                    return;
                tc::fence_after_sync();
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const uint32_t a = p_tmem + 32 * pg + 8 * k4;   // 16 tokens = 8 columns of bf16 pairs
                        const uint64_t bd = tc::sdesc_add(vdesc, pg * VSLOT + 2 * BOX * ch + 2048 * k4);
                        if (pg == 0 && k4 == 0 && i == 0)
                            tc::mma_pair_ts_bf16_k<false>(o_tmem + 128 * ch, a, bd, IDESC_PV);
                        else
                            tc::mma_pair_ts_bf16_k<true>(o_tmem + 128 * ch, a, bd, IDESC_PV);
                    }
                tc::commit_pair(c.bar(B_VEMPTY + pg), 0x3);
            }
            if (g != p.withhold) tc::commit_pair(c.bar(B_PVDONE + (g & 1)), 0x3);
        }
        ++item_n;
    }
}

// --------------------------------------------------------------------------- softmax + epilogue
// Eight warps, two per TMEM lane quadrant: warp w reads lanes [32 (w % 4), +32) and column half
// w / 4 of each S buffer, so thread t owns lane L = 32 (w % 4) + lane, i.e. head L % 64, tokens
// 64 (L / 64) + 32 (w / 4) + [0, 32) of the step.  The four threads of a head swap their maxima
// and, at the end, their sums through shared memory behind a named barrier.  Control flow does
// not depend on data or on a wait's outcome: a wait that runs out only records the error, so
// every thread always reaches every named barrier.
__device__ void run_softmax(const Ctx &c, const TcParams &p, uint32_t tmem, int pair, int n_pairs) {
    const int t = threadIdx.x;                     // 0..255
    const int warp = t / 32, lane = t % 32;
    const int quad = warp & 3, half = warp >> 2;
    const int L = 32 * quad + lane;                // TMEM lane
    const int hl = L & 63, hsel = L >> 6;
    const int head = 64 * (int)c.rank + hl;
    const uint32_t lane_addr = (uint32_t)(32 * quad) << 16;
    float *red = reinterpret_cast<float *>(c.sbase + OFF_RED);   // [2][2][128]
    auto others = [&](int buf, float v, float &a, float &b, float &d) {
        float *r = red + 256 * buf;
        r[128 * half + L] = v;
        tc::named_sync(1, SM_THREADS);
        a = r[128 * (half ^ 1) + L];
        b = r[128 * half + (L ^ 64)];
        d = r[128 * (half ^ 1) + (L ^ 64)];
    };
    int g = 0;
    for (int rnd = 0, k; (k = item_of_round(p.plan, pair, n_pairs, rnd)) >= 0; ++rnd) {
        const WorkItem it = p.plan.items[k];
        if (it.t1 <= it.t0) {
            if (hsel == 0 && half == 0) {
                p.part_ml[((size_t)k * H + head) * 2] = -INFINITY;
                p.part_ml[((size_t)k * H + head) * 2 + 1] = 0.f;
            }
            continue;
        }
        const int n_steps = ceil_div(it.t1 - it.t0, STEP);
        float m_run = -INFINITY, l_run = 0.f;
        for (int i = 0; i < n_steps; ++i, ++g) {
            const int sb = g & 1;
            warp_wait(c, c.bar(B_SFULL + sb), (uint32_t)(g >> 1) & 1u, p.err);
            tc::fence_after_sync();
            float s[32];
            tc::tmem_ld32(tmem + TM_S + 64 * sb + 32 * half + lane_addr, s);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive_cluster(c.lead_bar(B_SFREE + sb));

            const int tok0 = it.t0 + STEP * i + 64 * hsel + 32 * half;
            const int nvalid = min(32, max(0, it.t1 - tok0));
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                s[j] = j < nvalid ? s[j] : -INFINITY;
                m4[j & 3] = fmaxf(m4[j & 3], s[j]);
            }
            float o1, o2, o3;
            others(g & 1, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])), o1, o2, o3);
            const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            const float m_tile = fmaxf(fmaxf(mt, o1), fmaxf(o2, o3)) * p.scale_log2;   // head max, log2 units
            // One rescale decision for all heads keeps the tcgen05 loads below warp-uniform.
            const bool any = tc::named_sync_or(2, SM_THREADS, i > 0 && m_tile > m_run + RESCALE_LOG2);
            // P is double-buffered: writing P(g) needs only PV(g-2) complete.  A rescale of O needs
            // PV(g-1) complete (which implies PV(g-2)).  `any` is uniform over the CTA.
            if (any && g >= 1)
                warp_wait(c, c.bar(B_PVDONE + ((g - 1) & 1)), (uint32_t)((g - 1) >> 1) & 1u, p.err);
            else if (g >= 2)
                warp_wait(c, c.bar(B_PVDONE + (g & 1)), (uint32_t)((g - 2) >> 1) & 1u, p.err);
            tc::fence_after_sync();
            if (i == 0) {
                m_run = m_tile;
            } else if (any) {
                const float m_new = fmaxf(m_run, m_tile);
                const float alpha = tc::ex2(m_run - m_new);
#pragma unroll 1
                for (int q = 0; q < 2; ++q) {
                    float v[64];
                    const uint32_t a = tmem + TM_O + 128 * half + 64 * q + lane_addr;
                    tc::tmem_ld64(a, v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 64; ++j) v[j] *= alpha;
                    tc::tmem_st64(a, v);
                }
                tc::tmem_wait_st();
                l_run *= alpha;
                m_run = m_new;
            }
            const float neg_m = -m_run;
            float sum4[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float a = tc::ex2(fmaf(s[2 * j], p.scale_log2, neg_m));
                const float b2 = tc::ex2(fmaf(s[2 * j + 1], p.scale_log2, neg_m));
                sum4[j & 3] += a + b2;
                __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b2);
                pk[j] = *reinterpret_cast<uint32_t *>(&h2);
            }
            l_run += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
            // P(g) into TMEM buffer g & 1 as the A operand of the two-CTA PV MMA, which takes the
            // CTA's 64 rows twice (lanes L and L ^ 64 hold head L % 64 for all 128 tokens of the step;
            // column c = tokens 2c, 2c + 1).  This thread has tokens [64 hsel + 32 half, +32), i.e.
            // columns [32 hsel + 16 half, +16); the thread of lane L ^ 64 (warp w ^ 2, same half) has
            // the other page's, swapped through shared memory.
            {
                uint4 *xb = reinterpret_cast<uint4 *>(c.sbase + OFF_X);   // [half][lane L][4 x 16 B]
                const int sw = (lane >> 1) & 3;                          // conflict-free 16-byte slots
#pragma unroll
                for (int ch = 0; ch < 4; ++ch)
                    xb[(128 * half + L) * 4 + (ch ^ sw)] = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
                tc::named_sync(3 + 2 * half + (warp & 1), 64);   // warps w and w ^ 2
                uint32_t pp[16];
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const uint4 v = xb[(128 * half + (L ^ 64)) * 4 + (ch ^ sw)];
                    pp[4 * ch] = v.x;
                    pp[4 * ch + 1] = v.y;
                    pp[4 * ch + 2] = v.z;
                    pp[4 * ch + 3] = v.w;
                }
                const uint32_t pcol = tmem + TM_P + 64 * (g & 1) + 16 * half + lane_addr;
                tc::tmem_st16(pcol + 32 * hsel, pk);
                tc::tmem_st16(pcol + 32 * (hsel ^ 1), pp);
                tc::tmem_wait_st();
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive_cluster(c.lead_bar(B_PFULL + (g & 1)));
        }
        // Epilogue: the last PV of this item has landed; write the partial O, m, l.
        warp_wait(c, c.bar(B_PVDONE + ((g - 1) & 1)), (uint32_t)((g - 1) >> 1) & 1u, p.err);
        tc::fence_after_sync();
        float l1, l2, l3;
        others(g & 1, l_run, l1, l2, l3);
        const float l_tot = (l_run + l1) + (l2 + l3);
        // Partial O in the octet layout [item][64 column octets][H][8]: a warp (32 consecutive heads)
        // stores 32 whole 32-byte sectors per octet, 1 KiB contiguous, one 256-bit store per thread.
        // (Two 128-bit stores per thread left every sector half-written per instruction: the
        // partials of all CTAs took 4.6 us at ~4 TB/s.)
#pragma unroll 1
        for (int q = 0; q < 2; ++q) {
            float v[64];
            tc::tmem_ld64(tmem + TM_O + 128 * half + 64 * q + lane_addr, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int jo = 0; jo < 8; ++jo) {
                const int oct = 32 * half + 16 * hsel + 8 * q + jo;
                tc::st_global_v8(p.part_o + (((size_t)k * 64 + oct) * H + head) * 8, v + 8 * jo);
            }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_cluster(c.lead_bar(B_OFREE));
        if (hsel == 0 && half == 0) {
            p.part_ml[((size_t)k * H + head) * 2] = m_run * 0.69314718055994531f;
            p.part_ml[((size_t)k * H + head) * 2 + 1] = l_tot;
        }
        tc::named_sync(1, SM_THREADS);   // the next item's first exchange reuses buffer g & 1
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    tc_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, TcParams p) {
    // Barrier set-up and the tensor-memory allocation touch no global memory: they run while the
    // previous kernel (the query absorption) finishes; the roles start after step_wait_prev().
    step_allow_next();
    extern __shared__ uint8_t smem_raw[];
    Ctx c;
    const uint32_t raw = tc::smem_addr(smem_raw);
    c.base = (raw + 1023u) & ~1023u;
    c.sbase = smem_raw + (c.base - raw);
    c.rank = tc::cluster_rank();
    c.abort_flag = reinterpret_cast<volatile int *>(c.sbase + OFF_FLAG);
    c.wait_ns = p.wait_ns;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    uint32_t dyn_bytes;
    asm("mov.u32 %0, %dynamic_smem_size;" : "=r"(dyn_bytes));
    if (c.base - raw + SMEM_USED > dyn_bytes) {   // uniform for the whole cluster: nothing ran yet
        step_wait_prev();
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
        tc::mbar_init(c.bar(B_QEMPTY), 1);
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(c.bar(B_SFULL + i), 1);
            tc::mbar_init(c.bar(B_SFREE + i), 2 * SOFTMAX_WARPS);
            tc::mbar_init(c.bar(B_PVDONE + i), 1);
        }
        tc::mbar_init(c.bar(B_PFULL), 2 * SOFTMAX_WARPS);
        tc::mbar_init(c.bar(B_PFULL + 1), 2 * SOFTMAX_WARPS);
        tc::mbar_init(c.bar(B_OFREE), 2 * SOFTMAX_WARPS);
        tc::mbar_init(c.bar(B_VLOCAL), 1);
        tc::mbar_init(c.bar(B_VTAIL), 2);
        *c.abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == W_KPROD && lane == 0) {
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_v);
    }
    if (warp == W_MMA) tc::tmem_alloc_pair(c.base + OFF_TMEMPTR, TM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::cluster_sync();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(c.sbase + OFF_TMEMPTR);
    step_wait_prev();   // q_abs and the plan come from the previous kernel

    const int pair = blockIdx.x / 2, n_pairs = gridDim.x / 2;
    if (warp == W_KPROD) {
        if (lane == 0) run_k_producer(c, p, &tm_q, &tm_k, pair, n_pairs, 0, K_SPLIT);
    } else if (warp == W_KPROD2) {
        if (lane == 0) run_k_producer(c, p, &tm_q, &tm_k, pair, n_pairs, K_SPLIT, NK);
    } else if (warp == W_VPROD) {
        if (lane == 0)
            run_v_producer(c, p, &tm_v, pair, n_pairs);
        else
            run_v_tail(c, p, pair, n_pairs);
    } else if (warp == W_MMA) {
        if (c.rank == 0 && lane == 0) run_qk_issuer(c, p, tmem, pair, n_pairs);
    } else if (warp == W_PV) {
        if (c.rank == 0 && lane == 0) run_pv_issuer(c, p, tmem, pair, n_pairs);
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
    if (warp == W_MMA) {
        tc::fence_after_sync();
        tc::tmem_dealloc_pair(tmem, TM_COLS);
        tc::tmem_relinquish_pair();
    }
}

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once; the initialisation of a function-local static is thread-safe.
EncodeTiled encode_fn() {
    static const EncodeTiled fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiled>(ptr);
        return (EncodeTiled) nullptr;
    }();
    return fn;
}

// Views of a row-major [rows, 576] bf16 matrix whose innermost dimension is one 64-column
// block (128 bytes, swizzled), so one box gathers several blocks of 64 rows block-major into
// shared memory.  `nblk` = blocks per box; with `vsplit` the blocks are addressed as
// [4 blocks per 256-column chunk][2 chunks].  Zero fill past the end.
bool encode_blocks(CUtensorMap *m, const void *ptr, uint64_t rows, int nblk, bool vsplit) {
    EncodeTiled fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (!vsplit) {
        cuuint64_t dims[3] = {64, rows, 9};
        cuuint64_t strides[2] = {DROW * 2, 128};
        cuuint32_t box[3] = {64, 64, (cuuint32_t)nblk};
        return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    cuuint64_t dims[4] = {64, rows, 4, 2};
    cuuint64_t strides[3] = {DROW * 2, 128, 512};
    cuuint32_t box[4] = {64, 64, 2, 2};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The maps depend only on (base pointer, rows, box shape); a decode loop passes the same buffers
// every step, so recent encodings are reused (a host-side encoding costs about a microsecond).
bool encode_blocks_cached(CUtensorMap *m, const void *ptr, uint64_t rows, int nblk, bool vsplit) {
    struct Entry {
        const void *ptr;
        uint64_t rows;
        int nblk, device;
        bool vsplit;
        CUtensorMap map;
    };
    static std::mutex mu;
    static Entry cache[16];
    static int used = 0, next = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (cache[i].ptr == ptr && cache[i].rows == rows && cache[i].nblk == nblk && cache[i].vsplit == vsplit &&
                cache[i].device == dev) {
                *m = cache[i].map;
                return true;
            }
    }
    if (!encode_blocks(m, ptr, rows, nblk, vsplit)) return false;
    std::lock_guard<std::mutex> lock(mu);
    cache[next] = Entry{ptr, rows, nblk, dev, vsplit, *m};
    next = (next + 1) % 16;
    used = used < 16 ? used + 1 : 16;
    return true;
}

thread_local int g_test_withhold = -1;
thread_local uint64_t g_test_wait_ns = WAIT_NS;

}  // namespace

void tc_set_test_fault(int withhold_step, uint64_t wait_ns) {
    g_test_withhold = withhold_step < 0 ? -1 : withhold_step;
    g_test_wait_ns = wait_ns == 0 ? WAIT_NS : wait_ns;
}

bool tc_available() { return true; }
int tc_units(int sms) { return sms / 2; }
int tc_token_granule() { return STEP; }

cudaError_t launch_tc_decode(const Dims &d, const void *q_abs, const void *latent, const int *page_table,
                             const Plan &plan, int max_pages, int n_pages, int s_q, float *part_o, float *part_ml,
                             int *err, int sms, cudaStream_t st) {
    if (plan.n_work == 0) return cudaSuccess;
    CUtensorMap tm_q, tm_k, tm_v;
    const uint64_t kv_rows = (uint64_t)n_pages * PAGE;
    if (!encode_blocks_cached(&tm_q, q_abs, (uint64_t)plan.rows * H, 9, false) ||
        !encode_blocks_cached(&tm_k, latent, kv_rows, 3, false) || !encode_blocks_cached(&tm_v, latent, kv_rows, 0, true))
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
    p.wait_ns = g_test_wait_ns;
    p.withhold = g_test_withhold;
    cudaError_t e = raise_smem_limit((const void *)tc_decode_kernel, SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const int units = std::max(1, std::min(plan.n_work, std::max(1, sms / 2)));
    MLA_STEP_LAUNCH(tc_decode_kernel, dim3(2 * units), dim3(THREADS), SMEM_ALLOC, st, tm_q, tm_k, tm_v, p);
    return cudaGetLastError();
}

}  // namespace mla
