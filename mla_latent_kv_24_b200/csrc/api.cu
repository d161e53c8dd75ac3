// libmla host layer: argument checks, split planning, workspace layout and kernel launches
// behind the C ABI declared in include/mla.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>

#include "kernels.h"
#include "plan_host.h"
#include "tc_decode.h"

namespace mla {

// Per-device error word written by kernels (see report()).
__device__ int g_device_error;

namespace {

thread_local std::string g_last_error;
thread_local cudaEvent_t g_prof_start = nullptr, g_prof_stop = nullptr;

// Brackets the main attention kernel with the caller's profiling events, if set.
struct ProfileScope {
    cudaStream_t st;
    explicit ProfileScope(cudaStream_t s) : st(s) {
        if (g_prof_start && g_prof_stop) cudaEventRecord(g_prof_start, st);
    }
    ~ProfileScope() {
        if (g_prof_start && g_prof_stop) cudaEventRecord(g_prof_stop, st);
    }
};

mla_status fail(mla_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

mla_status cuda_fail(cudaError_t e, const char *what) {
    return fail(MLA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

constexpr int MAX_DEVICES = 64;
// Per-device constants, looked up on a device's first call.  The SM count is written before the
// error-word pointer is published (release), and readers load the pointer first (acquire), so a
// thread that sees the pointer also sees the count; concurrent first calls write the same values.
std::atomic<int *> g_err_ptr[MAX_DEVICES];
std::atomic<int> g_sm_count[MAX_DEVICES];

// Device address of the error word and SM count of the current device, looked up once.
mla_status device_info(int **err, int *sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= MAX_DEVICES) return fail(MLA_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
    int *ptr = g_err_ptr[dev].load(std::memory_order_acquire);
    if (!ptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_error);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
        g_sm_count[dev].store(n, std::memory_order_relaxed);
        ptr = (int *)p;
        g_err_ptr[dev].store(ptr, std::memory_order_release);
    }
    if (err) *err = ptr;
    if (sms) *sms = g_sm_count[dev].load(std::memory_order_relaxed);
    return MLA_OK;
}

bool is_standard_bf16(const mla_dims *d) {
    return d->dtype == MLA_BF16 && d->n_heads == 128 && d->d_c == 512 && d->d_rope == 64 && d->d_nope == 128 &&
           d->d_v == 128 && d->page_size == 64;
}

mla_status check_dims(const mla_dims *d, Dims *out) {
    if (!d) return fail(MLA_ERR_INVALID_ARG, "dims is NULL");
    if (d->dtype != MLA_BF16 && d->dtype != MLA_FP32) return fail(MLA_ERR_INVALID_ARG, "unknown dtype %d", (int)d->dtype);
    if (d->n_heads <= 0 || d->heads_per_group <= 0 || d->n_heads % d->heads_per_group)
        return fail(MLA_ERR_INVALID_ARG, "heads_per_group (%d) must divide n_heads (%d)", d->heads_per_group,
                    d->n_heads);
    if (d->d_c <= 0 || d->d_rope <= 0 || d->d_nope <= 0 || d->d_v <= 0 || d->page_size <= 0)
        return fail(MLA_ERR_INVALID_ARG, "dimensions must be positive");
    if (d->d_c % 8 || d->d_rope % 8 || d->d_nope % 8)
        return fail(MLA_ERR_UNSUPPORTED, "d_c, d_rope and d_nope must be multiples of 8");
    if (d->n_heads > 128 || d->d_c > 512 || d->d_rope > 64 || d->d_nope > 128 || d->d_v > 128)
        return fail(MLA_ERR_UNSUPPORTED, "dims exceed H<=128, d_c<=512, d_rope<=64, d_nope<=128, d_v<=128");
    if (d->page_size != 16 && d->page_size != 32 && d->page_size != 64 && d->page_size != 128)
        return fail(MLA_ERR_UNSUPPORTED, "page_size must be 16, 32, 64 or 128");
    if (!(d->rope_base > 0.f)) return fail(MLA_ERR_INVALID_ARG, "rope_base must be > 0");
    out->H = d->n_heads;
    out->hpw = d->heads_per_group;
    out->d_c = d->d_c;
    out->d_r = d->d_rope;
    out->d_n = d->d_nope;
    out->d_v = d->d_v;
    out->page = d->page_size;
    out->scale = d->softmax_scale > 0.f ? d->softmax_scale : (float)(1.0 / sqrt((double)(d->d_nope + d->d_rope)));
    out->base = d->rope_base;
    out->bf16 = d->dtype == MLA_BF16;
    return MLA_OK;
}

size_t elt(const Dims &d) { return d.bf16 ? 2 : 4; }
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }

mla_status check_batch(const Dims &d, int batch, int s_q, int max_pages, const int32_t *lens_host) {
    if (batch <= 0) return fail(MLA_ERR_INVALID_ARG, "batch must be > 0");
    if (s_q < 1 || s_q > 4) return fail(MLA_ERR_INVALID_ARG, "s_q must be 1..4 (got %d)", s_q);
    if (max_pages <= 0) return fail(MLA_ERR_INVALID_ARG, "max_pages must be > 0");
    if (!lens_host) return fail(MLA_ERR_INVALID_ARG, "seq_lens_host is NULL");
    if ((long long)batch * s_q > (1 << 20)) return fail(MLA_ERR_UNSUPPORTED, "batch * s_q too large");
    for (int b = 0; b < batch; ++b) {
        const long long L = lens_host[b];
        if (L < s_q || L > (long long)max_pages * d.page)
            return fail(MLA_ERR_INVALID_ARG, "seq_lens[%d] = %lld outside [s_q=%d, max_pages*page=%lld]", b, L, s_q,
                        (long long)max_pages * d.page);
    }
    return MLA_OK;
}

// Workspace layout of one decode call.
// Plan rows are (request, query) pairs, except on the tensor-core grouped path, where one work
// item covers all s_q queries of a request (they share every K/V tile), so the plan has one
// row per request and each item stores s_q partial results (qpi = queries per item).
struct Layout {
    size_t q_off, items_off, row_off, order_off, po_off, pml_off, total;
    int n_work, chunk, rows, plan_sq, qpi, DK, DV;
    bool tc;
};

enum Path { ABSORBED = 0, GROUPED = 1 };

mla_status make_layout(const Dims &d, Path path, bool tc, int sms, int batch, int s_q, const int32_t *lens,
                       Layout *L) {
    L->rows = batch * s_q;
    L->tc = tc;
    L->DK = path == ABSORBED ? d.d_c + d.d_r : d.d_n + d.d_r;
    L->DV = path == ABSORBED ? d.d_c : d.d_v;
    // Split policy: chunks sized so the number of concurrent units is covered about once.
    int units, granule;
    if (tc) {
        units = tc_units(sms);
        granule = tc_token_granule();
    } else if (path == GROUPED && grouped_tc_ok(d, s_q)) {
        units = grouped_units(d, sms);
        granule = grouped_token_granule();
    } else {
        const int hb = simt_heads_per_block(d, path == ABSORBED ? 0 : 1);
        units = std::max(1, 4 * sms / std::max(1, d.H / hb));
        granule = 32;
    }
    L->plan_sq = (path == GROUPED && grouped_tc_ok(d, s_q)) ? 1 : s_q;
    L->qpi = s_q / L->plan_sq;
    L->chunk = plan_chunk(lens, batch, L->plan_sq, units, granule);
    L->n_work = (int)plan_count(lens, batch, L->plan_sq, L->chunk);
    size_t off = 0;
    L->q_off = off;
    off = align256(off + (size_t)L->rows * d.H * L->DK * elt(d));
    L->items_off = off;
    off = align256(off + (size_t)L->n_work * sizeof(WorkItem));
    L->row_off = off;
    off = align256(off + (size_t)(batch * L->plan_sq + 1) * sizeof(int));
    L->order_off = off;   // the tcgen05 decode's take order of the items, and the plan's scratch
    off = align256(off + (tc ? (size_t)(L->n_work + batch * L->plan_sq + 1) * sizeof(int) : 0));
    L->po_off = off;
    off = align256(off + (size_t)L->n_work * L->qpi * d.H * L->DV * sizeof(float));
    L->pml_off = off;
    off = align256(off + (size_t)L->n_work * L->qpi * d.H * 2 * sizeof(float));
    L->total = off;
    return MLA_OK;
}

bool use_tc_absorbed(const mla_dims *dims) { return is_standard_bf16(dims) && tc_available(); }

mla_status check_ws(const Layout &L, void *ws, size_t bytes) {
    if (!ws) return fail(MLA_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", L.total);
    if (bytes < L.total) return fail(MLA_ERR_WORKSPACE, "workspace has %zu bytes, need %zu", bytes, L.total);
    if ((uintptr_t)ws & 255) return fail(MLA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    return MLA_OK;
}

#define MLA_TRY(x)                          \
    do {                                    \
        mla_status _s = (x);                \
        if (_s != MLA_OK) return _s;        \
    } while (0)
#define MLA_CUDA(x, what)                                  \
    do {                                                   \
        cudaError_t _e = (x);                              \
        if (_e != cudaSuccess) return cuda_fail(_e, what); \
    } while (0)

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" {

int32_t mla_version(void) { return 100; }

mla_status mla_set_profile_events(void *start_event, void *stop_event) {
    g_prof_start = (cudaEvent_t)start_event;
    g_prof_stop = (cudaEvent_t)stop_event;
    return MLA_OK;
}

const char *mla_last_error_string(void) { return g_last_error.c_str(); }

mla_status mla_get_device_status(mla_stream_t stream) {
    int *err = nullptr;
    MLA_TRY(device_info(&err, nullptr));
    MLA_CUDA(cudaStreamSynchronize((cudaStream_t)stream), "cudaStreamSynchronize");
    int v = 0;
    MLA_CUDA(cudaMemcpyFromSymbol(&v, g_device_error, sizeof v), "read device error word");
    if (v != 0) {
        const int zero = 0;
        MLA_CUDA(cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero), "clear device error word");
        return fail((mla_status)v, "device reported error %d", v);
    }
    return MLA_OK;
}

mla_status mla_debug_decode_fault(int32_t withhold_step, uint32_t wait_us) {
    g_last_error.clear();
    if (withhold_step < -1) return fail(MLA_ERR_INVALID_ARG, "withhold_step must be >= -1");
    if (wait_us > 2000000u) return fail(MLA_ERR_INVALID_ARG, "wait_us must be <= 2000000");
    tc_set_test_fault(withhold_step, (uint64_t)wait_us * 1000ull);
    return MLA_OK;
}

mla_status mla_cache_append(const mla_dims *dims, const void *h, int32_t hidden, const void *W_dkv,
                            const void *W_kr, const int32_t *req_idx, const int32_t *positions, int32_t n_tok,
                            const int32_t *page_table, int32_t batch, int32_t max_pages, int32_t n_pages_total,
                            void *latent_cache, mla_stream_t stream) {
    g_last_error.clear();
    Dims d;
    MLA_TRY(check_dims(dims, &d));
    if (n_tok < 0) return fail(MLA_ERR_INVALID_ARG, "n_tok < 0");
    if (n_tok == 0) return MLA_OK;
    if (!h || !req_idx || !positions || !page_table || !latent_cache)
        return fail(MLA_ERR_INVALID_ARG, "NULL device pointer");
    if ((W_dkv == nullptr) != (W_kr == nullptr)) return fail(MLA_ERR_INVALID_ARG, "W_dkv and W_kr must both be NULL or both set");
    if (W_dkv == nullptr && hidden != d.d_row())
        return fail(MLA_ERR_INVALID_ARG, "pre-projected input needs hidden == d_c + d_rope (%d), got %d", d.d_row(), hidden);
    if (hidden <= 0) return fail(MLA_ERR_INVALID_ARG, "hidden must be > 0");
    if (batch <= 0 || max_pages <= 0 || n_pages_total <= 0) return fail(MLA_ERR_INVALID_ARG, "batch, max_pages, n_pages_total must be > 0");
    int *err = nullptr;
    MLA_TRY(device_info(&err, nullptr));
    if (append_mma_ok(d, hidden, W_dkv != nullptr) && aligned16(h) && aligned16(W_dkv) && aligned16(W_kr))
        MLA_CUDA(launch_append_mma(d, h, hidden, W_dkv, W_kr, req_idx, positions, n_tok, page_table, batch, max_pages,
                                   n_pages_total, latent_cache, err, (cudaStream_t)stream),
                 "launch cache_append (tensor cores)");
    else
        MLA_CUDA(launch_append(d, h, hidden, W_dkv, W_kr, req_idx, positions, n_tok, page_table, batch, max_pages,
                               n_pages_total, latent_cache, err, (cudaStream_t)stream),
                 "launch cache_append");
    return MLA_OK;
}

static mla_status decode_workspace(const mla_dims *dims, Path path, int32_t batch, int32_t s_q,
                                   const int32_t *lens, size_t *bytes, Layout *L) {
    Dims d;
    MLA_TRY(check_dims(dims, &d));
    if (!bytes) return fail(MLA_ERR_INVALID_ARG, "bytes is NULL");
    if (batch <= 0 || s_q < 1 || s_q > 4 || !lens) return fail(MLA_ERR_INVALID_ARG, "bad batch / s_q / seq_lens_host");
    int sms = 0;
    MLA_TRY(device_info(nullptr, &sms));
    const bool tc = path == ABSORBED && use_tc_absorbed(dims);
    MLA_TRY(make_layout(d, path, tc, sms, batch, s_q, lens, L));
    *bytes = L->total;
    return MLA_OK;
}

mla_status mla_decode_workspace_size(const mla_dims *dims, int32_t batch, int32_t s_q, const int32_t *seq_lens_host,
                                     size_t *bytes) {
    g_last_error.clear();
    Layout L;
    return decode_workspace(dims, ABSORBED, batch, s_q, seq_lens_host, bytes, &L);
}

mla_status gqla_decode_workspace_size(const mla_dims *dims, int32_t batch, int32_t s_q,
                                      const int32_t *seq_lens_host, size_t *bytes) {
    g_last_error.clear();
    Layout L;
    return decode_workspace(dims, GROUPED, batch, s_q, seq_lens_host, bytes, &L);
}

static mla_status run_decode(Path path, const mla_dims *dims, const void *q, const void *W_uk, const void *W_uv,
                             const void *latent, const void *expanded, const int32_t *page_table,
                             const int32_t *seq_lens, const int32_t *lens_host, int32_t batch, int32_t s_q,
                             int32_t max_pages, int32_t n_pages, void *out, void *ws, size_t ws_bytes,
                             cudaStream_t st) {
    g_last_error.clear();
    Dims d;
    MLA_TRY(check_dims(dims, &d));
    MLA_TRY(check_batch(d, batch, s_q, max_pages, lens_host));
    if (!q || !latent || !page_table || !seq_lens || !out) return fail(MLA_ERR_INVALID_ARG, "NULL device pointer");
    if (path == ABSORBED && (!W_uk || !W_uv)) return fail(MLA_ERR_INVALID_ARG, "W_uk / W_uv is NULL");
    if (path == GROUPED && !expanded) return fail(MLA_ERR_INVALID_ARG, "expanded_cache is NULL");
    if (path == GROUPED && d.hpw > 16 && d.hpw % 16)
        return fail(MLA_ERR_UNSUPPORTED, "grouped path needs heads_per_group <= 16 or a multiple of 16");
    if (n_pages <= 0) return fail(MLA_ERR_INVALID_ARG, "n_pages_total must be > 0");
    if (!aligned16(q) || !aligned16(latent) || !aligned16(out) || (expanded && !aligned16(expanded)) ||
        (W_uk && !aligned16(W_uk)) || (W_uv && !aligned16(W_uv)))
        return fail(MLA_ERR_INVALID_ARG, "device tensors must be 16-byte aligned");
    int *err = nullptr, sms = 0;
    MLA_TRY(device_info(&err, &sms));
    const bool tc = path == ABSORBED && use_tc_absorbed(dims);
    Layout L;
    MLA_TRY(make_layout(d, path, tc, sms, batch, s_q, lens_host, &L));
    MLA_TRY(check_ws(L, ws, ws_bytes));
    char *w = (char *)ws;
    WorkItem *items = (WorkItem *)(w + L.items_off);
    int *row_first = (int *)(w + L.row_off);
    float *part_o = (float *)(w + L.po_off);
    float *part_ml = (float *)(w + L.pml_off);
    void *qp = w + L.q_off;
    int *order = tc ? (int *)(w + L.order_off) : nullptr;
    Plan plan{items, row_first, L.n_work, batch * L.plan_sq, L.chunk, order};

    const PlanArgs pa{seq_lens, batch, L.plan_sq, max_pages, d.page, L.chunk, L.n_work, items, row_first, err, order};
    if (path == ABSORBED) {
        if (q_absorb_mma_ok(d)) {
            MLA_CUDA(launch_q_absorb_mma(d, q, W_uk, seq_lens, batch, s_q, qp, pa, st),
                     "launch q_absorb (tensor cores) + plan");
        } else {
            MLA_CUDA(launch_plan(pa, st), "launch plan");
            MLA_CUDA(launch_q_absorb(d, q, W_uk, seq_lens, batch, s_q, qp, st), "launch q_absorb");
        }
        if (tc) {
            ProfileScope prof(st);
            MLA_CUDA(launch_tc_decode(d, qp, latent, page_table, plan, max_pages, n_pages, s_q, part_o, part_ml, err, sms,
                                      st),
                     "launch tcgen05 decode");
        } else {
            ProfileScope prof(st);
            SimtDecodeArgs a{qp, latent, nullptr, page_table, plan, max_pages, n_pages, s_q, 0, part_o, part_ml, err};
            MLA_CUDA(launch_decode_simt(d, a, st), "launch decode (CUDA cores)");
        }
        if (combine_mma_ok(d, L.DV, true)) {
            // The plan's row starts from the host lengths (the device plan is built from the same rule).
            int starts[RowStarts::MAX + 1];
            const int *sp = nullptr;
            if (L.rows <= RowStarts::MAX && L.plan_sq == s_q) {
                starts[0] = 0;
                for (int r = 0; r < L.rows; ++r) {
                    const int b = r / s_q, j = r % s_q;
                    starts[r + 1] = starts[r] + ceil_div(lens_host[b] - s_q + j + 1, L.chunk);
                }
                if (starts[L.rows] == L.n_work) sp = starts;
            }
            MLA_CUDA(launch_combine_mma(d, part_o, part_ml, row_first, sp, L.rows, tc, W_uv, out, st),
                     "launch combine + W_UV (tensor cores)");
        }
        else if (!tc)
            MLA_CUDA(launch_combine(d, part_o, part_ml, row_first, L.rows, 1, L.DV, W_uv, out, st), "launch combine");
        else
            return fail(MLA_ERR_UNSUPPORTED, "tcgen05 partials need the tensor-core combine");
    } else {
        MLA_CUDA(launch_q_rope(d, q, seq_lens, batch, s_q, qp, pa, st), "launch q_rope + plan");
        if (grouped_tc_ok(d, s_q)) {
            ProfileScope prof(st);
            MLA_CUDA(launch_grouped_decode(d, qp, expanded, latent, seq_lens, page_table, plan, max_pages, n_pages,
                                           s_q, part_o, part_ml, err, st),
                     "launch grouped decode");
        } else {
            ProfileScope prof(st);
            SimtDecodeArgs a{qp, latent, expanded, page_table, plan, max_pages, n_pages, s_q, 1, part_o, part_ml, err};
            MLA_CUDA(launch_decode_simt(d, a, st), "launch grouped decode (CUDA cores)");
        }
        MLA_CUDA(launch_combine(d, part_o, part_ml, row_first, L.rows, L.qpi, L.DV, nullptr, out, st), "launch combine");
    }
    return MLA_OK;
}

// Scratch of mla_decode_absorbed_noalloc: a file-scope device array, so callers that cannot
// allocate still get a workspace.  Host code must not use its name as an address (that names a
// host-side stand-in); each device's real address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

static void *g_noalloc_ptr[MAX_DEVICES];
static std::mutex g_noalloc_mu;

// Device address of the static scratch on the current device, looked up once per device.
static mla_status noalloc_scratch(void **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= MAX_DEVICES) return fail(MLA_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return MLA_OK;
}

mla_status mla_decode_absorbed_noalloc(const mla_dims *dims, const void *q, const void *W_uk, const void *W_uv,
                                       const void *latent_cache, const int32_t *page_table,
                                       const int32_t *seq_lens, const int32_t *seq_lens_host, int32_t batch,
                                       int32_t s_q, int32_t max_pages, int32_t n_pages_total, void *out,
                                       mla_stream_t stream) {
    g_last_error.clear();
    size_t need = 0;
    Layout L;
    MLA_TRY(decode_workspace(dims, ABSORBED, batch, s_q, seq_lens_host, &need, &L));
    if (need > (size_t)MLA_NOALLOC_SCRATCH_BYTES)
        return fail(MLA_ERR_WORKSPACE,
                    "this batch needs %zu bytes of scratch; the static scratch of the no-allocation entry point "
                    "holds %zu (use mla_decode_absorbed with a workspace)",
                    need, (size_t)MLA_NOALLOC_SCRATCH_BYTES);
    void *ws = nullptr;
    MLA_TRY(noalloc_scratch(&ws));
    return run_decode(ABSORBED, dims, q, W_uk, W_uv, latent_cache, nullptr, page_table, seq_lens, seq_lens_host,
                      batch, s_q, max_pages, n_pages_total, out, ws, MLA_NOALLOC_SCRATCH_BYTES,
                      (cudaStream_t)stream);
}

mla_status mla_decode_absorbed(const mla_dims *dims, const void *q, const void *W_uk, const void *W_uv,
                               const void *latent_cache, const int32_t *page_table, const int32_t *seq_lens,
                               const int32_t *seq_lens_host, int32_t batch, int32_t s_q, int32_t max_pages,
                               int32_t n_pages_total, void *out, void *workspace, size_t workspace_bytes,
                               mla_stream_t stream) {
    return run_decode(ABSORBED, dims, q, W_uk, W_uv, latent_cache, nullptr, page_table, seq_lens, seq_lens_host,
                      batch, s_q, max_pages, n_pages_total, out, workspace, workspace_bytes, (cudaStream_t)stream);
}

mla_status gqla_decode_grouped(const mla_dims *dims, const void *q, const void *expanded_cache,
                               const void *latent_cache, const int32_t *page_table, const int32_t *seq_lens,
                               const int32_t *seq_lens_host, int32_t batch, int32_t s_q, int32_t max_pages,
                               int32_t n_pages_total, void *out, void *workspace, size_t workspace_bytes,
                               mla_stream_t stream) {
    return run_decode(GROUPED, dims, q, nullptr, nullptr, latent_cache, expanded_cache, page_table, seq_lens,
                      seq_lens_host, batch, s_q, max_pages, n_pages_total, out, workspace, workspace_bytes,
                      (cudaStream_t)stream);
}

// Prefill layout: q_rot [batch*n_q, H, 192] bf16 | one work item per request | row starts |
// partial O [batch*n_q, H, d_v] fp32 | (m, l) [batch*n_q, H, 2].  One item per request: the
// (head, 16-query tile) CTAs already fill the GPU, and one partial per query keeps the scratch
// linear in n_q.
static mla_status prefill_layout(const mla_dims *dims, int32_t batch, int32_t n_q, const int32_t *lens, Dims *d,
                                 Layout *L) {
    MLA_TRY(check_dims(dims, d));
    if (!prefill_ok(*d)) return fail(MLA_ERR_UNSUPPORTED, "prefill needs bf16, d_nope = d_v = 128, d_rope = 64, d_c = 512, page 64");
    if (batch <= 0 || n_q < 1 || !lens) return fail(MLA_ERR_INVALID_ARG, "bad batch / n_q / seq_lens_host");
    if ((long long)batch * n_q > (1 << 20)) return fail(MLA_ERR_UNSUPPORTED, "batch * n_q too large");
    long long longest = 1;
    for (int b = 0; b < batch; ++b) {
        if (lens[b] < n_q) return fail(MLA_ERR_INVALID_ARG, "seq_lens[%d] = %d < n_q = %d", b, lens[b], n_q);
        longest = std::max<long long>(longest, lens[b]);
    }
    L->rows = batch * n_q;
    L->plan_sq = 1;
    L->qpi = n_q;
    L->DK = d->d_n + d->d_r;
    L->DV = d->d_v;
    L->tc = false;
    L->chunk = (int)((longest + d->page - 1) / d->page * d->page);
    L->n_work = batch;
    size_t off = 0;
    L->q_off = off;
    off = align256(off + (size_t)L->rows * d->H * L->DK * elt(*d));
    L->items_off = off;
    off = align256(off + (size_t)L->n_work * sizeof(WorkItem));
    L->row_off = off;
    off = align256(off + (size_t)(batch + 1) * sizeof(int));
    L->po_off = off;
    off = align256(off + (size_t)L->rows * d->H * L->DV * sizeof(float));
    L->pml_off = off;
    off = align256(off + (size_t)L->rows * d->H * 2 * sizeof(float));
    L->total = off;
    return MLA_OK;
}

mla_status mla_prefill_workspace_size(const mla_dims *dims, int32_t batch, int32_t n_q, const int32_t *seq_lens_host,
                                      size_t *bytes) {
    g_last_error.clear();
    if (!bytes) return fail(MLA_ERR_INVALID_ARG, "bytes is NULL");
    Dims d;
    Layout L;
    MLA_TRY(prefill_layout(dims, batch, n_q, seq_lens_host, &d, &L));
    *bytes = L.total;
    return MLA_OK;
}

mla_status mla_prefill_expanded(const mla_dims *dims, const void *q, const void *expanded_cache,
                                const void *latent_cache, const int32_t *page_table, const int32_t *seq_lens,
                                const int32_t *seq_lens_host, int32_t batch, int32_t n_q, int32_t max_pages,
                                int32_t n_pages_total, void *out, void *workspace, size_t workspace_bytes,
                                mla_stream_t stream) {
    g_last_error.clear();
    Dims d;
    Layout L;
    MLA_TRY(prefill_layout(dims, batch, n_q, seq_lens_host, &d, &L));
    if (max_pages <= 0 || n_pages_total <= 0) return fail(MLA_ERR_INVALID_ARG, "max_pages and n_pages_total must be > 0");
    for (int b = 0; b < batch; ++b)
        if ((long long)seq_lens_host[b] > (long long)max_pages * d.page)
            return fail(MLA_ERR_INVALID_ARG, "seq_lens[%d] = %d > max_pages * page", b, seq_lens_host[b]);
    if (!q || !expanded_cache || !latent_cache || !page_table || !seq_lens || !out)
        return fail(MLA_ERR_INVALID_ARG, "NULL device pointer");
    if (!aligned16(q) || !aligned16(expanded_cache) || !aligned16(latent_cache) || !aligned16(out))
        return fail(MLA_ERR_INVALID_ARG, "device tensors must be 16-byte aligned");
    MLA_TRY(check_ws(L, workspace, workspace_bytes));
    int *err = nullptr;
    MLA_TRY(device_info(&err, nullptr));
    cudaStream_t st = (cudaStream_t)stream;
    char *w = (char *)workspace;
    WorkItem *items = (WorkItem *)(w + L.items_off);
    int *row_first = (int *)(w + L.row_off);
    float *part_o = (float *)(w + L.po_off);
    float *part_ml = (float *)(w + L.pml_off);
    void *qp = w + L.q_off;
    Plan plan{items, row_first, L.n_work, batch, L.chunk};
    const PlanArgs pa{seq_lens, batch, 1, max_pages, d.page, L.chunk, L.n_work, items, row_first, err};
    MLA_CUDA(launch_q_rope(d, q, seq_lens, batch, n_q, qp, pa, st), "launch q_rope + plan");
    {
        ProfileScope prof(st);
        MLA_CUDA(launch_prefill_expanded(d, qp, expanded_cache, latent_cache, seq_lens, page_table, plan, max_pages,
                                         n_pages_total, n_q, part_o, part_ml, err, st),
                 "launch prefill");
    }
    MLA_CUDA(launch_combine(d, part_o, part_ml, row_first, L.rows, n_q, L.DV, nullptr, out, st), "launch combine");
    return MLA_OK;
}

mla_status mla_select_path(const mla_dims *dims, int32_t batch, int32_t s_q, const int32_t *seq_lens_host,
                           double hbm_bytes_per_s, double flops_per_s, int32_t tp, mla_path *path,
                           double *t_absorbed_s, double *t_grouped_s) {
    g_last_error.clear();
    Dims d;
    MLA_TRY(check_dims(dims, &d));
    if (!path) return fail(MLA_ERR_INVALID_ARG, "path is NULL");
    if (batch <= 0 || s_q < 1 || s_q > 4 || !seq_lens_host) return fail(MLA_ERR_INVALID_ARG, "bad batch / s_q / seq_lens_host");
    if (!(hbm_bytes_per_s > 0.0) || !(flops_per_s > 0.0)) return fail(MLA_ERR_INVALID_ARG, "peaks must be > 0");
    const int G = d.n_groups();
    if (tp < 1 || G % tp) return fail(MLA_ERR_INVALID_ARG, "tp = %d must divide the %d KV groups", tp, G);
    double tokens = 0.0, visible = 0.0;
    for (int b = 0; b < batch; ++b) {
        const double L = seq_lens_host[b];
        if (L < s_q) return fail(MLA_ERR_INVALID_ARG, "seq_lens_host[%d] = %d < s_q", b, seq_lens_host[b]);
        tokens += L;
        for (int j = 0; j < s_q; ++j) visible += L - s_q + j + 1;
    }
    const double e = (double)elt(d), heads = (double)d.H / tp, groups = (double)G / tp;
    const double abs_bytes = tokens * (d.d_c + d.d_r) * e + groups * (d.d_n + d.d_v) * d.d_c * e;
    const double abs_flops = visible * 2.0 * heads * (2.0 * d.d_c + d.d_r) + (double)batch * s_q * heads * 2.0 * d.d_c * (d.d_n + d.d_v);
    const double grp_bytes = tokens * (groups * (d.d_n + d.d_v) + d.d_r) * e;
    const double grp_flops = visible * 2.0 * heads * (d.d_n + d.d_r + d.d_v);
    const double t_abs = std::max(abs_bytes / hbm_bytes_per_s, abs_flops / flops_per_s);
    const double t_grp = std::max(grp_bytes / hbm_bytes_per_s, grp_flops / flops_per_s);
    *path = t_grp < t_abs ? MLA_PATH_GROUPED : MLA_PATH_ABSORBED;
    if (t_absorbed_s) *t_absorbed_s = t_abs;
    if (t_grouped_s) *t_grouped_s = t_grp;
    return MLA_OK;
}

mla_status gqla_expand_cache(const mla_dims *dims, const void *W_uk, const void *W_uv, const void *latent_cache,
                             const int32_t *page_ids, int32_t n_ids, int32_t n_pages_total, void *expanded_cache,
                             mla_stream_t stream) {
    g_last_error.clear();
    Dims d;
    MLA_TRY(check_dims(dims, &d));
    if (!W_uk || !W_uv || !latent_cache || !expanded_cache) return fail(MLA_ERR_INVALID_ARG, "NULL device pointer");
    if (n_pages_total <= 0) return fail(MLA_ERR_INVALID_ARG, "n_pages_total must be > 0");
    if (page_ids == nullptr) n_ids = n_pages_total;
    if (n_ids < 0) return fail(MLA_ERR_INVALID_ARG, "n_ids < 0");
    if (!aligned16(W_uk) || !aligned16(W_uv) || !aligned16(latent_cache) || !aligned16(expanded_cache))
        return fail(MLA_ERR_INVALID_ARG, "device tensors must be 16-byte aligned");
    int *err = nullptr;
    MLA_TRY(device_info(&err, nullptr));
    MLA_CUDA(launch_expand(d, W_uk, W_uv, latent_cache, page_ids, n_ids, n_pages_total, expanded_cache, err,
                           (cudaStream_t)stream),
             "launch gqla_expand_cache");
    return MLA_OK;
}

mla_status gqla_expand_tokens(const mla_dims *dims, const void *W_uk, const void *W_uv, const void *latent_cache,
                              const int32_t *req_idx, const int32_t *positions, int32_t n_tok,
                              const int32_t *page_table, int32_t batch, int32_t max_pages, int32_t n_pages_total,
                              void *expanded_cache, mla_stream_t stream) {
    g_last_error.clear();
    Dims d;
    MLA_TRY(check_dims(dims, &d));
    if (n_tok < 0) return fail(MLA_ERR_INVALID_ARG, "n_tok < 0");
    if (n_tok == 0) return MLA_OK;
    if (!W_uk || !W_uv || !latent_cache || !expanded_cache || !req_idx || !positions || !page_table)
        return fail(MLA_ERR_INVALID_ARG, "NULL device pointer");
    if (batch <= 0 || max_pages <= 0 || n_pages_total <= 0)
        return fail(MLA_ERR_INVALID_ARG, "batch, max_pages, n_pages_total must be > 0");
    if (!aligned16(W_uk) || !aligned16(W_uv) || !aligned16(latent_cache) || !aligned16(expanded_cache))
        return fail(MLA_ERR_INVALID_ARG, "device tensors must be 16-byte aligned");
    int *err = nullptr;
    MLA_TRY(device_info(&err, nullptr));
    MLA_CUDA(launch_expand_tokens(d, W_uk, W_uv, latent_cache, req_idx, positions, n_tok, page_table, batch,
                                  max_pages, n_pages_total, expanded_cache, err, (cudaStream_t)stream),
             "launch gqla_expand_tokens");
    return MLA_OK;
}

}  // extern "C"
