// moedec_api.cu -- the C ABI: argument checks, workspace, side stream, launch order.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "moedec.h"
#include "moedec_internal.h"

using namespace moedec;

extern "C" MOEDEC_API int moedec_kernels_per_step(moedec_handle *h, int batch);

struct moedec_handle {
    moedec_config cfg;
    Dims d;
    Weights w;
    Plan p;
    Work ws;
    ExpertMaps maps;  // TMA maps of the expert codes (maps.ok == 0: none)
    void *buf = nullptr;
    size_t buf_bytes = 0;
    cudaStream_t side = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    int device = 0, n_sm = 0;
    int last_batch = 0;
    const uint16_t *next_router = nullptr;  // moedec_set_next
    uint64_t launches[2] = {0, 0};
    char cuda_error[256] = {0};
    // per-kernel event timing (moedec_profile_enable)
    bool profiling = false;
    struct Mark {
        int kind;
        cudaEvent_t start, stop;
    };
    std::vector<Mark> marks;      // recorded, not yet read
    std::vector<cudaEvent_t> pool;  // free events
    double prof_ms[16] = {0};
    uint64_t prof_n[16] = {0};
};

namespace {

int record_cuda(moedec_handle *h, cudaError_t e) {
    if (e == cudaSuccess) return MOEDEC_OK;
    if (h) snprintf(h->cuda_error, sizeof(h->cuda_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return e == cudaErrorMemoryAllocation ? MOEDEC_ERR_OOM : MOEDEC_ERR_CUDA;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

int krange_for(int K) { return K % 512 == 0 ? 512 : K % 256 == 0 ? 256 : 128; }

// largest n <= max_n with K a multiple of n * unit (1 if none)
int small_split(int K, int unit, int max_n) {
    for (int n = max_n; n > 1; --n)
        if (K % (n * unit) == 0) return n;
    return 1;
}

SplitPlan split(int rows, int rows_per_block, int K) {
    SplitPlan s;
    s.blocks = (rows + rows_per_block - 1) / rows_per_block;
    s.krange = krange_for(K);
    s.splits = K / s.krange;
    return s;
}

typedef CUresult (*TensorMapEncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                      const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 2D uint8 map over `rows` rows of `row_bytes` bytes: boxes of 8 rows x 128 bytes, 128-byte swizzle.
bool encode_rows(TensorMapEncodeFn fn, CUtensorMap *m, const void *base, uint64_t row_bytes, uint64_t rows) {
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {128, 8}, elem[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The expert code maps of the split-K step's ring phases; left with ok == 0 (the step then stages
// activations per segment and streams weights through registers) when the dims do not fit, the
// driver has no tensor-map encoder, or MOEDEC_FLAG_NO_TMA_RING is set.
void make_expert_maps(moedec_handle *h) {
    ExpertMaps &m = h->maps;
    memset(&m, 0, sizeof(m));
    const Dims &d = h->d;
    if ((h->cfg.flags & MOEDEC_FLAG_NO_TMA_RING) || !ring_dims_ok(d)) return;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn) {
        cudaGetLastError();
        return;
    }
    const TensorMapEncodeFn enc = reinterpret_cast<TensorMapEncodeFn>(fn);
    const bool ok = encode_rows(enc, &m.gate, h->w.gate_q, (uint64_t)d.L / 2, (uint64_t)d.ne * d.I) &&
                    encode_rows(enc, &m.up, h->w.up_q, (uint64_t)d.L / 2, (uint64_t)d.ne * d.I) &&
                    encode_rows(enc, &m.down, h->w.down_q, (uint64_t)d.I / 2, (uint64_t)d.ne * d.L);
    m.ok = ok ? 1 : 0;
}

// carve aligned sub-buffers from one allocation
struct Carver {
    char *base;
    size_t off = 0;
    template <class T>
    T *take(size_t n) {
        off = (off + 255) & ~(size_t)255;
        T *p = base ? reinterpret_cast<T *>(base + off) : nullptr;
        off += n * sizeof(T);
        return p;
    }
};

void layout(moedec_handle *h, char *base) {
    const Dims &d = h->d;
    const size_t B = (size_t)d.max_batch;
    const Plan &p = h->p;
    Carver c{base};
    Work &w = h->ws;
    w.rt_part = c.take<double>((size_t)std::max(p.rt.splits, kSmallSplitRt) * B * d.E);
    w.logits = c.take<float>(B * d.E);
    w.rt_acc = c.take<double>(std::min<size_t>(B, kSmallMaxBatch) * d.E);
    w.dn_part = c.take<float>((size_t)std::max(p.dn.splits, kSmallSplitDn) * B * d.L);
    w.h = c.take<float>(B * d.L);
    w.h_shift = c.take<int>(B);
    w.idx = c.take<int>(B * d.k);
    w.wts = c.take<float>(B * d.k);
    w.n_active = c.take<int>(1);
    w.active_e = c.take<int>(d.E);
    w.active_cnt = c.take<int>(d.E);
    w.active_off = c.take<int>(d.E);
    w.entries = c.take<int>(B * d.k);
    w.egu_part = c.take<float>((size_t)kSmallSplitEgu * std::min<size_t>(B, kSmallMaxBatch) * d.k * 2 * d.I);
    w.a = c.take<float>(B * d.k * d.I);
    w.a_amax = c.take<unsigned>(B * d.k);
    w.y = c.take<float>(B * d.k * d.L);
    w.ylat = c.take<float>(B * d.L);
    w.sgu_part = c.take<float>((size_t)std::max(p.sgu.splits, kSmallSplitSgu) * B * 2 * d.Is);
    w.sh_a = c.take<float>(B * d.Is);
    w.sd_part = c.take<float>((size_t)std::max(p.sd.splits, kSmallSplitSd) * B * d.H);
    w.sh = c.take<float>(B * d.H);
    w.up_part = c.take<float>((size_t)std::max(p.up.splits, kSmallSplitUp) * B * d.H);
    w.up_tap = (h->cfg.flags & MOEDEC_FLAG_TAPS) ? c.take<float>(B * d.H) : nullptr;
    {  // streaming small-batch step: at most 2 tokens
        const StreamPlan &sp = p.st;
        const size_t Is = d.n_shared ? d.Is : 512, nent = (size_t)2 * d.k;
        w.st_rt_part = c.take<double>((size_t)sp.s_rt * 2 * d.E);
        w.st_key = c.take<unsigned>((size_t)2 * d.E);
        w.st_dn_part = c.take<float>((size_t)sp.s_dn * 2 * d.L);
        w.st_sgu_part = c.take<float>((size_t)sp.s_sgu * 2 * 2 * Is);
        w.st_egu_part = c.take<float>((size_t)sp.s_egu * nent * 2 * d.I);
        w.st_sd_part = c.take<float>((size_t)sp.s_sd * 2 * d.H);
        w.st_up_part = c.take<float>((size_t)sp.s_up * 2 * d.H);
    }
    w.tickets = c.take<unsigned>((size_t)p.n_tickets);
    w.ctl = c.take<unsigned>((size_t)p.ctl_words);
    w.trace = (h->cfg.flags & MOEDEC_FLAG_TRACE) ? c.take<unsigned long long>((size_t)h->n_sm * kTraceRowsPerSm * kTraceStamps) : nullptr;
    w.err = c.take<unsigned>(1);
    h->buf_bytes = c.off;
}

int check_scales(moedec_handle *h) {
    const Dims &d = h->d;
    unsigned *bad = nullptr;
    cudaError_t e = cudaMalloc(&bad, sizeof(unsigned));
    if (e != cudaSuccess) return record_cuda(h, e);
    struct {
        const uint8_t *p;
        size_t n;
    } arrs[] = {
        {h->w.gate_s, (size_t)d.ne * d.I * (d.L / 32)}, {h->w.up_s, (size_t)d.ne * d.I * (d.L / 32)},
        {h->w.down_s, (size_t)d.ne * d.L * (d.I / 32)}, {h->w.sh_gate_s, d.n_shared ? (size_t)d.Is * (d.H / 32) : 0},
        {h->w.sh_up_s, d.n_shared ? (size_t)d.Is * (d.H / 32) : 0}, {h->w.sh_down_s, d.n_shared ? (size_t)d.H * (d.Is / 32) : 0},
    };
    unsigned host_bad = 0;
    e = cudaMemsetAsync(bad, 0, sizeof(unsigned), h->side);
    for (auto &a : arrs)
        if (e == cudaSuccess) e = launch_scale_check(a.p, a.n, bad, h->side);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host_bad, bad, sizeof(unsigned), cudaMemcpyDeviceToHost, h->side);
    if (e == cudaSuccess) e = cudaStreamSynchronize(h->side);
    cudaFree(bad);
    if (e != cudaSuccess) return record_cuda(h, e);
    return host_bad ? MOEDEC_ERR_UNSUPPORTED : MOEDEC_OK;
}

enum KernelKind {
    K_ROUTER_DN, K_TOPK, K_EXPERT_GU, K_EXPERT_DOWN, K_COMBINE, K_UP, K_SHARED_GU, K_SHARED_DOWN, K_FUSED,
    K_FUSED_SMALL, K_FUSED_STREAM, K_COUNT
};
const char *const kKernelNames[K_COUNT] = {"router_dn", "topk",        "expert_gate_up", "expert_down",
                                           "combine",   "up",          "shared_gate_up", "shared_down",
                                           "fused_step_splitk", "fused_step_small", "fused_step_stream"};

cudaEvent_t pool_get(moedec_handle *h) {
    if (!h->pool.empty()) {
        cudaEvent_t e = h->pool.back();
        h->pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Launch `fn` on `s`; when profiling, bracket it with an event pair on the same stream.
template <class F>
cudaError_t timed(moedec_handle *h, int kind, cudaStream_t s, F fn) {
    if (!h->profiling) return fn();
    cudaEvent_t a = pool_get(h), b = pool_get(h);
    if (!a || !b) return cudaErrorMemoryAllocation;
    // Under stream capture a plain record only expresses a dependency; an external record
    // becomes an event-record node that timestamps every replay of the graph.
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cs);
    const unsigned flags = (cs == cudaStreamCaptureStatusActive) ? cudaEventRecordExternal : 0u;
    if (e == cudaSuccess) e = cudaEventRecordWithFlags(a, s, flags);
    if (e == cudaSuccess) e = fn();
    if (e == cudaSuccess) e = cudaEventRecordWithFlags(b, s, flags);
    if (e == cudaSuccess) h->marks.push_back({kind, a, b});
    return e;
}

int read_device_error(moedec_handle *h, cudaStream_t s) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, h->ws.err, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return record_cuda(h, e);
    if (v == 0) return MOEDEC_OK;
    cudaMemsetAsync(h->ws.err, 0, sizeof(unsigned), s);
    // an aborted small-batch step may have left router sums behind: they are zero at rest
    cudaMemsetAsync(h->ws.rt_acc, 0, std::min<size_t>(h->d.max_batch, kSmallMaxBatch) * h->d.E * sizeof(double), s);
    cudaStreamSynchronize(s);
    return (v & kErrTimeout) ? MOEDEC_ERR_TIMEOUT : MOEDEC_ERR_DEVICE;
}

}  // namespace

extern "C" {

MOEDEC_API const char *moedec_status_string(int status) {
    switch (status) {
        case MOEDEC_OK: return "MOEDEC_OK";
        case MOEDEC_ERR_INVALID_ARG: return "MOEDEC_ERR_INVALID_ARG";
        case MOEDEC_ERR_UNSUPPORTED: return "MOEDEC_ERR_UNSUPPORTED";
        case MOEDEC_ERR_CUDA: return "MOEDEC_ERR_CUDA";
        case MOEDEC_ERR_OOM: return "MOEDEC_ERR_OOM";
        case MOEDEC_ERR_TIMEOUT: return "MOEDEC_ERR_TIMEOUT";
        case MOEDEC_ERR_DEVICE: return "MOEDEC_ERR_DEVICE";
        default: return "MOEDEC_ERR_UNKNOWN";
    }
}

MOEDEC_API const char *moedec_last_cuda_error(moedec_handle *h) { return h ? h->cuda_error : ""; }

}  // extern "C"

namespace {

int create_handle(const moedec_config *cfg, const moedec_weights *w, int e0, int ne, moedec_handle **out) {
    if (!out) return MOEDEC_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg || !w || cfg->abi_version != MOEDEC_ABI_VERSION) return MOEDEC_ERR_INVALID_ARG;
    const moedec_config &c = *cfg;
    if (e0 < 0 || ne < 1 || e0 + ne > c.n_experts) return MOEDEC_ERR_INVALID_ARG;
    if (ne != c.n_experts && (c.flags & MOEDEC_FLAG_STREAM)) return MOEDEC_ERR_UNSUPPORTED;
    if (c.hidden <= 0 || c.latent <= 0 || c.n_experts <= 0 || c.top_k <= 0 || c.expert_inter <= 0 || c.max_batch <= 0 ||
        (c.n_shared != 0 && c.n_shared != 1) || (c.n_shared && c.shared_inter <= 0))
        return MOEDEC_ERR_INVALID_ARG;
    if (c.hidden % 128 || c.latent % 128 || c.expert_inter % 128 || (c.n_shared && c.shared_inter % 128) ||
        c.n_experts > kMaxExperts || c.top_k > c.n_experts || c.top_k > kMaxTopK || c.max_batch > kMaxBatch ||
        c.max_batch * c.top_k > kMaxEntries)
        return MOEDEC_ERR_UNSUPPORTED;
    const void *ptrs[] = {w->router, w->w_down_lat, w->w_up_lat, w->gate_q, w->gate_s, w->up_q, w->up_s, w->down_q, w->down_s};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return MOEDEC_ERR_INVALID_ARG;
    if (c.n_shared) {
        const void *sp[] = {w->sh_gate_q, w->sh_gate_s, w->sh_up_q, w->sh_up_s, w->sh_down_q, w->sh_down_s};
        for (const void *p : sp)
            if (!p || !aligned16(p)) return MOEDEC_ERR_INVALID_ARG;
    }
    moedec_handle *h = new (std::nothrow) moedec_handle();
    if (!h) return MOEDEC_ERR_OOM;
    h->cfg = c;
    h->d = Dims{c.hidden, c.latent, c.n_experts, c.top_k, c.expert_inter, c.n_shared ? c.shared_inter : 128,
                c.n_shared, c.max_batch, e0, ne};
    h->w = Weights{w->router, w->w_down_lat, w->w_up_lat, w->gate_q, w->gate_s, w->up_q, w->up_s, w->down_q, w->down_s,
                   w->sh_gate_q, w->sh_gate_s, w->sh_up_q, w->sh_up_s, w->sh_down_q, w->sh_down_s};
    const Dims &d = h->d;
    Plan &p = h->p;
    p.rt = split(d.E, kRouterRows, d.H);
    p.dn = split(d.L, kDenseRows, d.H);
    p.up = split(d.H, kDenseRows, d.L);
    p.sgu = split(d.Is, kDenseRows, d.H);
    // K ranges of 1024 for the shared gate/up when H allows: half the items and half the splits
    // that the last CTA of a row block adds up (its reduction was the tail that delayed a few
    // CTAs' start of the expert phase; B = 16 280.2 -> 277.2 us)
    if (d.H % 1024 == 0) {
        p.sgu.krange = 1024;
        p.sgu.splits = d.H / 1024;
    }
    p.sd = split(d.H, kDenseRows, d.Is);
    p.ticket_rt = 0;
    p.ticket_dn = p.ticket_rt + p.rt.blocks;
    p.ticket_up = p.ticket_dn + p.dn.blocks;
    p.ticket_sgu = p.ticket_up + p.up.blocks;
    p.ticket_sd = p.ticket_sgu + p.sgu.blocks;
    p.ticket_topk = p.ticket_sd + p.sd.blocks;
    p.n_tickets = p.ticket_topk + 1;
    p.ctl_gu = CTL_FIXED;
    p.ctl_comb = p.ctl_gu + d.E;
    p.ctl_ylat = p.ctl_comb + d.max_batch * (d.L / 16);
    p.ctl_hamax = p.ctl_ylat + d.L / 16;
    p.ctl_shamax = p.ctl_hamax + d.max_batch;
    p.ctl_tk = p.ctl_shamax + d.max_batch;
    p.ctl_tk_words = (d.E + 7) / 8 + d.L / 16 + d.Is / 16 + 2 * (d.H / 16) + d.E * (d.I / 16);
    p.s_rt = small_split(d.H, 32, kSmallSplitRt);
    p.s_dn = small_split(d.H, 32, kSmallSplitDn);
    p.s_sgu = small_split(d.H, 128, kSmallSplitSgu);
    p.s_egu = small_split(d.L, 128, kSmallSplitEgu);
    p.s_sd = small_split(d.Is, 128, kSmallSplitSd);
    p.s_up = small_split(d.L, 32, kSmallSplitUp);
    stream_plan(d, p.st, p.ctl_tk + p.ctl_tk_words);
    p.ctl_words = p.st.words;
    p.wait_limit_ns = (c.flags & (MOEDEC_FLAG_TEST_STALL | MOEDEC_FLAG_TEST_STALL_EXPERTS)) ? 20000000LL : 1000000000LL;

    int rc = MOEDEC_OK;
    cudaError_t e = cudaGetDevice(&h->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->n_sm, cudaDevAttrMultiProcessorCount, h->device);
    if (e == cudaSuccess) e = init_kernel_attributes();
    if (e == cudaSuccess) e = init_fused_attributes();
    if (e == cudaSuccess) e = init_fused_small_attributes();
    if (e == cudaSuccess) e = init_stream_attributes();
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming);
    if (e == cudaSuccess) {
        layout(h, nullptr);
        e = cudaMalloc(&h->buf, h->buf_bytes);
    }
    if (e == cudaSuccess) {
        layout(h, static_cast<char *>(h->buf));
        e = cudaMemsetAsync(h->buf, 0, h->buf_bytes, h->side);
        if (e == cudaSuccess) e = cudaStreamSynchronize(h->side);
    }
    if (e != cudaSuccess) rc = record_cuda(h, e);
    if (rc == MOEDEC_OK && !(c.flags & MOEDEC_FLAG_SKIP_SCALE_CHECK)) rc = check_scales(h);
    if (rc == MOEDEC_OK) make_expert_maps(h);
    if (rc != MOEDEC_OK) {
        moedec_destroy(h);
        return rc;
    }
    *out = h;
    return MOEDEC_OK;
}

}  // namespace

extern "C" {

MOEDEC_API int moedec_create(const moedec_config *cfg, const moedec_weights *w, moedec_handle **out) {
    return create_handle(cfg, w, 0, cfg ? cfg->n_experts : 0, out);
}

MOEDEC_API int moedec_create_shard(const moedec_config *cfg, const moedec_weights *w, int32_t expert_begin,
                                   int32_t expert_count, moedec_handle **out) {
    return create_handle(cfg, w, expert_begin, expert_count, out);
}

MOEDEC_API int moedec_destroy(moedec_handle *h) {
    if (!h) return MOEDEC_OK;
    if (h->side) cudaStreamSynchronize(h->side);
    for (auto &m : h->marks) {
        cudaEventSynchronize(m.stop);
        cudaEventDestroy(m.start);
        cudaEventDestroy(m.stop);
    }
    for (auto e : h->pool) cudaEventDestroy(e);
    if (h->buf) cudaFree(h->buf);
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    if (h->side) cudaStreamDestroy(h->side);
    delete h;
    return MOEDEC_OK;
}

}  // extern "C"

namespace {

// One step into bf16 out (out_f32 == nullptr) or into the fp32 partial out_f32 (out == nullptr).
int step_impl(moedec_handle *h, const uint16_t *x, int batch, uint16_t *out, float *out_f32, void *stream) {
    if (!h || batch < 0) return MOEDEC_ERR_INVALID_ARG;
    if (batch > h->d.max_batch) return MOEDEC_ERR_UNSUPPORTED;
    if (batch == 0) return MOEDEC_OK;
    void *dst = out ? static_cast<void *>(out) : static_cast<void *>(out_f32);
    if (!x || !dst || !aligned16(x) || !aligned16(dst)) return MOEDEC_ERR_INVALID_ARG;
    const size_t xbytes = (size_t)batch * h->d.H * 2, obytes = (size_t)batch * h->d.H * (out ? 2 : 4);
    const char *xb = reinterpret_cast<const char *>(x), *ob = reinterpret_cast<const char *>(dst);
    if (xb < ob + obytes && ob < xb + xbytes) return MOEDEC_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    StepArgs a;
    a.d = h->d;
    a.w = h->w;
    a.ws = h->ws;
    a.p = h->p;
    a.next_router = h->next_router;
    a.x = x;
    a.out = out;
    a.out_f32 = out_f32;
    a.B = batch;
    a.flags = h->cfg.flags;
    cudaError_t e = cudaSuccess;
    const int variant = batch <= 4 ? 0 : 1;
    if (!(h->cfg.flags & MOEDEC_FLAG_MULTI_KERNEL)) {
        // the streaming schedule writes bf16 only: a partial step takes the small-batch kernel
        const bool stream_sched = (h->cfg.flags & MOEDEC_FLAG_STREAM) && !out_f32 && stream_supports(h->d, batch);
        if (stream_sched)
            e = timed(h, K_FUSED_STREAM, s, [&] { return launch_stream(a, s, h->n_sm); });
        else if (fused_small_supports(h->d, batch))
            e = timed(h, K_FUSED_SMALL, s, [&] { return launch_fused_small(a, h->maps, s, h->n_sm); });
        else
            e = timed(h, K_FUSED, s, [&] { return launch_fused(a, h->maps, s, h->n_sm); });
        if (e != cudaSuccess) return record_cuda(h, e);
        h->launches[variant] += stream_sched ? (uint64_t)kStreamLaunches : 1u;
        h->last_batch = batch;
        return MOEDEC_OK;
    }
    if (h->d.n_shared) {
        e = cudaEventRecord(h->ev_fork, s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(h->side, h->ev_fork, 0);
        if (e == cudaSuccess) e = timed(h, K_SHARED_GU, h->side, [&] { return launch_shared_gate_up(a, h->side); });
        if (e == cudaSuccess) e = timed(h, K_SHARED_DOWN, h->side, [&] { return launch_shared_down(a, h->side); });
        if (e == cudaSuccess) e = cudaEventRecord(h->ev_join, h->side);
    }
    if (e == cudaSuccess) e = timed(h, K_ROUTER_DN, s, [&] { return launch_router_dn(a, s); });
    if (e == cudaSuccess) e = timed(h, K_TOPK, s, [&] { return launch_topk(a, s); });
    if (e == cudaSuccess) e = timed(h, K_EXPERT_GU, s, [&] { return launch_expert_gate_up(a, s, h->n_sm); });
    if (e == cudaSuccess) e = timed(h, K_EXPERT_DOWN, s, [&] { return launch_expert_down(a, s, h->n_sm); });
    if (e == cudaSuccess) e = timed(h, K_COMBINE, s, [&] { return launch_combine(a, s); });
    if (e == cudaSuccess && h->d.n_shared) e = cudaStreamWaitEvent(s, h->ev_join, 0);
    if (e == cudaSuccess) e = timed(h, K_UP, s, [&] { return launch_up(a, s); });
    if (e != cudaSuccess) return record_cuda(h, e);
    h->launches[variant] += (uint64_t)kernels_per_step(h->d);
    h->last_batch = batch;
    return MOEDEC_OK;
}

}  // namespace

extern "C" {

MOEDEC_API int moedec_step(moedec_handle *h, const uint16_t *x, int batch, uint16_t *out, void *stream) {
    return step_impl(h, x, batch, out, nullptr, stream);
}

MOEDEC_API int moedec_step_partial(moedec_handle *h, const uint16_t *x, int batch, float *partial, void *stream) {
    return step_impl(h, x, batch, nullptr, partial, stream);
}

MOEDEC_API int moedec_ep_publish(moedec_handle *h, uint32_t *const *slots, int world, uint32_t epoch, void *stream) {
    if (!h || !slots || world < 1 || world > kEpMaxWorld) return MOEDEC_ERR_INVALID_ARG;
    EpSlots sl{};
    for (int g = 0; g < world; ++g) {
        if (!slots[g] || reinterpret_cast<uintptr_t>(slots[g]) % 4) return MOEDEC_ERR_INVALID_ARG;
        sl.p[g] = slots[g];
    }
    const cudaError_t e = launch_ep_publish(sl, world, epoch, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOEDEC_OK : record_cuda(h, e);
}

MOEDEC_API int moedec_ep_combine(moedec_handle *h, const float *const *parts, const uint32_t *flags, int world,
                                 uint32_t epoch, int batch, uint16_t *out, void *stream) {
    if (!h || !parts || world < 1 || world > kEpMaxWorld || batch < 0) return MOEDEC_ERR_INVALID_ARG;
    if (batch > h->d.max_batch) return MOEDEC_ERR_UNSUPPORTED;
    if (batch == 0) return MOEDEC_OK;
    if (!out || !aligned16(out) || (flags && reinterpret_cast<uintptr_t>(flags) % 4)) return MOEDEC_ERR_INVALID_ARG;
    EpParts pp{};
    for (int g = 0; g < world; ++g) {
        if (!parts[g] || !aligned16(parts[g])) return MOEDEC_ERR_INVALID_ARG;
        pp.p[g] = parts[g];
    }
    const cudaError_t e = launch_ep_combine(pp, flags, world, epoch, (size_t)batch * h->d.H, out, h->ws.err,
                                            h->p.wait_limit_ns, h->n_sm, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOEDEC_OK : record_cuda(h, e);
}

MOEDEC_API int moedec_ipc_export(const void *ptr, void *handle, uint64_t *offset) {
    if (!ptr || !handle || !offset) return MOEDEC_ERR_INVALID_ARG;
    // the handle names the whole allocation that contains ptr (an allocator may hand out pieces
    // of a larger one), so the offset of ptr inside it travels with the handle
    typedef CUresult (*AddressRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn) {
        cudaGetLastError();
        return MOEDEC_ERR_CUDA;
    }
    CUdeviceptr base = 0;
    size_t size = 0;
    if (reinterpret_cast<AddressRangeFn>(fn)(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
        return MOEDEC_ERR_CUDA;
    cudaIpcMemHandle_t m;
    if (cudaIpcGetMemHandle(&m, reinterpret_cast<void *>(base)) != cudaSuccess) {
        cudaGetLastError();
        return MOEDEC_ERR_CUDA;
    }
    static_assert(sizeof(m) == MOEDEC_IPC_HANDLE_BYTES, "IPC handle size");
    memcpy(handle, &m, sizeof(m));
    *offset = (uint64_t)(reinterpret_cast<CUdeviceptr>(ptr) - base);
    return MOEDEC_OK;
}

MOEDEC_API int moedec_ipc_open(const void *handle, void **ptr) {
    if (!handle || !ptr) return MOEDEC_ERR_INVALID_ARG;
    *ptr = nullptr;
    cudaIpcMemHandle_t m;
    memcpy(&m, handle, sizeof(m));
    if (cudaIpcOpenMemHandle(ptr, m, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
        cudaGetLastError();
        *ptr = nullptr;
        return MOEDEC_ERR_CUDA;
    }
    return MOEDEC_OK;
}

MOEDEC_API int moedec_ipc_close(void *ptr) {
    if (!ptr) return MOEDEC_ERR_INVALID_ARG;
    return cudaIpcCloseMemHandle(ptr) == cudaSuccess ? MOEDEC_OK : MOEDEC_ERR_CUDA;
}

MOEDEC_API int moedec_set_next(moedec_handle *h, const moedec_handle *next) {
    if (!h) return MOEDEC_ERR_INVALID_ARG;
    if (next && (next->d.H != h->d.H || next->d.E != h->d.E || next->device != h->device)) return MOEDEC_ERR_INVALID_ARG;
    h->next_router = next ? next->w.router : nullptr;
    return MOEDEC_OK;
}

MOEDEC_API int moedec_tma_ring(const moedec_handle *h) {
    if (!h) return MOEDEC_ERR_INVALID_ARG;
    return h->maps.ok ? 1 : 0;
}

MOEDEC_API int moedec_get_routing(moedec_handle *h, int32_t *idx, float *w, int batch, void *stream) {
    if (!h || batch != h->last_batch || batch <= 0) return MOEDEC_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t n = (size_t)batch * h->d.k;
    cudaError_t e = cudaSuccess;
    if (idx) e = cudaMemcpyAsync(idx, h->ws.idx, n * sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess && w) e = cudaMemcpyAsync(w, h->ws.wts, n * sizeof(float), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return record_cuda(h, e);
    return read_device_error(h, s);
}

MOEDEC_API int moedec_get_taps(moedec_handle *h, float *logits, float *hlat, float *ylat, float *sh, float *up, int batch,
                               void *stream) {
    if (!h || batch != h->last_batch || batch <= 0) return MOEDEC_ERR_INVALID_ARG;
    if (up && !h->ws.up_tap) return MOEDEC_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Dims &d = h->d;
    const size_t B = (size_t)batch;
    struct {
        void *dst;
        const void *src;
        size_t bytes;
    } cp[] = {{logits, h->ws.logits, B * d.E * 4}, {hlat, h->ws.h, B * d.L * 4}, {ylat, h->ws.ylat, B * d.L * 4},
              {sh, h->ws.sh, B * d.H * 4}, {up, h->ws.up_tap, B * d.H * 4}};
    cudaError_t e = cudaSuccess;
    if (sh && !d.n_shared) e = cudaMemsetAsync(sh, 0, B * d.H * 4, s);
    for (auto &c : cp) {
        if (!c.dst || e != cudaSuccess) continue;
        if (c.src == h->ws.sh && !d.n_shared) continue;
        e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyDeviceToDevice, s);
    }
    if (e != cudaSuccess) return record_cuda(h, e);
    return read_device_error(h, s);
}

MOEDEC_API int moedec_get_scores(moedec_handle *h, float *scores, int batch, void *stream) {
    if (!h || !scores || batch != h->last_batch || batch <= 0) return MOEDEC_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_scores(h->ws.logits, scores, (size_t)batch * h->d.E, s);
    if (e != cudaSuccess) return record_cuda(h, e);
    return read_device_error(h, s);
}

MOEDEC_API int moedec_get_launch_counts(moedec_handle *h, uint64_t *launches, int *n_variants) {
    if (!h || !launches || !n_variants || *n_variants < 1) return MOEDEC_ERR_INVALID_ARG;
    const int n = *n_variants < 2 ? *n_variants : 2;
    for (int i = 0; i < n; ++i) launches[i] = h->launches[i];
    *n_variants = 2;
    return MOEDEC_OK;
}

MOEDEC_API int moedec_profile_enable(moedec_handle *h, int enable) {
    if (!h) return MOEDEC_ERR_INVALID_ARG;
    if (!enable) {  // stop recording; recorded marks stay readable
        h->profiling = false;
        return MOEDEC_OK;
    }
    for (auto &m : h->marks) {
        cudaEventSynchronize(m.stop);
        h->pool.push_back(m.start);
        h->pool.push_back(m.stop);
    }
    h->marks.clear();
    for (int i = 0; i < K_COUNT; ++i) {
        h->prof_ms[i] = 0.0;
        h->prof_n[i] = 0;
    }
    h->profiling = true;
    return MOEDEC_OK;
}

MOEDEC_API int moedec_profile_read(moedec_handle *h, double *total_ms, uint64_t *launches, const char **names, int *n) {
    if (!h || !n || *n < 0) return MOEDEC_ERR_INVALID_ARG;
    for (auto &m : h->marks) {
        cudaError_t e = cudaEventSynchronize(m.stop);
        float ms = 0.0f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, m.start, m.stop);
        if (e != cudaSuccess) return record_cuda(h, e);
        h->prof_ms[m.kind] += ms;
        h->prof_n[m.kind] += 1;
        h->pool.push_back(m.start);
        h->pool.push_back(m.stop);
    }
    h->marks.clear();
    const int cap = *n;
    for (int i = 0; i < K_COUNT && i < cap; ++i) {
        if (total_ms) total_ms[i] = h->prof_ms[i];
        if (launches) launches[i] = h->prof_n[i];
        if (names) names[i] = kKernelNames[i];
    }
    *n = K_COUNT;
    return MOEDEC_OK;
}

MOEDEC_API int moedec_get_trace(moedec_handle *h, uint64_t *out, int *n_cta, void *stream) {
    const int rows = h ? h->n_sm * kTraceRowsPerSm : 0;
    if (!h || !out || !n_cta || !h->ws.trace || *n_cta < rows) return MOEDEC_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(out, h->ws.trace, (size_t)rows * kTraceStamps * sizeof(uint64_t),
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return record_cuda(h, e);
    *n_cta = rows;
    return MOEDEC_OK;
}

MOEDEC_API int moedec_kernels_per_step(moedec_handle *h, int batch) {
    if (!h || batch <= 0) return 0;
    if (h->cfg.flags & MOEDEC_FLAG_MULTI_KERNEL) return kernels_per_step(h->d);
    return ((h->cfg.flags & MOEDEC_FLAG_STREAM) && stream_supports(h->d, batch)) ? kStreamLaunches : 1;
}

}  // extern "C"
