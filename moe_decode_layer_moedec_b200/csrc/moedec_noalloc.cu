// moedec_noalloc.cu -- router logits for callers that must not allocate device memory.
//
// Same kernel body as the step's router part (moedec_router.cuh), but its split-K scratch (the
// fp64 partial sums and the per-row-block tickets) lives in one file-scope __device__ array of
// kNoAllocScratchBytes instead of a handle's cudaMalloc'd workspace.  The caller passes the
// router weights, the tokens and the output; nothing is allocated on any call.
#include <mutex>

#include "moedec.h"
#include "moedec_internal.h"
#include "moedec_router.cuh"

using namespace moedec;

namespace {

// 2 MiB per device: ticket words in the first 4 KiB, fp64 partials after them.
constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;
constexpr size_t kTicketBytes = 4096;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch per device, looked up once with that device current (a
// host-side reference to the array is only a stand-in and must never reach a kernel).
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

cudaError_t scratch_for_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

__global__ void __launch_bounds__(256) k_router_logits_noalloc(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ unsigned s_flag;
    router_block(a, blockIdx.x, smem, &s_flag);
}

int krange(int K) { return K % 512 == 0 ? 512 : K % 256 == 0 ? 256 : 128; }

}  // namespace

extern "C" MOEDEC_API int moedec_router_logits_noalloc(const uint16_t *router, const uint16_t *x, int n_experts,
                                                       int hidden, int batch, float *logits, void *stream) {
    if (batch < 0 || n_experts <= 0 || hidden <= 0) return MOEDEC_ERR_INVALID_ARG;
    if (batch == 0) return MOEDEC_OK;
    if (!router || !x || !logits || ((uintptr_t)router & 15u) || ((uintptr_t)x & 15u) || ((uintptr_t)logits & 3u))
        return MOEDEC_ERR_INVALID_ARG;
    if (hidden % 128 || n_experts > kMaxExperts) return MOEDEC_ERR_UNSUPPORTED;
    StepArgs a = {};
    a.p.rt.blocks = (n_experts + kRouterRows - 1) / kRouterRows;
    a.p.rt.krange = krange(hidden);
    a.p.rt.splits = hidden / a.p.rt.krange;
    a.p.ticket_rt = 0;
    const size_t partial_bytes = (size_t)a.p.rt.splits * batch * n_experts * sizeof(double);
    if ((size_t)a.p.rt.blocks * sizeof(unsigned) > kTicketBytes || kTicketBytes + partial_bytes > kNoAllocScratchBytes)
        return MOEDEC_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    cudaError_t e = scratch_for_current_device(&scratch);
    if (e != cudaSuccess) return MOEDEC_ERR_CUDA;
    // 32 tokens x (512 + 8) bf16 = 33 KB: within the default dynamic shared-memory limit
    const size_t smem = router_smem(a.p.rt.krange);
    a.d.E = n_experts;
    a.d.H = hidden;
    a.d.max_batch = batch;
    a.B = batch;
    a.x = x;
    a.w.router = router;
    a.ws.tickets = static_cast<unsigned *>(scratch);
    a.ws.rt_part = reinterpret_cast<double *>(static_cast<unsigned char *>(scratch) + kTicketBytes);
    a.ws.logits = logits;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // tickets must start at zero on every call (the scratch keeps whatever the last call left)
    e = cudaMemsetAsync(a.ws.tickets, 0, (size_t)a.p.rt.blocks * sizeof(unsigned), s);
    if (e != cudaSuccess) return MOEDEC_ERR_CUDA;
    k_router_logits_noalloc<<<a.p.rt.blocks * a.p.rt.splits, 256, smem, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? MOEDEC_OK : MOEDEC_ERR_CUDA;
}
