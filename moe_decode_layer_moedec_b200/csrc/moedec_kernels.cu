// moedec_kernels.cu -- sm_100a kernels of the sparse latent-MoE decode layer step.
//
// One step runs eight kernels (the step's parts as "快是可以生成的，可信只能证明（vLLM 重写 Kimi K3
// 解码路径…）" lists them in section 他们换掉了什么: router scoring and the latent projection, the
// experts, the shared expert on its own stream):
//
//   main stream   k_router_dn    router logits (fp64 m8n8k4 MMA) + h = W_dn x (bf16 MMA), split-K
//                 k_topk         sigmoid scores, top-k, weights, per-expert token buckets
//                 k_expert_gu    a = silu(G_e h) * (U_e h) per (expert, token)   MXFP4, fp16 MMA
//                 k_expert_down  y = D_e a                                       MXFP4, fp16 MMA
//                 k_combine      ylat = sum_r w_r y_r (fixed slot order)
//                 k_up           out = bf16(W_up ylat + sh)                      bf16 MMA, split-K
//   side stream   k_shared_gu    sh_a = silu(SG x) * (SU x)                      MXFP4, split-K
//                 k_shared_down  sh = SD sh_a                                    MXFP4, split-K
//
// Split-K partial sums are reduced by the last CTA of each row block (release/acquire ticket)
// in split order, so every result is deterministic.  Decode is HBM-bound; every kernel streams
// its weights once with 128-bit loads and keeps the decode tokens on chip.
#include <algorithm>

#include "moedec_device.cuh"
#include "moedec_internal.h"
#include "moedec_items.cuh"

namespace moedec {

// ---------------------------------------------------------------------------------------------
// multi-kernel schedule: one kernel per part of the step, ordered by the stream

// K1: router logits (fp64) and h = W_dn x, one grid.  Blocks [0, rt.blocks*rt.splits) are router
// items, the rest W_dn items.
template <int NT>
__global__ void __launch_bounds__(256) k_router_dn(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ unsigned s_flag;
    const int nrt = a.p.rt.blocks * a.p.rt.splits;
    if ((int)blockIdx.x < nrt)
        item_router<false>(a, blockIdx.x, smem, &s_flag);
    else
        item_dn<false, NT>(a, blockIdx.x - nrt, smem, &s_flag);
}

// top-k: one CTA of 256 threads per token; the last one builds the expert buckets
__global__ void __launch_bounds__(256) k_topk(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];  // candidate and bucket lists
    __shared__ TopkSmem t;
    item_topk<false>(a, blockIdx.x, t, smem);
}

// routed experts: every warp takes a contiguous range of (expert, 16-row) warp items
template <bool DOWN>
__global__ void __launch_bounds__(256) k_expert(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_ent[8][kExpertTokGroup];
    __shared__ int s_shift[8][kExpertTokGroup];
    const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem + (size_t)warp * expert_warp_smem(a.B));
    const int tiles = (DOWN ? a.d.L : a.d.I) / 16;
    const int n_items = __ldcg(a.ws.n_active) * tiles;
    const long long gw = (long long)blockIdx.x * nw + warp, tw = (long long)gridDim.x * nw;
    const int i0 = (int)(gw * n_items / tw), i1 = (int)((gw + 1) * n_items / tw);
    for (int item = i0; item < i1; ++item) warp_expert_item<false, DOWN>(a, xs, item, s_ent[warp], s_shift[warp]);
}

// combine: ylat[b][l] = sum_r w[b][r] y[b*K + r][l], slots in rank order; the token's staging
// maximum of h is cleared for the next step (its last reader, the gate/up kernel, is done)
__global__ void __launch_bounds__(256) k_combine(StepArgs a) {
    const int b = blockIdx.y, l = blockIdx.x * blockDim.x + threadIdx.x;
    if (l < a.d.L) combine_rows(a, b, l);
    if (blockIdx.x == 0 && threadIdx.x == 0) a.ws.ctl[a.p.ctl_hamax + b] = 0u;
}

template <int NT>
__global__ void __launch_bounds__(256) k_up(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ unsigned s_flag;
    __shared__ int s_ok;
    item_up<false, NT>(a, blockIdx.x, smem, &s_flag, &s_ok);
}

template <int NT>
__global__ void __launch_bounds__(256) k_shared_gu(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ unsigned s_flag;
    item_sgu<false, NT>(a, blockIdx.x, smem, &s_flag);
}

template <int NT, bool SPLIT>
__global__ void __launch_bounds__(256) k_shared_down(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ unsigned s_flag;
    __shared__ int s_ok;
    item_sd<false, NT, SPLIT>(a, blockIdx.x, smem, &s_flag, &s_ok);
}

// ---------------------------------------------------------------------------------------------
// create-time scan of the E8M0 scale bytes: any byte outside [104, 140] sets *bad.

__global__ void k_scale_check(const uint8_t *s, size_t n, unsigned *bad) {
    unsigned found = 0u;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const unsigned v = s[i];
        found |= (v < 104u || v > 140u) ? 1u : 0u;
    }
    if (__syncthreads_or(found) && threadIdx.x == 0) atomicOr(bad, 1u);
}

// ---------------------------------------------------------------------------------------------
// score tap: scores[i] = router_score(logits[i]) for n logits, the same function the top-k ranks by

__global__ void k_scores(const float *logits, float *scores, size_t n) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        scores[i] = router_score(__ldcg(logits + i));
}

// ---------------------------------------------------------------------------------------------
// host launchers


template <int NT>
static cudaError_t launch_router_dn_nt(const StepArgs &a, cudaStream_t s) {
    const size_t dn_smem = (size_t)8 * NT * bf16_pitch(a.p.dn.krange) * 2;
    const size_t sm = router_smem(a.p.rt.krange) > dn_smem ? router_smem(a.p.rt.krange) : dn_smem;
    const int grid = a.p.rt.blocks * a.p.rt.splits + a.p.dn.blocks * a.p.dn.splits;
    k_router_dn<NT><<<grid, 256, sm, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_router_dn(const StepArgs &a, cudaStream_t s) {
    switch (nt_for_cols(a.B)) {
        case 1: return launch_router_dn_nt<1>(a, s);
        case 2: return launch_router_dn_nt<2>(a, s);
        case 4: return launch_router_dn_nt<4>(a, s);
        default: return launch_router_dn_nt<8>(a, s);
    }
}

cudaError_t launch_topk(const StepArgs &a, cudaStream_t s) {
    k_topk<<<a.B, 256, topk_lists_smem(a.d.E, a.B), s>>>(a);
    return cudaGetLastError();
}

static cudaError_t launch_expert(const StepArgs &a, cudaStream_t s, int n_sm, bool down) {
    const size_t sm = 8 * expert_warp_smem(a.B);
    auto kern = down ? k_expert<true> : k_expert<false>;
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, sm);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    kern<<<n_sm * per_sm, 256, sm, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_expert_gate_up(const StepArgs &a, cudaStream_t s, int n_sm) { return launch_expert(a, s, n_sm, false); }
cudaError_t launch_expert_down(const StepArgs &a, cudaStream_t s, int n_sm) { return launch_expert(a, s, n_sm, true); }

cudaError_t launch_combine(const StepArgs &a, cudaStream_t s) {
    dim3 grid((a.d.L + 255) / 256, a.B);
    k_combine<<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

template <int NT>
static cudaError_t launch_up_nt(const StepArgs &a, cudaStream_t s) {
    const size_t sm = (size_t)8 * NT * bf16_pitch(up_chunk(NT, a.p.up.krange)) * 2;
    k_up<NT><<<a.p.up.blocks * a.p.up.splits, 256, sm, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_up(const StepArgs &a, cudaStream_t s) {
    switch (nt_for_cols(2 * a.B)) {
        case 1: return launch_up_nt<1>(a, s);
        case 2: return launch_up_nt<2>(a, s);
        case 4: return launch_up_nt<4>(a, s);
        case 8: return launch_up_nt<8>(a, s);
        default: return launch_up_nt<16>(a, s);
    }
}

template <int NT>
static cudaError_t launch_sgu_nt(const StepArgs &a, cudaStream_t s) {
    const size_t sm = (size_t)8 * NT * f16_pitch(a.p.sgu.krange) * 2;
    k_shared_gu<NT><<<a.p.sgu.blocks * a.p.sgu.splits, 256, sm, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_shared_gate_up(const StepArgs &a, cudaStream_t s) {
    switch (nt_for_cols(a.B)) {
        case 1: return launch_sgu_nt<1>(a, s);
        case 2: return launch_sgu_nt<2>(a, s);
        case 4: return launch_sgu_nt<4>(a, s);
        default: return launch_sgu_nt<8>(a, s);
    }
}

template <int NT, bool SPLIT>
static cudaError_t launch_sd_nt(const StepArgs &a, cudaStream_t s) {
    const size_t sm = (size_t)8 * NT * f16_pitch(a.p.sd.krange) * 2;
    k_shared_down<NT, SPLIT><<<a.p.sd.blocks * a.p.sd.splits, 256, sm, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_shared_down(const StepArgs &a, cudaStream_t s) {
    if (a.B <= 4) return launch_sd_nt<1, true>(a, s);
    switch (nt_for_cols(a.B)) {
        case 1: return launch_sd_nt<1, false>(a, s);
        case 2: return launch_sd_nt<2, false>(a, s);
        case 4: return launch_sd_nt<4, false>(a, s);
        default: return launch_sd_nt<8, false>(a, s);
    }
}

cudaError_t launch_scores(const float *logits, float *scores, size_t n, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    const int grid = (int)std::min<size_t>((n + 255) / 256, 1184);
    k_scores<<<grid, 256, 0, st>>>(logits, scores, n);
    return cudaGetLastError();
}

cudaError_t launch_scale_check(const uint8_t *sc, size_t n, unsigned *bad, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    k_scale_check<<<592, 256, 0, st>>>(sc, n, bad);
    return cudaGetLastError();
}

int kernels_per_step(const Dims &d) { return d.n_shared ? 8 : 6; }

// Raise the dynamic shared-memory limit of every kernel instantiation once per device (kept out
// of the launch path so that steps can be captured into CUDA graphs).
cudaError_t init_kernel_attributes() {
    const int lim = 160 * 1024;
    const void *fns[] = {
        (const void *)k_topk, (const void *)k_router_dn<1>, (const void *)k_router_dn<2>, (const void *)k_router_dn<4>,
        (const void *)k_router_dn<8>, (const void *)k_expert<true>, (const void *)k_expert<false>,
        (const void *)k_up<1>, (const void *)k_up<2>, (const void *)k_up<4>, (const void *)k_up<8>,
        (const void *)k_up<16>, (const void *)k_shared_gu<1>, (const void *)k_shared_gu<2>,
        (const void *)k_shared_gu<4>, (const void *)k_shared_gu<8>, (const void *)k_shared_down<1, true>,
        (const void *)k_shared_down<1, false>, (const void *)k_shared_down<2, false>,
        (const void *)k_shared_down<4, false>, (const void *)k_shared_down<8, false>};
    for (const void *f : fns) {
        cudaError_t err = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace moedec
