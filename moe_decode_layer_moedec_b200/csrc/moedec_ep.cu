// moedec_ep.cu -- the exchange step of an expert-parallel layer.
//
// With the routed experts split over G ranks (each rank's handle a shard: its own contiguous
// range of experts and a slice of the shared expert's inner width), a step on rank r gives the
// fp32 partial out_r = W_up ylat_r + sh_r, where ylat_r sums the routed experts of rank r only and
// sh_r is the shared expert over its slice.  Both terms are linear in those pieces, so the layer's
// output is bf16(sum_r out_r).  The pages run the MoE tensor-parallel over the GPUs of one NVLink
// domain and write partial results into buffers every GPU can reach, followed by one fused
// reduction ("快是可以生成的，可信只能证明（vLLM 重写 Kimi K3 解码路径…）", section 他们换掉了什么);
// here the same exchange is two small kernels over peer memory:
//
//   k_ep_publish  after rank r's partial step (stream order): lane g of one warp fences at system
//                 scope and release-stores the step's epoch into flag slot r of rank g's flag array.
//   k_ep_combine  in every block, thread g waits (bounded, %globaltimer) until flag word g of this
//                 rank reaches the epoch (acquire, system scope), then the block sums the G partials element by
//                 element in rank order in fp32 and rounds once to bf16.  The partials are read
//                 with loads that bypass the non-coherent caches (ld.global.cv), since a peer
//                 may have written them while this kernel was already resident.
//
// The partial buffers of a step are reused two steps later (the caller alternates two by epoch
// parity): rank r writes buffer p again only in step e + 2, after its combine of step e + 1, which
// waited for every rank's publish of e + 1, which each rank issued after its own combine of step
// e had read buffer p.  Epochs only grow, so no flag is ever reset.  No TMA and no multicast: peer
// memory is read with plain loads.
#include <algorithm>

#include "moedec_device.cuh"
#include "moedec_internal.h"

namespace moedec {

namespace {

DEVI unsigned long long ep_now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

DEVI unsigned ld_acquire_sys(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

DEVI void st_release_sys(unsigned *p, unsigned v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// one warp: lane g fences and release-stores into rank g's flag array (the stores go out together)
__global__ void k_ep_publish(EpSlots slots, int world, unsigned epoch) {
    const int g = threadIdx.x;
    if (blockIdx.x == 0 && g < world) {
        __threadfence_system();
        st_release_sys(slots.p[g], epoch);
    }
}

__global__ void __launch_bounds__(256) k_ep_combine(EpParts parts, const unsigned *flags, int world, unsigned epoch,
                                                    size_t n4, uint16_t *out, unsigned *err, long long wait_ns) {
    // thread g polls rank g's flag word (all ranks' flags at once, not one after another)
    int ok = 1;
    if (flags && threadIdx.x < world) {
        const unsigned long long t0 = ep_now_ns();
        while ((int)(ld_acquire_sys(flags + threadIdx.x) - epoch) < 0) {
            if ((long long)(ep_now_ns() - t0) > wait_ns) {
                atomicOr(err, kErrTimeout);
                ok = 0;
                break;
            }
            __nanosleep(32);
        }
    }
    if (!__syncthreads_and(ok)) return;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        float4 s = __ldcv(reinterpret_cast<const float4 *>(parts.p[0]) + i);
        for (int g = 1; g < world; ++g) {
            const float4 v = __ldcv(reinterpret_cast<const float4 *>(parts.p[g]) + i);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        const uint2 o = make_uint2((unsigned)f32_to_bf16_rne(s.x) | ((unsigned)f32_to_bf16_rne(s.y) << 16),
                                   (unsigned)f32_to_bf16_rne(s.z) | ((unsigned)f32_to_bf16_rne(s.w) << 16));
        reinterpret_cast<uint2 *>(out)[i] = o;
    }
}

}  // namespace

cudaError_t launch_ep_publish(const EpSlots &slots, int world, unsigned epoch, cudaStream_t s) {
    k_ep_publish<<<1, 32, 0, s>>>(slots, world, epoch);
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const EpParts &parts, const unsigned *flags, int world, unsigned epoch, size_t n,
                              uint16_t *out, unsigned *err, long long wait_ns, int n_sm, cudaStream_t s) {
    const size_t n4 = n / 4;
    const size_t want = (n4 + 255) / 256;
    const int grid = (int)std::max<size_t>(1, std::min<size_t>(want, (size_t)n_sm * 4));
    k_ep_combine<<<grid, 256, 0, s>>>(parts, flags, world, epoch, n4, out, err, wait_ns);
    return cudaGetLastError();
}

}  // namespace moedec
