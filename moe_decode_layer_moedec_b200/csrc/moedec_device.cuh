// moedec_device.cuh -- device primitives of the sm_100a decode-step kernels.
//
// Design rules that every kernel here follows:
//   * Static weights are streamed with 128-bit non-coherent loads (ld.global.nc); they never
//     change while a handle exists.  Activations and partial sums are never read through the
//     non-coherent path: an activation written by another CTA of the same kernel is read only
//     after that kernel's release/acquire ticket, with an L1-bypassing load.  This is the load
//     rule the Kimi K3 decode work arrived at after an audit found a compiler moving activation
//     reads ahead of a synchronisation wait; only the static weights may use the early,
//     non-coherent load type ("NVIDIA uses a 12,000-line Megakernel to optimize Kimi K3
//     inference…", section 写在最后; "快是可以生成的，可信只能证明", section 踩过的坑).
//   * Matrix-vector work goes through warp-level tensor-core MMAs (m16n8k16 with fp32
//     accumulators, m8n8k4 in fp64 for the router), weights as the 16-row A operand and the
//     decode tokens as the 8-column B operand.  The point is instruction count, not FLOPs: one
//     MMA consumes 256 weight elements, and FP4 codes turn into fp16 pairs with one cvt each.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#define DEVI __device__ __forceinline__

namespace moedec {

// ---------------------------------------------------------------------------------------------
// memory

// Weight loads and MMAs are pure (no volatile): the compiler may hoist the loads of later rounds
// ahead of earlier MMAs, which is what keeps enough bytes in flight per warp.

// L2 policy for bytes read once per step (the weights): first to be evicted, so that the
// 148 MB or more of weights a step streams through the 126 MB L2 do not push out what is read
// again (the step's activations, partial sums, counters and the kernel's own code).
DEVI uint64_t l2_evict_first() {
    uint64_t pol;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// 16 bytes of static weights: non-coherent path, do not keep in L1, evict first from L2 (read
// once per step).
DEVI uint4 ldg_weights(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p), "l"(l2_evict_first()));
    return r;
}

// 16 bytes of static weights that a CTA re-reads (kept in L1).
DEVI uint4 ldg_weights_l1(const void *p) {
    uint4 r;
    asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

// 4 bytes of static weights (4-byte aligned).
DEVI uint32_t ldg_weights_u32(const void *p) {
    uint32_t r;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.u32 %0, [%1], %2;" : "=r"(r) : "l"(p), "l"(l2_evict_first()));
    return r;
}

DEVI uint32_t ldg_weight_byte(const uint8_t *p) {
    uint16_t r;
    asm("ld.global.nc.u8 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

// Bulk prefetch of `bytes` (multiple of 16, 16-byte aligned start) into L2; no data returns to the
// SM and nothing waits on it.  Issued for the weights of a CTA's or warp's next work item.
DEVI void prefetch_l2(const void *p, uint32_t bytes) {
    if (bytes == 0 || ((reinterpret_cast<uintptr_t>(p) | bytes) & 15u)) return;  // a hint: skip odd shapes
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------------------------------------
// number formats

// Four packed bytes (eight E2M1 codes, element 2i in the low nibble of byte i) -> four f16x2
// words; word i holds elements (2i, 2i+1) with element 2i in the low half.  The conversion is
// the sm_100a hardware cvt, exact for every code.
DEVI void e2m1x8_to_f16x2(uint32_t codes, uint32_t (&out)[4]) {
    asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
        "mov.b32 {c0, c1, c2, c3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, c0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, c1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, c2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, c3;\n\t}"
        : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
        : "r"(codes));
}

// E8M0 scale byte s -> 2^(s-127) as an f16 pair.  Exact for s in [104, 140]: the product with
// any E2M1 value is then an exact fp16 number (the create-time scan enforces that range).
DEVI uint32_t e8m0_to_f16x2(uint32_t s) {
    uint32_t h = (s >= 113u) ? ((s - 112u) << 10) : (1u << (s - 103u));
    return h | (h << 16);
}

DEVI uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

DEVI uint32_t pack_f16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

DEVI uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

DEVI float f16_lo(uint32_t v) {
    float f;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, l;\n\t}" : "=f"(f) : "r"(v));
    return f;
}

DEVI float f16_hi(uint32_t v) {
    float f;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, h;\n\t}" : "=f"(f) : "r"(v));
    return f;
}

DEVI float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
DEVI float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
DEVI float bf16_bits_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Exponent shift t with |v| * 2^-t <= 2^14 for |v| <= amax (fp16 staging stays far below 65504),
// clamped to [-100, 100] so that 2^t and 2^-t are normal floats.
DEVI int prescale_shift(float amax) {
    if (!(amax > 0.0f) || !isfinite(amax)) return 0;
    const int t = ilogbf(amax) - 13;
    return t < -100 ? -100 : (t > 100 ? 100 : t);
}

// Router score of one logit: fp32(1 / (1 + exp(-logit))) evaluated in fp64 (CUDA exp(double)),
// so that the fp32 result is the correctly rounded sigmoid except in astronomically rare cases.
// Every kernel that ranks experts, and the score tap, call this one function.
DEVI float router_score(float logit) { return (float)(1.0 / (1.0 + exp(-(double)logit))); }

DEVI uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// Shared-memory swizzle of staged fp16/fp64 activation units: within each group of 16 units of 16
// bytes, unit u is stored at u ^ bit3(u), so that the four lane quads of a phase hit distinct
// bank groups (see the staging layouts in moedec_kernels.cu).
__host__ __device__ __forceinline__ int swz(int u) { return u ^ ((u >> 3) & 1); }

// ---------------------------------------------------------------------------------------------
// tensor-core MMAs (warp-wide)

// D[16x8] += A[16x16] * B[16x8], fp16 inputs, fp32 accumulate.
DEVI void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulate.
DEVI void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D[8x8] += A[8x4] * B[4x8] in fp64.
DEVI void mma_f64(double &d0, double &d1, double a, double b) {
    asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                 : "+d"(d0), "+d"(d1)
                 : "d"(a), "d"(b));
}

// ---------------------------------------------------------------------------------------------
// bounded waits and tickets

// Release this CTA's global writes, take a ticket; returns true in every thread of the CTA that
// drew the last of `expected` tickets (that CTA then owns all partials).  The counter is reset
// by the last CTA so the same slot serves the next launch.
DEVI bool cta_ticket_last(unsigned int *counter, unsigned int expected, unsigned int *s_flag) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned int t = atomicAdd(counter, 1u);
        bool last = (t == expected - 1u);
        if (last) *counter = 0u;  // no other CTA touches it again in this launch
        *s_flag = last ? 1u : 0u;
    }
    __syncthreads();
    bool last = (*s_flag != 0u);
    if (last) __threadfence();  // acquire: partials of the other CTAs are visible from here on
    return last;
}

}  // namespace moedec
