// moedec_router.cuh -- one CTA of the router-logit product (fp64 m8n8k4 MMAs, split-K).
//
// Router scoring is its own part of the Kimi K3 decode step ("快是可以生成的，可信只能证明（vLLM 重写
// Kimi K3 解码路径…）", section 他们换掉了什么).  logit[b][e] = fp32(sum_j R[e][j] x[b][j]) with the
// exact bf16 products accumulated in fp64: each CTA sums one K range of 64 router rows into fp64
// partials, and the last CTA of a row block (ticket) adds the partials in split order and rounds
// once to fp32.
#pragma once

#include "moedec_device.cuh"
#include "moedec_internal.h"
#include "moedec_tiles.cuh"

namespace moedec {

// Returns true in every thread of the CTA that reduced its row block (the last of its splits).
DEVI bool router_block(const StepArgs &a, int bid, unsigned char *smem, unsigned *s_flag) {
    const int E = a.d.E, H = a.d.H, B = a.B, maxB = a.d.max_batch;
    const int rb = bid / a.p.rt.splits, ks = bid % a.p.rt.splits;
    const int KR = a.p.rt.krange, k0 = ks * KR;
    double *xs = reinterpret_cast<double *>(smem);  // [8][KR + 4]: pitch 32 bytes mod 128
    const int pitch = KR + 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int row = rb * kRouterRows + warp * 8 + g;
    const bool row_ok = row < E;
    const uint16_t *rrow = a.w.router + (size_t)(row_ok ? row : 0) * H + k0 + 8 * q;
    const int half_units = KR / 2;  // units of two doubles
    const int nchunks = KR / 32;    // <= 16
    for (int tg = 0; tg < B; tg += 8) {
        const int ntok = min(8, B - tg);
        // the first 8 chunks of the router rows are in flight while the tokens are staged; each
        // further chunk is requested 8 chunks ahead of its use (L1-allocating: token groups
        // after the first re-read these rows)
        uint4 A[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
            A[c] = (row_ok && c < nchunks) ? ldg_weights_l1(rrow + 32 * c) : make_uint4(0u, 0u, 0u, 0u);
        __syncthreads();
        for (int i = threadIdx.x; i < 8 * half_units; i += blockDim.x) {
            const int t = i / half_units, u = i % half_units;
            double2 v = make_double2(0.0, 0.0);
            if (t < ntok) {
                const uint32_t pr = *reinterpret_cast<const uint32_t *>(a.x + (size_t)(tg + t) * H + k0 + 2 * u);
                v.x = (double)bf16_lo(pr);
                v.y = (double)bf16_hi(pr);
            }
            *reinterpret_cast<double2 *>(xs + (size_t)t * pitch + 2 * swz(u)) = v;
        }
        __syncthreads();
        // m8n8k4 fp64: lane (g,q) holds A[row g][slot q] and B[slot q][token g]; MMA step s of
        // chunk c maps slot q to k = 32c + 8q + s.  Two accumulator pairs halve the MMA chain.
        double c0 = 0.0, c1 = 0.0, d0 = 0.0, d1 = 0.0;
        const double *xr = xs + (size_t)g * pitch;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            if (c < nchunks) {
                const uint4 Ac = A[c & 7];
                if (c + 8 < nchunks) A[c & 7] = row_ok ? ldg_weights_l1(rrow + 32 * (c + 8)) : make_uint4(0u, 0u, 0u, 0u);
                const double av[8] = {bf16_lo(Ac.x), bf16_hi(Ac.x), bf16_lo(Ac.y), bf16_hi(Ac.y),
                                      bf16_lo(Ac.z), bf16_hi(Ac.z), bf16_lo(Ac.w), bf16_hi(Ac.w)};
                double2 xv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int u = (16 * c + 4 * q + i) ^ (q >> 1);
                    xv[i] = *reinterpret_cast<const double2 *>(xr + 2 * u);
                }
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    mma_f64(c0, c1, av[2 * s2], xv[s2].x);
                    mma_f64(d0, d1, av[2 * s2 + 1], xv[s2].y);
                }
            }
        }
        c0 += d0;
        c1 += d1;
        if (row_ok) {
            if (2 * q < ntok) a.ws.rt_part[((size_t)ks * maxB + tg + 2 * q) * E + row] = c0;
            if (2 * q + 1 < ntok) a.ws.rt_part[((size_t)ks * maxB + tg + 2 * q + 1) * E + row] = c1;
        }
    }
    const bool last = cta_ticket_last(a.ws.tickets + a.p.ticket_rt + rb, a.p.rt.splits, s_flag);
    if (last) {
        for (int i = threadIdx.x; i < kRouterRows * B; i += blockDim.x) {
            const int r = rb * kRouterRows + (i % kRouterRows), b = i / kRouterRows;
            if (r >= E) continue;
            const double s = sum_splits(a.ws.rt_part + (size_t)b * E + r, (size_t)maxB * E, a.p.rt.splits);
            a.ws.logits[(size_t)b * E + r] = (float)s;
        }
    }
    return last;
}

}  // namespace moedec
