// moedec_router.cuh -- one CTA of the router-logit product (fp64 m8n8k4 MMAs, split-K).
//
// Router scoring is its own part of the Kimi K3 decode step ("快是可以生成的，可信只能证明（vLLM 重写
// Kimi K3 解码路径…）", section 他们换掉了什么).  logit[b][e] = fp32(sum_j R[e][j] x[b][j]) with the
// exact bf16 products accumulated in fp64: each CTA sums one K range of 64 router rows into fp64
// partials, and the last CTA of a row block (ticket) adds the partials in split order and rounds
// once to fp32.  Within a K range a logit's products are added in k order (8 per chunk, chunk
// after chunk) into one fp64 accumulator.
#pragma once

#include "moedec_device.cuh"
#include "moedec_internal.h"
#include "moedec_tiles.cuh"

namespace moedec {

// Tokens per pass of a router item: the row block's weights are read once per pass (into
// registers) and meet the pass's tokens as four independent 8-token DMMA chains.
constexpr int kRouterPassTok = 32;
__host__ __device__ inline int router_xs_pitch(int krange) { return krange + 8; }  // bf16 elements
__host__ __device__ inline size_t router_smem(int krange) { return (size_t)kRouterPassTok * router_xs_pitch(krange) * 2; }

// Returns true in every thread of the CTA that reduced its row block (the last of its splits).
DEVI bool router_block(const StepArgs &a, int bid, unsigned char *smem, unsigned *s_flag) {
    const int E = a.d.E, H = a.d.H, B = a.B, maxB = a.d.max_batch;
    const int rb = bid / a.p.rt.splits, ks = bid % a.p.rt.splits;
    const int KR = a.p.rt.krange, k0 = ks * KR;
    // tokens x[t][k0 .. k0+KR) as bf16, token pitch KR + 8 elements: the 8 lanes of one slot q
    // (rows g = 0..7 of a token group) hit 8 distinct 16-byte bank groups
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    const int pitch = router_xs_pitch(KR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int row = rb * kRouterRows + warp * 8 + g;
    const bool row_ok = row < E;
    const uint16_t *rrow = a.w.router + (size_t)(row_ok ? row : 0) * H + k0 + 8 * q;
    const int nchunks = KR / 32;    // <= 16
    for (int tp = 0; tp < B; tp += kRouterPassTok) {
        const int nb = min(kRouterPassTok, B - tp), ngrp = (nb + 7) / 8;
        // the first 8 chunks of the router rows are in flight while the tokens are staged; each
        // further chunk is requested 8 chunks ahead of its use (L1-allocating: later passes
        // re-read these rows)
        uint4 A[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
            A[c] = (row_ok && c < nchunks) ? ldg_weights_l1(rrow + 32 * c) : make_uint4(0u, 0u, 0u, 0u);
        __syncthreads();
        stage_bf16(xs, pitch, a.x + (size_t)tp * H, H, nb, 8 * ngrp, k0, KR);
        __syncthreads();
        // m8n8k4 fp64: lane (g,q) holds A[row g][slot q] and B[slot q][token g]; MMA step s of
        // chunk c maps slot q to k = 32c + 8q + s.  One accumulator pair per 8-token group.
        double acc[kRouterPassTok / 8][2];
#pragma unroll
        for (int i = 0; i < kRouterPassTok / 8; ++i) acc[i][0] = acc[i][1] = 0.0;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            if (c < nchunks) {
                const uint4 Ac = A[c & 7];
                if (c + 8 < nchunks) A[c & 7] = row_ok ? ldg_weights_l1(rrow + 32 * (c + 8)) : make_uint4(0u, 0u, 0u, 0u);
                const double av[8] = {bf16_lo(Ac.x), bf16_hi(Ac.x), bf16_lo(Ac.y), bf16_hi(Ac.y),
                                      bf16_lo(Ac.z), bf16_hi(Ac.z), bf16_lo(Ac.w), bf16_hi(Ac.w)};
#pragma unroll
                for (int tg = 0; tg < kRouterPassTok / 8; ++tg) {
                    if (tg < ngrp) {
                        const uint4 xb = *reinterpret_cast<const uint4 *>(xs + (size_t)(8 * tg + g) * pitch + 32 * c + 8 * q);
                        const double xv[8] = {bf16_lo(xb.x), bf16_hi(xb.x), bf16_lo(xb.y), bf16_hi(xb.y),
                                              bf16_lo(xb.z), bf16_hi(xb.z), bf16_lo(xb.w), bf16_hi(xb.w)};
#pragma unroll
                        for (int s2 = 0; s2 < 8; ++s2) mma_f64(acc[tg][0], acc[tg][1], av[s2], xv[s2]);
                    }
                }
            }
        }
        if (row_ok) {
#pragma unroll
            for (int tg = 0; tg < kRouterPassTok / 8; ++tg) {
                const int t0 = tp + 8 * tg + 2 * q;
                if (t0 < B) a.ws.rt_part[((size_t)ks * maxB + t0) * E + row] = acc[tg][0];
                if (t0 + 1 < B) a.ws.rt_part[((size_t)ks * maxB + t0 + 1) * E + row] = acc[tg][1];
            }
        }
    }
    const bool last = cta_ticket_last(a.ws.tickets + a.p.ticket_rt + rb, a.p.rt.splits, s_flag);
    if (last) {
        constexpr int NP = 2;  // (row, token) sums per thread and pass, their loads in flight together
        for (int i0 = threadIdx.x; i0 < kRouterRows * B; i0 += NP * blockDim.x) {
            const double *pp[NP];
            bool ok[NP];
            size_t o[NP];
            double sum[NP];
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                const int i = i0 + j * blockDim.x, r = rb * kRouterRows + (i % kRouterRows), b = i / kRouterRows;
                ok[j] = i < kRouterRows * B && r < E;
                o[j] = ok[j] ? (size_t)b * E + r : 0;
                pp[j] = a.ws.rt_part + o[j];
            }
            sum_splits_batch<NP, 8>(pp, ok, (size_t)maxB * E, a.p.rt.splits, sum);
#pragma unroll
            for (int j = 0; j < NP; ++j)
                if (ok[j]) a.ws.logits[o[j]] = (float)sum[j];
        }
    }
    return last;
}

}  // namespace moedec
