// moedec_fused_small.cu -- the decode layer step for batches of at most 4 tokens, one persistent
// kernel of independent warps.
//
// This is the small-matrix variant of the step: the Kimi K3 decode work picks a small-matrix
// kernel shape at batch 1-2 and split-K above ("快是可以生成的，可信只能证明（vLLM 重写 Kimi K3
// 解码路径…）", section 他们换掉了什么).  Decode at this batch is pure weight streaming, and on
// B200 a loaded HBM access takes on the order of 2 us, so an SM must keep ~64 KB of weights in
// flight.  Every work item is therefore a warp item (16 weight rows x a K range) that a warp
// streams on its own with a software-pipelined register ring; warps never wait for each other
// inside a phase, so while one warp starts an item the others keep the SM's loads in flight.
// A CTA only synchronises when it enters a phase, to stage that phase's activations (all tokens,
// full K) in shared memory once.  K splits of a tile are added by the warp that finishes last
// (per-tile ticket), in split order; routed experts read the staged columns of their own tokens.
//
// The grid is split in two groups of CTAs.  The routed chain (most CTAs) runs, in order:
//   router       8 rows x K/16           fp64 MMAs                    -> logits (per 8 rows)
//   top-k        one CTA per token       waits: all logits            -> routing, buckets
//   W_dn         16 rows x K/16          bf16 MMAs (not the top-k CTAs) -> h rows, max |h|
//   expert g/u   16 rows of one expert   waits: buckets, all of h     -> a rows, max |a|
//   expert down  16 rows of one expert   waits: its g/u rows          -> w * y rows added into ylat
//                                                                        (fp32 reductions)
//   W_up         16 rows x K/4           waits: ylat (sh: a tile's last split) -> out rows
// and the shared expert (an eighth of the grid) runs beside it:
//   shared g/u   16 rows x K/8, g and u  MXFP4, x staged as fp16      -> sh_a rows, max |sh_a|
//   shared down  16 rows x K             waits: all of sh_a           -> sh rows
// Every phase entry is a CTA-wide barrier (the phase's activations are staged once per CTA), so
// the shared parts, which nothing on the chain needs before W_up, must not sit between the
// chain's phases: a CTA there would hold the chain until its slowest shared item ends.
#include <algorithm>

#include "moedec_ring.cuh"

namespace moedec {

enum SmallQueue { QS_ROUTER = 0, QS_TOPK, QS_DN, QS_SGU, QS_EGU, QS_SD, QS_EDOWN, QS_UP };
constexpr int kWarps = 8;
constexpr size_t kSmallSmemLimit = 100 * 1024;  // dynamic shared memory of one CTA (two CTAs per SM)

// K chunk of the expert-down activation staging (per warp: the expert's entries, fp16 hi/lo):
// all of I when the eight warps' buffers fit, so that an item stages once and streams its
// weights in one pass; else 512
__host__ __device__ inline int edown_kc(int I, int B) {
    return (size_t)kWarps * 2 * B * f16_pitch(I) * 2 <= kSmallSmemLimit ? I : (kKChunk < I ? kKChunk : I);
}

// ---------------------------------------------------------------------------------------------
// one 16-row tile x one 8-column token tile; `col` is the staged column that this lane's MMA
// column (g) reads, or -1 for a zero operand

template <int D>
DEVI void s_bf16(const uint16_t *__restrict__ W, size_t ldw, int row0, int kg, int nrounds, const uint16_t *xs,
                 int pitch, int kofs, int col, float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const uint16_t *wa = W + (size_t)(row0 + g) * ldw + kg + 8 * q;
    const uint16_t *wb = wa + 8 * ldw;
    const uint16_t *xr = xs + (size_t)(col >= 0 ? col : 0) * pitch + kofs + 8 * q;
    float acc2[4] = {0.f, 0.f, 0.f, 0.f};
    uint4 A[D], Bm[D];
#pragma unroll
    for (int s = 0; s < D; ++s)
        if (s < nrounds) {
            A[s] = ldg_weights(wa + 32 * s);
            Bm[s] = ldg_weights(wb + 32 * s);
        }
    for (int r0 = 0; r0 < nrounds; r0 += D) {
#pragma unroll
        for (int s = 0; s < D; ++s) {
            const int r = r0 + s;
            if (r < nrounds) {
                const uint4 a = A[s], b = Bm[s];
                if (r + D < nrounds) {
                    A[s] = ldg_weights(wa + 32 * (r + D));
                    Bm[s] = ldg_weights(wb + 32 * (r + D));
                }
                uint4 xb = make_uint4(0u, 0u, 0u, 0u);
                if (col >= 0) xb = *reinterpret_cast<const uint4 *>(xr + 32 * r);
                mma_bf16(acc, a.x, b.x, a.y, b.y, xb.x, xb.y);
                mma_bf16(acc2, a.z, b.z, a.w, b.w, xb.z, xb.w);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] += acc2[j];
}

struct NoPre {
    DEVI void operator()() const {}
};

// pre() runs between the ring's first D rounds of weight loads and their first use: work that
// the weights do not depend on (a wait, the activation staging) overlaps their flight.
template <int D, bool PAIR, class Pre = NoPre>
DEVI void s_fp4(const uint8_t *__restrict__ Qa, const uint8_t *__restrict__ Sa, const uint8_t *__restrict__ Qb,
                const uint8_t *__restrict__ Sb, size_t ldq, size_t lds, int row0, int kg, int nrounds, const uint16_t *xs,
                int pitch, int kofs, int col, float (&acc)[4], float (&acc2)[4], Pre pre = Pre()) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const size_t ra = (size_t)(row0 + g), rb = ra + 8;
    const uint8_t *qa0 = Qa + ra * ldq + kg / 2 + 16 * q, *qa1 = Qa + rb * ldq + kg / 2 + 16 * q;
    const uint8_t *sa0 = Sa + ra * lds + kg / 32, *sa1 = Sa + rb * lds + kg / 32;
    const uint8_t *qb0 = qa0, *qb1 = qa1, *sb0 = sa0, *sb1 = sa1;
    if (PAIR) {
        qb0 = Qb + ra * ldq + kg / 2 + 16 * q;
        qb1 = Qb + rb * ldq + kg / 2 + 16 * q;
        sb0 = Sb + ra * lds + kg / 32;
        sb1 = Sb + rb * lds + kg / 32;
    }
    const uint16_t *xc = xs + (size_t)(col >= 0 ? col : 0) * pitch;
    const int ubase = kofs / 8 + 4 * q, flip = q >> 1, sh = 8 * q;
    float odd[4] = {0.f, 0.f, 0.f, 0.f};  // second MMA of each step pair: an independent chain
    Fp4Round fa[D], fb[PAIR ? D : 1];
#pragma unroll
    for (int s = 0; s < D; ++s)
        if (s < nrounds) {
            fp4_load(fa[s], qa0, qa1, sa0, sa1, s);
            if (PAIR) fp4_load(fb[PAIR ? s : 0], qb0, qb1, sb0, sb1, s);
        }
    pre();
    for (int r0 = 0; r0 < nrounds; r0 += D) {
#pragma unroll
        for (int s = 0; s < D; ++s) {
            const int r = r0 + s;
            if (r < nrounds) {
                const Fp4Round a = fa[s];
                Fp4Round b = a;
                if (PAIR) b = fb[PAIR ? s : 0];
                if (r + D < nrounds) {
                    fp4_load(fa[s], qa0, qa1, sa0, sa1, r + D);
                    if (PAIR) fp4_load(fb[PAIR ? s : 0], qb0, qb1, sb0, sb1, r + D);
                }
                const uint32_t fa0 = e8m0_to_f16x2((a.s0 >> sh) & 0xffu), fa1 = e8m0_to_f16x2((a.s1 >> sh) & 0xffu);
                const uint32_t fb0 = e8m0_to_f16x2((b.s0 >> sh) & 0xffu), fb1 = e8m0_to_f16x2((b.s1 >> sh) & 0xffu);
                const uint32_t wa0[4] = {a.c0.x, a.c0.y, a.c0.z, a.c0.w}, wa1[4] = {a.c1.x, a.c1.y, a.c1.z, a.c1.w};
                const uint32_t wb0[4] = {b.c0.x, b.c0.y, b.c0.z, b.c0.w}, wb1[4] = {b.c1.x, b.c1.y, b.c1.z, b.c1.w};
                const int u = ubase + 16 * r;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (col >= 0) v = *reinterpret_cast<const uint4 *>(xc + 8 * ((u + w) ^ flip));
                    uint32_t d0[4], d1[4];
                    fp4_decode_word(wa0[w], fa0, d0);
                    fp4_decode_word(wa1[w], fa1, d1);
                    mma_f16(acc, d0[0], d1[0], d0[1], d1[1], v.x, v.y);
                    if (PAIR) {
                        mma_f16(acc, d0[2], d1[2], d0[3], d1[3], v.z, v.w);
                        uint32_t e0[4], e1[4];
                        fp4_decode_word(wb0[w], fb0, e0);
                        fp4_decode_word(wb1[w], fb1, e1);
                        mma_f16(acc2, e0[0], e1[0], e0[1], e1[1], v.x, v.y);
                        mma_f16(acc2, e0[2], e1[2], e0[3], e1[3], v.z, v.w);
                    } else {
                        mma_f16(odd, d0[2], d1[2], d0[3], d1[3], v.z, v.w);
                    }
                }
            }
        }
    }
    if (!PAIR)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] += odd[j];
}

// ---------------------------------------------------------------------------------------------
// warp-level ticket: publish this warp's partial, count it; true (in every lane) for the warp
// that completes the tile, which then owns every partial of it

DEVI bool warp_ticket_last(unsigned *counter, unsigned expected) {
    __threadfence();
    __syncwarp();
    unsigned last = 0;
    if ((threadIdx.x & 31) == 0) {
        last = (atomicAdd(counter, 1u) == expected - 1u) ? 1u : 0u;
        if (last) *counter = 0u;  // every other split has counted already
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) __threadfence();  // acquire the other splits' partials
    return last != 0;
}

// ---------------------------------------------------------------------------------------------
// warp items

// router: 8 rows x K/s_rt (fp64 m8n8k4; slot q of step s of chunk c holds k = 32c + 8q + s).
// pre() runs once the ring's first D chunks are requested (the first item stages x there).
template <class Pre = NoPre>
DEVI void w_router(const StepArgs &a, int item, const uint16_t *xs, Pre pre = Pre()) {
    const int E = a.d.E, H = a.d.H, B = a.B;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int rg = item / a.p.s_rt, ks = item % a.p.s_rt;
    const int row = rg * 8 + g;
    const bool row_ok = row < E;
    const int KW = H / a.p.s_rt, k0 = ks * KW, nch = KW / 32;
    const uint16_t *rrow = a.w.router + (size_t)(row_ok ? row : 0) * H + k0 + 8 * q;
    const uint16_t *xr = xs + (size_t)(g < B ? g : 0) * bf16_pitch(H) + k0 + 8 * q;
    double c0 = 0.0, c1 = 0.0, d0 = 0.0, d1 = 0.0;
    constexpr int D = 8;
    uint4 A[D];
#pragma unroll
    for (int s = 0; s < D; ++s) A[s] = (row_ok && s < nch) ? ldg_weights(rrow + 32 * s) : make_uint4(0u, 0u, 0u, 0u);
    pre();
    for (int c0i = 0; c0i < nch; c0i += D) {
#pragma unroll
        for (int s = 0; s < D; ++s) {
            const int c = c0i + s;
            if (c < nch) {
                const uint4 Ac = A[s];
                if (c + D < nch) A[s] = row_ok ? ldg_weights(rrow + 32 * (c + D)) : make_uint4(0u, 0u, 0u, 0u);
                uint4 xb = make_uint4(0u, 0u, 0u, 0u);
                if (g < B) xb = *reinterpret_cast<const uint4 *>(xr + 32 * c);
                const double av[8] = {bf16_lo(Ac.x), bf16_hi(Ac.x), bf16_lo(Ac.y), bf16_hi(Ac.y),
                                      bf16_lo(Ac.z), bf16_hi(Ac.z), bf16_lo(Ac.w), bf16_hi(Ac.w)};
                const double xv[8] = {bf16_lo(xb.x), bf16_hi(xb.x), bf16_lo(xb.y), bf16_hi(xb.y),
                                      bf16_lo(xb.z), bf16_hi(xb.z), bf16_lo(xb.w), bf16_hi(xb.w)};
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    mma_f64(c0, c1, av[2 * s2], xv[2 * s2]);
                    mma_f64(d0, d1, av[2 * s2 + 1], xv[2 * s2 + 1]);
                }
            }
        }
    }
    c0 += d0;
    c1 += d1;
    // the K splits of a logit meet in fp64 reductions (the top-k rounds the sum to fp32 once
    // every router item has signalled, and clears the accumulator for the next step)
    if (row_ok) {
        if (2 * q < B) atomicAdd(a.ws.rt_acc + (size_t)(2 * q) * E + row, c0);
        if (2 * q + 1 < B) atomicAdd(a.ws.rt_acc + (size_t)(2 * q + 1) * E + row, c1);
    }
    if (!(a.flags & kFlagTestStall)) warp_signal_add(a.ws.ctl + CTL_RT_DONE, 1u);
}

// W_dn: 16 rows x K/s_dn
DEVI void w_dn(const StepArgs &a, int item, const uint16_t *xs) {
    const int L = a.d.L, H = a.d.H, B = a.B, maxB = a.d.max_batch;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int tile = item / a.p.s_dn, ks = item % a.p.s_dn, row0 = tile * 16;
    const int KW = H / a.p.s_dn, k0 = ks * KW;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    s_bf16<6>(a.w.w_dn, H, row0, k0, KW / 32, xs, bf16_pitch(H), k0, g < B ? g : -1, acc);
    float *part = a.ws.dn_part + (size_t)ks * maxB * L;
    for (int j = 0; j < 2; ++j)
        if (2 * q + j < B) {
            part[(size_t)(2 * q + j) * L + row0 + g] = acc[j];
            part[(size_t)(2 * q + j) * L + row0 + g + 8] = acc[2 + j];
        }
    if (!warp_ticket_last(a.ws.ctl + a.p.ctl_tk + (a.d.E + 7) / 8 + tile, a.p.s_dn)) return;
    // the lane's (token, row) sums: tokens 2q, 2q+1 x rows g, g+8, their loads in flight together
    const float *pp[4];
    bool okv[4];
    float sv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int b = 2 * q + (i >> 1), r = row0 + g + 8 * (i & 1);
        okv[i] = b < B;
        pp[i] = a.ws.dn_part + (okv[i] ? (size_t)b * L + r : 0);
    }
    sum_splits_batch<4, 8>(pp, okv, (size_t)maxB * L, a.p.s_dn, sv);
    for (int j = 0; j < 2; ++j) {
        const int b = 2 * q + j;
        float m = 0.0f;
        if (b < B)
            for (int h2 = 0; h2 < 2; ++h2) {
                const int r = row0 + g + 8 * h2;
                const float v = sv[2 * j + h2];
                a.ws.h[(size_t)b * L + r] = v;
                m = fmaxf(m, fabsf(v));
            }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        if (b < B && g == 0) atomicMax(a.ws.ctl + a.p.ctl_hamax + b, __float_as_uint(m));
    }
    warp_signal_add(a.ws.ctl + CTL_DN_DONE, 1u);
}

// shared gate/up: 16 rows of gate and up x K/s_sgu; x staged as fp16 * 2^-xshift[token]
DEVI void w_sgu(const StepArgs &a, int item, const uint16_t *xs16, const int *xshift) {
    const int H = a.d.H, Is = a.d.Is, B = a.B, maxB = a.d.max_batch;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int tile = item / a.p.s_sgu, ks = item % a.p.s_sgu, row0 = tile * 16;
    const int KW = H / a.p.s_sgu, k0 = ks * KW;
    float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
    s_fp4<3, true>(a.w.sh_gate_q, a.w.sh_gate_s, a.w.sh_up_q, a.w.sh_up_s, H / 2, H / 32, row0, k0, KW / 128, xs16,
                   f16_pitch(H), k0, g < B ? g : -1, accg, accu);
    float *part = a.ws.sgu_part + (size_t)ks * maxB * 2 * Is;
    for (int j = 0; j < 2; ++j)
        if (2 * q + j < B) {
            float *p = part + (size_t)(2 * q + j) * 2 * Is + row0;
            p[g] = accg[j];
            p[g + 8] = accg[2 + j];
            p[Is + g] = accu[j];
            p[Is + g + 8] = accu[2 + j];
        }
    const int tk = a.p.ctl_tk + (a.d.E + 7) / 8 + a.d.L / 16 + tile;
    if (!warp_ticket_last(a.ws.ctl + tk, a.p.s_sgu)) return;
    for (int j = 0; j < 2; ++j) {
        const int b = 2 * q + j;
        float m = 0.0f;
        if (b < B) {
            const float sc = exp2i(xshift[b]);
            const float *p = a.ws.sgu_part + (size_t)b * 2 * Is;
            // gate and up sums of rows g, g+8, their loads in flight together
            const float *pp[4] = {p + row0 + g, p + Is + row0 + g, p + row0 + g + 8, p + Is + row0 + g + 8};
            const bool okv[4] = {true, true, true, true};
            float sv[4];
            sum_splits_batch<4, 8>(pp, okv, (size_t)maxB * 2 * Is, a.p.s_sgu, sv);
            for (int h2 = 0; h2 < 2; ++h2) {
                const int r = row0 + g + 8 * h2;
                const float gs = sv[2 * h2] * sc;
                const float us = sv[2 * h2 + 1] * sc;
                const float v = gs / (1.0f + expf(-gs)) * us;
                a.ws.sh_a[(size_t)b * Is + r] = v;
                m = fmaxf(m, fabsf(v));
            }
        }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        if (b < B && g == 0) atomicMax(a.ws.ctl + a.p.ctl_shamax + b, __float_as_uint(m));
    }
    warp_signal_add(a.ws.ctl + CTL_SGU_DONE, 1u);
}

using RouteSmem = RouteTables<kSmallMaxBatch * kMaxTopK, kSmallMaxBatch * kMaxTopK>;

// this warp's entries of active expert slot j: ent[i] for i < cnt (lane i holds entry i)
struct Entries {
    int e, cnt, my_ent;
};

DEVI Entries warp_entries(const RouteSmem &rt, int j) {
    const int lane = threadIdx.x & 31;
    Entries r;
    r.e = rt.e[j];
    r.cnt = rt.cnt[j];
    r.my_ent = lane < r.cnt ? rt.ent[rt.off[j] + lane] : 0;
    return r;
}

// expert gate/up: 16 rows of active expert slot j x K/s_egu; h of all tokens staged as fp16
// hi/lo columns (2b, 2b+1) with a per-token exponent; the last split applies silu(gate) * up
DEVI void w_egu(const StepArgs &a, const RouteSmem &rt, int item, const uint16_t *hs, const int *hshift) {
    const int L = a.d.L, I = a.d.I, K = a.d.k, S = a.p.s_egu;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int tiles = I / 16, ks = item % S, jt = item / S, j = jt / tiles, row0 = (jt % tiles) * 16;
    const int KW = L / S, k0 = ks * KW;
    const Entries en = warp_entries(rt, j);
    // MMA column g: entry g/2, hi (g even) or lo (g odd) part of its token's staged h
    const int ent_g = __shfl_sync(0xffffffffu, en.my_ent, (g >> 1) & 31);
    const int col = (g >> 1) < en.cnt ? 2 * (ent_g / K) + (g & 1) : -1;
    const size_t eq = (size_t)en.e * I * (L / 2), es = (size_t)en.e * I * (L / 32);
    float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
    s_fp4<2, true>(a.w.gate_q + eq, a.w.gate_s + es, a.w.up_q + eq, a.w.up_s + es, L / 2, L / 32, row0, k0, KW / 128, hs,
                   f16_pitch(L), k0, col, accg, accu);
    // accumulator columns 2q, 2q+1 are entry q's hi and lo parts
    const int ent_q = __shfl_sync(0xffffffffu, en.my_ent, q);
    const bool ok = q < en.cnt;
    const size_t nent = (size_t)(a.B < kSmallMaxBatch ? a.B : kSmallMaxBatch) * K;  // entries per split
    if (ok) {
        float *p = a.ws.egu_part + ((size_t)ks * nent + ent_q) * 2 * I + row0;
        p[g] = accg[0] + accg[1];
        p[g + 8] = accg[2] + accg[3];
        p[I + g] = accu[0] + accu[1];
        p[I + g + 8] = accu[2] + accu[3];
    }
    const int tk = a.p.ctl_tk + (a.d.E + 7) / 8 + a.d.L / 16 + a.d.Is / 16 + 2 * (a.d.H / 16) + jt;
    if (S > 1 && !warp_ticket_last(a.ws.ctl + tk, (unsigned)S)) return;
    float m = 0.0f;
    if (ok) {
        const float sc = exp2i(hshift[ent_q / K]);
        const float *p = a.ws.egu_part + (size_t)ent_q * 2 * I + row0;
        const size_t st = nent * 2 * I;
        float *dst = a.ws.a + (size_t)ent_q * I + row0;
        // gate and up sums of rows g, g+8, their loads in flight together
        const float *pp[4] = {p + g, p + I + g, p + g + 8, p + I + g + 8};
        const bool okv[4] = {true, true, true, true};
        float sv[4];
        sum_splits_batch<4, 2>(pp, okv, st, S, sv);
        for (int h2 = 0; h2 < 2; ++h2) {
            const int r = g + 8 * h2;
            const float gs = sv[2 * h2] * sc;
            const float us = sv[2 * h2 + 1] * sc;
            const float v = gs / (1.0f + expf(-gs)) * us;
            dst[r] = v;
            m = fmaxf(m, fabsf(v));
        }
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
    if (ok && g == 0) atomicMax(a.ws.a_amax + ent_q, __float_as_uint(m));
    warp_signal_add(a.ws.ctl + a.p.ctl_gu + j, 1u);
}

// shared down: 16 rows x K/s_sd; sh_a staged as fp16 hi/lo columns (2b, 2b+1)
DEVI void w_sd(const StepArgs &a, int item, const uint16_t *ss, const int *sshift) {
    const int H = a.d.H, Is = a.d.Is, B = a.B, maxB = a.d.max_batch;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int tile = item / a.p.s_sd, ks = item % a.p.s_sd, row0 = tile * 16;
    const int KW = Is / a.p.s_sd, k0 = ks * KW;
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, dummy[4];
    s_fp4<5, false>(a.w.sh_down_q, a.w.sh_down_s, nullptr, nullptr, Is / 2, Is / 32, row0, k0, KW / 128, ss,
                    f16_pitch(Is), k0, g < 2 * B ? g : -1, acc, dummy);
    if (a.p.s_sd == 1) {  // the item covers all of K: the tile is final here (no partials, no ticket)
        if (q < B) {
            const float sc = exp2i(sshift[q]);
            a.ws.sh[(size_t)q * H + row0 + g] = (acc[0] + acc[1]) * sc;
            a.ws.sh[(size_t)q * H + row0 + g + 8] = (acc[2] + acc[3]) * sc;
        }
        warp_signal_add(a.ws.ctl + CTL_SD_DONE, 1u);
        return;
    }
    float *part = a.ws.sd_part + (size_t)ks * maxB * H;
    if (q < B) {
        part[(size_t)q * H + row0 + g] = acc[0] + acc[1];
        part[(size_t)q * H + row0 + g + 8] = acc[2] + acc[3];
    }
    const int tk = a.p.ctl_tk + (a.d.E + 7) / 8 + a.d.L / 16 + a.d.Is / 16 + tile;
    if (!warp_ticket_last(a.ws.ctl + tk, a.p.s_sd)) return;
    if (q < B) {
        const float sc = exp2i(sshift[q]);
        for (int h2 = 0; h2 < 2; ++h2) {
            const int r = row0 + g + 8 * h2;
            a.ws.sh[(size_t)q * H + r] = sum_splits(a.ws.sd_part + (size_t)q * H + r, (size_t)maxB * H, a.p.s_sd) * sc;
        }
    }
    warp_signal_add(a.ws.ctl + CTL_SD_DONE, 1u);
}

// expert down: 16 rows of L of active expert slot j, full K; a staged per warp (fp16 hi/lo of
// the expert's entries, 512 k at a time).  The combine is folded in: each entry's rows, times
// its routing weight, are added into ylat (fp32 reductions, so the order of the K slots of a
// token is not fixed), and the tile's ylat count grows by the number of entries.
DEVI bool w_edown(const StepArgs &a, const RouteSmem &rt, int item, uint16_t *ws) {
    const int L = a.d.L, I = a.d.I, K = a.d.k;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int tiles = L / 16, j = item / tiles, tile = item % tiles, row0 = tile * 16;
    const Entries en = warp_entries(rt, j);
    __shared__ int s_ent[kWarps][kMaxTopK], s_shift[kWarps][kMaxTopK];  // cnt <= B <= 4
    const int warp = threadIdx.x >> 5;
    const size_t eq = (size_t)en.e * L * (I / 2), es = (size_t)en.e * L * (I / 32);
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, dummy[4];
    const int kc = edown_kc(I, a.B);
    bool ok = true;
    int c0 = 0;
    // Only the activations wait for the expert's gate/up items: each pass issues its first
    // weight loads, then (first pass) waits and takes the entries' exponents, and stages its
    // K chunk of a.  After an abort the pass still runs on whatever is staged; nothing of it is
    // published.
    auto pre = [&]() {
        if (c0 == 0) {
            ok = warp_wait_geq(a, a.ws.ctl + a.p.ctl_gu + j, (unsigned)(I / 16));
            __syncwarp();
            if (lane < en.cnt) {
                s_ent[warp][lane] = en.my_ent;
                s_shift[warp][lane] = prescale_shift(__uint_as_float(__ldcg(a.ws.a_amax + en.my_ent)));
            }
        }
        __syncwarp();
        stage_f16_from_f32<true>(ws, f16_pitch(kc), a.ws.a, I, en.cnt, [&](int t) { return s_ent[warp][t]; },
                                 s_shift[warp], c0, kc, lane, 32);
        __syncwarp();
    };
    for (; c0 < I; c0 += kc)
        s_fp4<5, false>(a.w.down_q + eq, a.w.down_s + es, nullptr, nullptr, I / 2, I / 32, row0, c0, kc / 128, ws,
                        f16_pitch(kc), 0, g < 2 * en.cnt ? g : -1, acc, dummy, pre);
    if (!ok) return false;
    if (q < en.cnt) {
        const int ent = s_ent[warp][q];
        const float ws_ = rt.w[ent] * exp2i(s_shift[warp][q]);
        float *dst = a.ws.ylat + (size_t)(ent / K) * L + row0;
        atomicAdd(dst + g, (acc[0] + acc[1]) * ws_);
        atomicAdd(dst + g + 8, (acc[2] + acc[3]) * ws_);
    }
    warp_signal_add(a.ws.ctl + a.p.ctl_ylat + tile, (unsigned)en.cnt);
    return true;
}

// W_up: 16 rows x K/s_up; ylat staged as bf16 hi/lo columns (2b, 2b+1); out = bf16(. + sh).
// Returns false if the step was aborted while the tile's last split waited for sh.
DEVI bool w_up(const StepArgs &a, int item, const uint16_t *ys) {
    const int H = a.d.H, L = a.d.L, B = a.B, maxB = a.d.max_batch;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int tile = item / a.p.s_up, ks = item % a.p.s_up, row0 = tile * 16;
    const int KW = L / a.p.s_up, k0 = ks * KW;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    s_bf16<6>(a.w.w_up, L, row0, k0, KW / 32, ys, bf16_pitch(L), k0, g < 2 * B ? g : -1, acc);
    float *part = a.ws.up_part + (size_t)ks * maxB * H;
    if (q < B) {
        part[(size_t)q * H + row0 + g] = acc[0] + acc[1];
        part[(size_t)q * H + row0 + g + 8] = acc[2] + acc[3];
    }
    const int tk = a.p.ctl_tk + (a.d.E + 7) / 8 + a.d.L / 16 + a.d.Is / 16 + a.d.H / 16 + tile;
    if (!warp_ticket_last(a.ws.ctl + tk, a.p.s_up)) return true;
    // only the warp that completes the tile adds the shared expert's rows: the rest of W_up
    // streams while the shared expert finishes
    if (a.d.n_shared && !warp_wait_geq(a, a.ws.ctl + CTL_SD_DONE, (unsigned)(H / 16))) return false;
    if (q < B) {
        const float *pp[2] = {a.ws.up_part + (size_t)q * H + row0 + g, a.ws.up_part + (size_t)q * H + row0 + g + 8};
        const bool okv[2] = {true, true};
        float sv[2], shv[2];
        for (int h2 = 0; h2 < 2; ++h2) shv[h2] = a.d.n_shared ? __ldcg(a.ws.sh + (size_t)q * H + row0 + g + 8 * h2) : 0.0f;
        sum_splits_batch<2, 4>(pp, okv, (size_t)maxB * H, a.p.s_up, sv);
        for (int h2 = 0; h2 < 2; ++h2) {
            const int r = row0 + g + 8 * h2;
            if (a.ws.up_tap) a.ws.up_tap[(size_t)q * H + r] = sv[h2];
            if (a.out_f32) a.out_f32[(size_t)q * H + r] = sv[h2] + shv[h2];
            else a.out[(size_t)q * H + r] = f32_to_bf16_rne(sv[h2] + shv[h2]);
        }
    }
    return true;
}

// ---------------------------------------------------------------------------------------------
// the kernel

__host__ __device__ inline size_t fused_small_smem(const StepArgs &a, bool ring) {
    const int B = a.B;
    size_t m = (size_t)B * bf16_pitch(a.d.H) * 2;                        // x, bf16
    auto mx = [&](size_t v) { m = v > m ? v : m; };
    mx((size_t)B * f16_pitch(a.d.H) * 2);                                 // x, fp16
    mx((size_t)2 * B * f16_pitch(a.d.L) * 2);                             // h, fp16 hi/lo
    mx((size_t)2 * B * f16_pitch(a.d.Is) * 2);                            // sh_a, fp16 hi/lo
    mx((size_t)kWarps * 2 * B * f16_pitch(edown_kc(a.d.I, B)) * 2);  // a, per warp
    mx((size_t)2 * B * bf16_pitch(a.d.L) * 2);                            // ylat, bf16 hi/lo
    mx(topk_lists_smem(a.d.E, B));                                        // top-k lists
    if (ring) mx(ring_rows_smem(kRingStagesSmall, a.d));                    // expert TMA rings
    return m;
}

__global__ void __launch_bounds__(256, 2) k_fused_small(StepArgs a, const __grid_constant__ ExpertMaps maps) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ TopkSmem topk;
    __shared__ int s_shift[kSmallMaxBatch], s_ok;
    __shared__ unsigned s_amax[kSmallMaxBatch];
    __shared__ CtaTake claim;
    __shared__ RouteSmem route;
    __shared__ RingSync rs;
    __shared__ SegPlan segp;
    __shared__ int s_scan[32];
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    // routed experts through the per-warp TMA rings (as in the split-K step), when the maps exist
    constexpr int NSW = kRingStagesSmall;
    const bool use_ring = maps.ok != 0;
    uint8_t *ring = smem + ((1024u - (smem_u32(smem) & 1023u)) & 1023u);
    uint16_t *ring_xs = reinterpret_cast<uint16_t *>(ring + 8 * NSW * kRingBytes);
    __shared__ RingGroup ring_gr;
    unsigned ring_pos = 0;
    if (use_ring) ring_init(rs, maps);
    unsigned *ctl = a.ws.ctl;
    const int H = a.d.H, L = a.d.L, I = a.d.I, Is = a.d.Is, B = a.B, E = a.d.E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    bool alive = true;
    unsigned long long *trace = a.ws.trace ? a.ws.trace + (size_t)blockIdx.x * kTraceStamps : nullptr;
    auto stamp = [&](int i) {
        if (trace && threadIdx.x == 0) trace[i] = global_ns();
    };
    stamp(0);
    const int n_rt = (E + 7) / 8 * a.p.s_rt, n_dn = L / 16 * a.p.s_dn;
    const int n_sgu = a.d.n_shared ? Is / 16 * a.p.s_sgu : 0, n_sd = a.d.n_shared ? H / 16 * a.p.s_sd : 0;
    const int n_up = H / 16 * a.p.s_up;

    // The shared expert runs on its own CTAs (the last G_sh of the grid), so that the routed
    // chain (router -> top-k -> expert gate/up -> expert down -> W_up) never waits for the
    // CTA-wide phase entries of the shared parts; a CTA's items come from its static range of
    // its group's queues.
    const int G = gridDim.x;
    const int G_sh = a.d.n_shared ? max(1, G * kSmallSharedPer64 / 64) : 0, G_m = G - G_sh;
    // the top-k CTAs (one per token) take no W_dn items: all of h is awaited right after routing
    const int n_tk = B < G_m ? B : 0;
    const int c_m = blockIdx.x, c_sh = (int)blockIdx.x - G_m;
    const bool sh_cta = c_sh >= 0;
    // warps take items of queue qi until this CTA's range of it runs dry
    auto warp_queue = [&](int qi, int n, int c, int g, auto body) {
        int ok = 1;
        for (;;) {
            int it = -1;
            if (lane == 0) it = cta_take(claim, qi, n, c, g);
            it = __shfl_sync(0xffffffffu, it, 0);
            if (it < 0) break;
            if (!body(it)) {
                ok = 0;
                break;
            }
        }
        return ok;
    };
    auto stage_x_bf16 = [&]() {
        stage_bf16(xs, bf16_pitch(H), a.x, H, B, B, 0, H);
        __syncthreads();
    };

    cta_take_init(claim);
    if (sh_cta) {
        // ---- shared expert CTAs: gate/up on x, then down on sh_a (off the routed chain) ----
        if (threadIdx.x < B) s_amax[threadIdx.x] = 0u;
        __syncthreads();
        // x as fp16 with a per-token exponent over all of H
        for (int i = threadIdx.x; i < B * (H / 8); i += blockDim.x) {
            const int t = i / (H / 8), u = i % (H / 8);
            const uint4 v = *reinterpret_cast<const uint4 *>(a.x + (size_t)t * H + 8 * u);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            float m = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w4[k])), fabsf(bf16_hi(w4[k]))));
            atomicMax(s_amax + t, __float_as_uint(m));
        }
        __syncthreads();
        if (threadIdx.x < B) s_shift[threadIdx.x] = prescale_shift(__uint_as_float(s_amax[threadIdx.x]));
        __syncthreads();
        stage_f16_from_bf16(xs, f16_pitch(H), a.x, H, B, s_shift, 0, H);
        __syncthreads();
        warp_queue(QS_SGU, n_sgu, c_sh, G_sh, [&](int it) { w_sgu(a, it, xs, s_shift); return true; });
        stamp(4);
        // shared down: all of sh_a final; stage it (fp16 hi/lo)
        alive = cta_wait_geq(a, ctl + CTL_SGU_DONE, (unsigned)(Is / 16), &s_ok);
        if (alive) {
            if (threadIdx.x < B) s_shift[threadIdx.x] = prescale_shift(__uint_as_float(__ldcg(ctl + a.p.ctl_shamax + threadIdx.x)));
            __syncthreads();
            stage_f16_from_f32<true>(xs, f16_pitch(Is), a.ws.sh_a, Is, B, [](int t) { return t; }, s_shift, 0, Is);
            __syncthreads();
            warp_queue(QS_SD, n_sd, c_sh, G_sh, [&](int it) { w_sd(a, it, xs, s_shift); return true; });
        }
        stamp(7);
        prefetch_next_router(a, c_sh, G_sh);  // nothing left to do here: pull the next layer's router
    } else {
        // ---- routed chain CTAs ----
        // router and W_dn read x as bf16: each warp requests its first router item's rows, then
        // the CTA stages x (every warp takes part in the staging once, item or not)
        __syncthreads();  // the claim counters are initialised
        int it0 = -1;
        if (lane == 0) it0 = cta_take(claim, QS_ROUTER, n_rt, c_m, G_m);
        it0 = __shfl_sync(0xffffffffu, it0, 0);
        if (it0 >= 0) {
            w_router(a, it0, xs, [&]() { stage_x_bf16(); });
            warp_queue(QS_ROUTER, n_rt, c_m, G_m, [&](int it) { w_router(a, it, xs); return true; });
        } else {
            stage_x_bf16();
        }
        stamp(1);
        __syncthreads();
        for (int it = c_m; alive && it < B; it += G_m)
            alive = item_topk<true>(a, it, topk, smem, (unsigned)n_rt,  // the top-k CTAs take no W_dn item: xs is free
                                    trace ? a.ws.trace + (size_t)(G + blockIdx.x) * kTraceStamps : nullptr, a.ws.ylat,
                                    a.ws.rt_acc);
        stamp(2);
        if (alive && c_m >= n_tk)
            warp_queue(QS_DN, n_dn, c_m - n_tk, G_m - n_tk, [&](int it) { w_dn(a, it, xs); return true; });
        stamp(3);
        // expert gate/up: routing and all of h final; stage h of every token (fp16 hi/lo)
        if (alive) alive = cta_wait_geq(a, ctl + CTL_ROUTE_READY, 1u, &s_ok);
        stamp(11);
        if (alive) alive = cta_wait_geq(a, ctl + CTL_DN_DONE, (unsigned)(L / 16), &s_ok);
        stamp(5);
        auto range = [&](int n, int &lo, int &hi) {  // the chain CTAs' static split of a ring phase
            lo = (int)((long long)n * c_m / G_m);
            hi = (int)((long long)n * (c_m + 1) / G_m);
        };
        auto ring_counters = [&]() {
            for (int i = threadIdx.x; i < kRingMaxBlocks; i += blockDim.x) rs.blk[i] = 0u;
        };
        int n_act = 0;
        if (alive && use_ring) {
            n_act = __ldcg(a.ws.n_active);
            ring_plan(a, segp, s_scan, n_act);
            ring_counters();
            __syncthreads();
            int lo, hi;
            range((I / 8) * segp.ngroups, lo, hi);
            const bool ok = ring_rows<true, NSW>(a, maps, n_act, segp, rs, ring_gr, ring, ring_xs, lo, hi, ring_pos);
            alive = __syncthreads_and(ok ? 1 : 0) != 0;
        } else if (alive) {
            if (threadIdx.x < B) s_shift[threadIdx.x] = prescale_shift(__uint_as_float(__ldcg(ctl + a.p.ctl_hamax + threadIdx.x)));
            cta_load_routing(a, route);
            __syncthreads();
            stage_f16_from_f32<true>(xs, f16_pitch(L), a.ws.h, L, B, [](int t) { return t; }, s_shift, 0, L);
            __syncthreads();
            const int n = route.n_active * (I / 16) * a.p.s_egu;
            warp_queue(QS_EGU, n, c_m, G_m, [&](int it) { w_egu(a, route, it, xs, s_shift); return true; });
        }
        stamp(6);
        // expert down (ring phase, or per-warp staging of the expert's entries)
        if (alive && use_ring) {
            __syncthreads();
            ring_counters();
            __syncthreads();
            int lo, hi;
            range((L / 16) * segp.ngroups, lo, hi);
            const bool ok = ring_rows<false, NSW>(a, maps, n_act, segp, rs, ring_gr, ring, ring_xs, lo, hi, ring_pos);
            ring_publish_down(a, rs);
            alive = __syncthreads_and(ok ? 1 : 0) != 0;
        } else if (alive) {
            __syncthreads();
            const int n = route.n_active * (L / 16);
            uint16_t *ws = xs + (size_t)warp * 2 * B * f16_pitch(edown_kc(I, B));
            const int ok = warp_queue(QS_EDOWN, n, c_m, G_m, [&](int it) { return w_edown(a, route, it, ws); });
            alive = __syncthreads_and(ok) != 0;
        }
        stamp(8);
        // W_up: every ylat block complete (all B*k entries added); stage ylat (bf16 hi/lo).  The
        // shared expert's sh is awaited only by the warp that completes each tile
        if (alive) {
            int ok = 1;
            for (int blk = threadIdx.x; blk < L / 16; blk += blockDim.x)
                ok &= wait_geq(a, ctl + a.p.ctl_ylat + blk, (unsigned)(B * a.d.k)) ? 1 : 0;
            __threadfence();
            alive = __syncthreads_and(ok) != 0;
            if (alive) {
                stage_bf16split_from_f32(xs, bf16_pitch(L), a.ws.ylat, L, B, 0, L);
                __syncthreads();
                warp_queue(QS_UP, n_up, c_m, G_m, [&](int it) { return w_up(a, it, xs); });
            }
        }
    }
    stamp(9);
    // leave; the last CTA out clears the control block for the next step
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_ok = (atomicAdd(ctl + CTL_EXIT, 1u) == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    stamp(10);
    if (s_ok) {
        __threadfence();
        for (int i = threadIdx.x; i < CTL_FIXED; i += blockDim.x) ctl[i] = 0u;
        for (int i = threadIdx.x; i < E; i += blockDim.x) ctl[a.p.ctl_gu + i] = 0u;
        for (int i = threadIdx.x; i < B * (L / 16); i += blockDim.x) ctl[a.p.ctl_comb + i] = 0u;
        for (int i = threadIdx.x; i < L / 16; i += blockDim.x) ctl[a.p.ctl_ylat + i] = 0u;
        for (int i = threadIdx.x; i < B; i += blockDim.x) {
            ctl[a.p.ctl_hamax + i] = 0u;
            ctl[a.p.ctl_shamax + i] = 0u;
        }
        // tickets: all but the expert gate/up ones, then those of the active slots
        const int n_fixed_tk = (E + 7) / 8 + L / 16 + Is / 16 + 2 * (H / 16);
        const int n_egu_tk = __ldcg(a.ws.n_active) * (I / 16);
        for (int i = threadIdx.x; i < n_fixed_tk + n_egu_tk; i += blockDim.x) ctl[a.p.ctl_tk + i] = 0u;
    }
}

bool fused_small_supports(const Dims &d, int B) {
    // K splits of whole bf16 (32) and MXFP4 (128) rounds; at most 4 tokens so that the hi/lo
    // columns of every part fit one 8-column MMA tile
    const int kc = edown_kc(d.I, B);
    const size_t x16 = (size_t)B * (d.H + 32) * 2, hl = (size_t)2 * B * (d.L + 32) * 2;
    const size_t smem = std::max(std::max(x16, hl), std::max((size_t)2 * B * (d.Is + 16) * 2,
                                                             (size_t)kWarps * 2 * B * (kc + 16) * 2));
    return B <= kSmallMaxBatch && d.H % 128 == 0 && d.L % 128 == 0 && d.I % 128 == 0 && d.I % kc == 0 &&
           (d.n_shared == 0 || d.Is % 128 == 0) && d.k <= kMaxTopK && smem <= kSmallSmemLimit;
}

cudaError_t launch_fused_small(const StepArgs &a, const ExpertMaps &maps, cudaStream_t s, int n_sm) {
    int per_sm = 0;
    // one token: the register path (the ring's shared memory costs the register-fed phases more L1
    // than its few units per warp gain); two to four tokens: the TMA rings
    ExpertMaps m = maps;
    if (a.B < 2) m.ok = 0;
    const size_t sm = fused_small_smem(a, m.ok != 0);
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_fused_small, 256, sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (per_sm > kMaxCtasPerSm) per_sm = kMaxCtasPerSm;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_sm * per_sm);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_fused_small, a, m);
}

cudaError_t init_fused_small_attributes() {
    return cudaFuncSetAttribute(k_fused_small, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmallSmemLimit);
}

}  // namespace moedec
