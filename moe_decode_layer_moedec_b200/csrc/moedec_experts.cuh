// moedec_experts.cuh -- routed-expert phases of the split-K step (batches above 4 tokens).
//
// At 5..64 tokens most active experts see one or two tokens and a few hot ones see tens, so the
// expert phases are weight streaming with almost no reuse: the MXFP4 gate/up rows (2.2 MB per
// expert) and down rows (1.1 MB) must flow through the SMs at HBM rate.  The layout of the work
// follows from that:
//   * Work items are (active expert slot j, token group g of at most 16 of its tokens, 128-row
//     block b), listed in that order.  CTA c owns the contiguous range [n c / G, n (c+1) / G) of
//     the list, so its range is a few runs ("segments") of consecutive blocks of one expert and
//     token group; no item is claimed through a global counter.
//   * A segment stages its tokens' activations in shared memory once (the CTA's three barriers),
//     and each warp streams its 16 rows of every block of the segment as one software-pipelined
//     register ring: the ring does not drain between tiles, only at segment ends, and the first
//     rounds of a segment's weights are in flight while its activations are staged.
//   * Expert down waits for its expert's gate/up tiles only (a per-expert counter), so the two
//     phases overlap across CTAs.
// The per-warp tile ring is the small-matrix kernel shape of the Kimi K3 decode work applied per
// expert; above two tokens its page has split-K instead ("快是可以生成的，可信只能证明（vLLM 重写
// Kimi K3 解码路径…）", section 他们换掉了什么); here the latent dimension is short enough (2048)
// that one warp covers the whole K of its rows and no split is needed.
#pragma once

#include "moedec_items.cuh"

namespace moedec {

// Tokens of one expert per group: 16 (two 8-column MMA tiles) in the one-CTA-per-SM layout, 8 (one
// tile, one code path, fewer registers) in the two-CTAs-per-SM layout.
constexpr int kSegTok = 16;

// One MXFP4 weight stream of a warp: `ntiles` 16-row tiles (tile t starts at row row0 + t *
// tstride), each over the whole K (rpt = K / 128 rounds of 16 code bytes and one scale byte per
// lane and row).  PAIR streams a second matrix of the same shape (gate and up) against the same
// token columns.  D rounds are in flight per lane; the ring runs across tile boundaries.
// pre() runs once the first D rounds are requested; epi(t, acc, acc2) runs after tile t.
template <int NT, bool PAIR, int D, class Pre, class Epi>
DEVI void ring_fp4_tiles(const uint8_t *__restrict__ Qa, const uint8_t *__restrict__ Sa, const uint8_t *__restrict__ Qb,
                         const uint8_t *__restrict__ Sb, int K, int row0, int tstride, int ntiles, const uint16_t *xs,
                         int pitch, int ncols, Pre pre, Epi epi) {
    constexpr int C = PAIR ? 1 : chains_fp4(NT);
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const size_t ldq = (size_t)K / 2, lds = (size_t)K / 32;
    const int rpt = K / 128, nr = ntiles * rpt;
    // load cursor: tile lt, round lkr; row pointers of rows g and g + 8 of tile lt
    int lt = 0, lkr = 0;
    auto load = [&](Fp4Round &f, const uint8_t *Q, const uint8_t *S) {
        const size_t ra = (size_t)(row0 + lt * tstride + g);
        f.c0 = ldg_weights(Q + ra * ldq + 64 * lkr + 16 * q);
        f.c1 = ldg_weights(Q + (ra + 8) * ldq + 64 * lkr + 16 * q);
        f.s0 = ldg_weights_u32(S + ra * lds + 4 * lkr);
        f.s1 = ldg_weights_u32(S + (ra + 8) * lds + 4 * lkr);
    };
    auto advance = [&]() {
        if (++lkr == rpt) {
            lkr = 0;
            ++lt;
        }
    };
    Fp4Round fa[D], fb[PAIR ? D : 1];
#pragma unroll
    for (int s = 0; s < D; ++s)
        if (s < nr) {
            load(fa[s], Qa, Sa);
            if (PAIR) load(fb[PAIR ? s : 0], Qb, Sb);
            advance();
        }
    pre();
    float ch[C][NT][4], acc2[NT][4];
#pragma unroll
    for (int c = 0; c < C; ++c)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) ch[c][nt][j] = acc2[nt][j] = 0.0f;
    const int flip = q >> 1, sh = 8 * q;
    int ct = 0, ckr = 0;  // compute cursor
    for (int r0 = 0; r0 < nr; r0 += D) {
#pragma unroll
        for (int s = 0; s < D; ++s) {
            if (r0 + s < nr) {
                const Fp4Round a = fa[s];
                Fp4Round b = a;
                if (PAIR) b = fb[PAIR ? s : 0];
                if (r0 + s + D < nr) {
                    load(fa[s], Qa, Sa);
                    if (PAIR) load(fb[PAIR ? s : 0], Qb, Sb);
                    advance();
                }
                const uint32_t fa0 = e8m0_to_f16x2((a.s0 >> sh) & 0xffu), fa1 = e8m0_to_f16x2((a.s1 >> sh) & 0xffu);
                const uint32_t fb0 = e8m0_to_f16x2((b.s0 >> sh) & 0xffu), fb1 = e8m0_to_f16x2((b.s1 >> sh) & 0xffu);
                const uint32_t wa0[4] = {a.c0.x, a.c0.y, a.c0.z, a.c0.w}, wa1[4] = {a.c1.x, a.c1.y, a.c1.z, a.c1.w};
                const uint32_t wb0[4] = {b.c0.x, b.c0.y, b.c0.z, b.c0.w}, wb1[4] = {b.c1.x, b.c1.y, b.c1.z, b.c1.w};
                const int u = 4 * q + 16 * ckr;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t d0[4], d1[4], e0[4], e1[4];
                    fp4_decode_word(wa0[w], fa0, d0);
                    fp4_decode_word(wa1[w], fa1, d1);
                    if (PAIR) {
                        fp4_decode_word(wb0[w], fb0, e0);
                        fp4_decode_word(wb1[w], fb1, e1);
                    }
                    const int uw = (u + w) ^ flip;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const int col = nt * 8 + g;
                        uint4 v = *reinterpret_cast<const uint4 *>(xs + (size_t)col * pitch + 8 * uw);
                        if (col >= ncols) v = make_uint4(0u, 0u, 0u, 0u);
                        mma_f16(ch[(2 * w) % C][nt], d0[0], d1[0], d0[1], d1[1], v.x, v.y);
                        mma_f16(ch[(2 * w + 1) % C][nt], d0[2], d1[2], d0[3], d1[3], v.z, v.w);
                        if (PAIR) {
                            mma_f16(acc2[nt], e0[0], e1[0], e0[1], e1[1], v.x, v.y);
                            mma_f16(acc2[nt], e0[2], e1[2], e0[3], e1[3], v.z, v.w);
                        }
                    }
                }
                if (++ckr == rpt) {
                    float acc[NT][4];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float t = ch[0][nt][j];
#pragma unroll
                            for (int c = 1; c < C; ++c) t += ch[c][nt][j];
                            acc[nt][j] = t;
                        }
                    epi(ct, acc, acc2);
#pragma unroll
                    for (int c = 0; c < C; ++c)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int j = 0; j < 4; ++j) ch[c][nt][j] = acc2[nt][j] = 0.0f;
                    ckr = 0;
                    ++ct;
                }
            }
        }
    }
}

// Token groups of the active expert slots, in slot order: slot j's groups are [gpref[j],
// gpref[j+1]), ceil(cnt_j / 16) of them.  An expert phase with nb 128-row blocks per expert has
// nb * ngroups items, item i = (group i / nb, block i % nb).
struct SegPlan {
    int gpref[kMaxExperts];
    int ngroups;
};

// all threads (blockDim.x == 256: four slots per thread, 1024 at most); a barrier must follow
template <int SEGTOK, class RT>
DEVI void seg_plan(SegPlan &sp, const RT &rt, int *s_warp) {
    int c[4], tot = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = 4 * threadIdx.x + i;
        c[i] = j < rt.n_active ? (rt.cnt[j] + SEGTOK - 1) / SEGTOK : 0;
        tot += c[i];
    }
    int n;
    int base = block_exclusive_scan(tot, s_warp, &n);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = 4 * threadIdx.x + i;
        if (j < rt.n_active) sp.gpref[j] = base;
        base += c[i];
    }
    if (threadIdx.x == 0) sp.ngroups = n;
}

// slot j of global group gi (gpref[j] <= gi < gpref[j+1]), by binary search over the slots
DEVI int seg_slot(const SegPlan &sp, int n_active, int gi) {
    int lo = 0, hi = n_active - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sp.gpref[mid] <= gi) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

struct SegSmem {
    int ent[kSegTok];    // entries of the segment's token group
    int shift[kSegTok];  // staging exponent of each column's source row
    float w[kSegTok];    // routing weight of each entry (down)
    int ok;
};

// The CTA's segments in order: body(j, g, b0, b1) for each maximal run of items of one token
// group (slot j, group g) inside [lo, hi) of an expert phase with nb blocks per expert.  Uniform
// over the CTA.  Returns false as soon as a body does.
template <class RT, class Body>
DEVI bool for_each_segment(const SegPlan &sp, const RT &rt, int nb, int lo, int hi, Body body) {
    int i = lo;
    while (i < hi) {
        const int gi = i / nb, b0 = i % nb, b1 = min(nb, b0 + (hi - i));
        const int j = seg_slot(sp, rt.n_active, gi);
        if (!body(j, gi - sp.gpref[j], b0, b1)) return false;
        i += b1 - b0;
    }
    return true;
}

// ---------------------------------------------------------------------------------------------
// expert gate/up: a = silu(G_e h) * (U_e h) for the entries of one token group, 128-row blocks
// [b0, b1) of expert slot j (warp w: rows 128 b + 16 w).  Activations: h of the group's tokens,
// fp16 hi/lo column pairs for at most 4 tokens, one fp16 column each otherwise (per-token
// power-of-two prescale).  Each warp adds its number of tiles to ctl_gu[j] once its a rows of the
// segment are written.

template <int NT, int SEGTOK, int D, class RT>
DEVI void seg_gate_up(const StepArgs &a, const RT &rt, SegSmem &ss, uint16_t *xs, int j, int g, int b0, int b1) {
    const int L = a.d.L, I = a.d.I, K = a.d.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gq = lane >> 2, q = lane & 3;
    const int e = rt.e[j], ntok = min(SEGTOK, rt.cnt[j] - g * SEGTOK), off = rt.off[j] + g * SEGTOK;
    const size_t eq = (size_t)e * I * (L / 2), es = (size_t)e * I * (L / 32);
    const int pitch = f16_pitch(L);
    const bool split = ntok <= 4;  // hi/lo column pairs (only with NT == 1)
    auto pre = [&]() {
        __syncthreads();  // every warp is done with the previous segment's staged columns
        if (threadIdx.x < ntok) {
            const int en = rt.ent[off + threadIdx.x];
            ss.ent[threadIdx.x] = en;
            ss.shift[threadIdx.x] = prescale_shift(__uint_as_float(__ldcg(a.ws.ctl + a.p.ctl_hamax + en / K)));
        }
        __syncthreads();
        if (NT == 1 && split)
            stage_f16_from_f32<true>(xs, pitch, a.ws.h, L, ntok, [&](int t) { return ss.ent[t] / K; }, ss.shift, 0, L);
        else
            stage_f16_from_f32<false>(xs, pitch, a.ws.h, L, ntok, [&](int t) { return ss.ent[t] / K; }, ss.shift, 0, L);
        __syncthreads();
    };
    auto epi = [&](int t, const float (&accg)[NT][4], const float (&accu)[NT][4]) {
        const int row0 = (b0 + t) * 128 + warp * 16;
        const bool sp = NT == 1 && split;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                if (sp && jj) break;
                const int tk = sp ? q : nt * 8 + 2 * q + jj;
                const bool ok = tk < ntok;
                const float sc = ok ? exp2i(ss.shift[tk]) : 0.0f;
                float g0, g1, u0, u1;
                if (sp) {
                    g0 = accg[nt][0] + accg[nt][1];
                    g1 = accg[nt][2] + accg[nt][3];
                    u0 = accu[nt][0] + accu[nt][1];
                    u1 = accu[nt][2] + accu[nt][3];
                } else {
                    g0 = accg[nt][jj];
                    g1 = accg[nt][2 + jj];
                    u0 = accu[nt][jj];
                    u1 = accu[nt][2 + jj];
                }
                g0 *= sc;
                g1 *= sc;
                u0 *= sc;
                u1 *= sc;
                const float a0 = g0 / (1.0f + expf(-g0)) * u0, a1 = g1 / (1.0f + expf(-g1)) * u1;
                float m = ok ? fmaxf(fabsf(a0), fabsf(a1)) : 0.0f;
                if (ok) {
                    float *dst = a.ws.a + (size_t)ss.ent[tk] * I + row0;
                    dst[gq] = a0;
                    dst[gq + 8] = a1;
                }
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
                if (ok && gq == 0) atomicMax(a.ws.a_amax + ss.ent[tk], __float_as_uint(m));
            }
        }
    };
    ring_fp4_tiles<NT, true, D>(a.w.gate_q + eq, a.w.gate_s + es, a.w.up_q + eq, a.w.up_s + es, L, b0 * 128 + warp * 16,
                                128, b1 - b0, xs, pitch, split ? 2 * ntok : ntok, pre, epi);
    // the warp's a rows of this segment are written: count its tiles (one fence per segment)
    warp_signal_add(a.ws.ctl + a.p.ctl_gu + j, (unsigned)(b1 - b0));
}

// MINB: CTAs per SM of the calling kernel (2: 8-token groups, a shallower ring, one code path)
template <int MINB, class RT>
DEVI void seg_gate_up_any(const StepArgs &a, const RT &rt, SegSmem &ss, uint16_t *xs, int j, int g, int b0, int b1) {
    if (MINB > 1) {
        seg_gate_up<1, 8, 2>(a, rt, ss, xs, j, g, b0, b1);
        return;
    }
    const int ntok = min(kSegTok, rt.cnt[j] - g * kSegTok);
    if (ntok <= 8) seg_gate_up<1, kSegTok, 4>(a, rt, ss, xs, j, g, b0, b1);
    else seg_gate_up<2, kSegTok, 2>(a, rt, ss, xs, j, g, b0, b1);
}

// ---------------------------------------------------------------------------------------------
// expert down: y = D_e a for the entries of one token group, 128-row blocks [b0, b1) of L; the
// combine is folded in (w * y added into ylat with fp32 reductions; after the segment each of the
// warp's 16-row tiles counts its tokens into ctl_ylat).  Waits for every gate/up tile of expert slot j (all its groups) first,
// with the segment's first weight rounds already in flight.  Returns false after an abort.

template <int NT, int SEGTOK, int D, class RT>
DEVI bool seg_down(const StepArgs &a, const RT &rt, SegSmem &ss, uint16_t *xs, int j, int g, int b0, int b1) {
    const int L = a.d.L, I = a.d.I, K = a.d.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gq = lane >> 2, q = lane & 3;
    const int e = rt.e[j], ntok = min(SEGTOK, rt.cnt[j] - g * SEGTOK), off = rt.off[j] + g * SEGTOK;
    const unsigned gu_tiles = (unsigned)((rt.cnt[j] + SEGTOK - 1) / SEGTOK * (I / 16));
    const size_t eq = (size_t)e * L * (I / 2), es = (size_t)e * L * (I / 32);
    const int pitch = f16_pitch(I);
    const bool split = NT == 1 && ntok <= 4;  // hi/lo column pairs
    bool ok = true;
    auto pre = [&]() {
        ok = cta_wait_geq(a, a.ws.ctl + a.p.ctl_gu + j, gu_tiles, &ss.ok);  // starts with a barrier
        if (threadIdx.x < ntok) {
            const int en = rt.ent[off + threadIdx.x];
            ss.ent[threadIdx.x] = en;
            ss.w[threadIdx.x] = rt.w[en];
            ss.shift[threadIdx.x] = prescale_shift(__uint_as_float(__ldcg(a.ws.a_amax + en)));
        }
        __syncthreads();
        if (ok && split)
            stage_f16_from_f32<true>(xs, pitch, a.ws.a, I, ntok, [&](int t) { return ss.ent[t]; }, ss.shift, 0, I);
        else if (ok)
            stage_f16_from_f32<false>(xs, pitch, a.ws.a, I, ntok, [&](int t) { return ss.ent[t]; }, ss.shift, 0, I);
        __syncthreads();
    };
    auto epi = [&](int t, const float (&acc)[NT][4], const float (&)[NT][4]) {
        if (!ok) return;
        const int row0 = (b0 + t) * 128 + warp * 16;
        auto add = [&](int tk, int r, float v) {
            atomicAdd(a.ws.ylat + (size_t)(ss.ent[tk] / K) * L + row0 + r, v * exp2i(ss.shift[tk]) * ss.w[tk]);
        };
        if (split) tile_foreach<NT, true>(acc, ntok, add);
        else tile_foreach<NT, false>(acc, ntok, add);
    };
    (void)gq;
    (void)q;
    ring_fp4_tiles<NT, false, D>(a.w.down_q + eq, a.w.down_s + es, nullptr, nullptr, I, b0 * 128 + warp * 16, 128,
                                 b1 - b0, xs, pitch, split ? 2 * ntok : ntok, pre, epi);
    // the warp's ylat additions of this segment are done: one fence, then each tile's count
    if (ok) {
        __threadfence();
        __syncwarp();
        if (lane == 0)
            for (int b = b0; b < b1; ++b) atomicAdd(a.ws.ctl + a.p.ctl_ylat + (b * 128 + warp * 16) / 16, (unsigned)ntok);
    }
    return ok;
}

template <int MINB, class RT>
DEVI bool seg_down_any(const StepArgs &a, const RT &rt, SegSmem &ss, uint16_t *xs, int j, int g, int b0, int b1) {
    if (MINB > 1) return seg_down<1, 8, 4>(a, rt, ss, xs, j, g, b0, b1);
    const int ntok = min(kSegTok, rt.cnt[j] - g * kSegTok);
    if (ntok <= 8) return seg_down<1, kSegTok, 8>(a, rt, ss, xs, j, g, b0, b1);
    return seg_down<2, kSegTok, 4>(a, rt, ss, xs, j, g, b0, b1);
}

// tokens per group of the layout with MINB CTAs per SM
__host__ __device__ constexpr int seg_tok(int minb) { return minb > 1 ? 8 : kSegTok; }

// shared memory of the staged activations of one segment (bytes)
__host__ __device__ inline size_t seg_smem(const Dims &d, int segtok) {
    const int K = d.L > d.I ? d.L : d.I;
    return (size_t)segtok * f16_pitch(K) * 2;
}

}  // namespace moedec
