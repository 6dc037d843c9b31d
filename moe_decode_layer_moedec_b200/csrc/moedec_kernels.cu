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
#include "moedec_device.cuh"
#include "moedec_internal.h"
#include "moedec_router.cuh"

namespace moedec {

// ---------------------------------------------------------------------------------------------
// shared-memory layouts of staged activations
//
// fp16 columns feeding MXFP4 rows: a 128-element round is 16 units of 16 bytes; lane quad q
// reads units 4q..4q+3.  Unit u is stored at u ^ bit3(u), and the column pitch is 32 bytes mod
// 128, so the eight lanes of each shared-memory phase hit eight distinct bank groups.
__host__ __device__ __forceinline__ int f16_pitch(int kc) { return kc + 16; }   // halfs
// bf16 columns feeding bf16 rows: lane quad q reads unit 4r + q; pitch 64 bytes mod 128.
__host__ __device__ __forceinline__ int bf16_pitch(int kc) { return kc + 32; }  // elements

// K chunk of the up-projection so that its 8*NT staged bf16 columns stay near 70 KB.
__host__ __device__ constexpr int up_chunk(int nt, int krange) {
    return (nt <= 8 ? 512 : 256) < krange ? (nt <= 8 ? 512 : 256) : krange;
}

DEVI float exp2i(int t) { return __int_as_float((127 + t) << 23); }  // 2^t, |t| < 127

// block-wide max of non-negative floats (every thread gets the result); s_red has >= 32 slots
DEVI float block_max(float v, float *s_red) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
    __syncthreads();
    float m = 0.0f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, s_red[i]);
    return m;
}

// Exclusive prefix sum over the block of one int per thread; returns the prefix, *total gets the sum.
DEVI int block_exclusive_scan(int v, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    int base = 0, tot = 0;
    for (int i = 0; i < nw; ++i) {
        if (i < warp) base += s_warp[i];
        tot += s_warp[i];
    }
    *total = tot;
    return base + x - v;
}

// ---------------------------------------------------------------------------------------------
// warp tiles: 16 weight rows x (8*NT) token columns over a K range
//
// Fragment mapping (m16n8k16): lane = 4g + q.  A rows g and g+8, B column g, accumulators
// rows g / g+8 x columns 2q, 2q+1.  Within every MMA the k slots (2q,2q+1,2q+8,2q+9) of lane q
// are filled from that lane's own contiguous slice of the row, and the token operand is staged
// in the same permuted order, so each lane streams whole 16-byte pieces of its rows.

// bf16 rows W[row][k], k in [kg, kg + 32*nrounds); staged bf16 columns xs[col][k - kc0].
template <int NT>
DEVI void tile_bf16(const uint16_t *__restrict__ W, size_t ldw, int row0, int kg, int nrounds,
                    const uint16_t *xs, int pitch, int kofs, int ncols, float (&acc)[NT][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const uint16_t *wa = W + (size_t)(row0 + g) * ldw + kg + 8 * q;
    const uint16_t *wb = wa + 8 * ldw;
    const uint16_t *xr = xs + kofs + 8 * q;
#pragma unroll 4
    for (int r = 0; r < nrounds; ++r) {
        uint4 A = ldg_weights(wa + 32 * r), Bm = ldg_weights(wb + 32 * r);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int col = nt * 8 + g;
            uint4 xb = *reinterpret_cast<const uint4 *>(xr + (size_t)col * pitch + 32 * r);
            if (col >= ncols) xb = make_uint4(0u, 0u, 0u, 0u);
            mma_bf16(acc[nt], A.x, Bm.x, A.y, Bm.y, xb.x, xb.y);
            mma_bf16(acc[nt], A.z, Bm.z, A.w, Bm.w, xb.z, xb.w);
        }
    }
}

// MXFP4 rows: codes Q[row][k/2], scales S[row][k/32]; lane quad q owns 32-element block
// (kg/32 + 4r + q) of each round.  PAIR = gate and up rows share the token operand.
// The E8M0 scale is folded into the fp16 weights (exact for scale bytes 104..140).
template <int NT, bool PAIR>
DEVI void tile_fp4(const uint8_t *__restrict__ Qa, const uint8_t *__restrict__ Sa, const uint8_t *__restrict__ Qb,
                   const uint8_t *__restrict__ Sb, size_t ldq, size_t lds, int row0, int kg, int nrounds,
                   const uint16_t *xs, int pitch, int kofs, int ncols, float (&acc)[NT][4], float (&acc2)[NT][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const size_t ra = (size_t)(row0 + g), rb = ra + 8;
    const uint8_t *qa0 = Qa + ra * ldq + kg / 2 + 16 * q, *qa1 = Qa + rb * ldq + kg / 2 + 16 * q;
    const uint8_t *sa0 = Sa + ra * lds + kg / 32 + q, *sa1 = Sa + rb * lds + kg / 32 + q;
    const uint8_t *qb0 = nullptr, *qb1 = nullptr, *sb0 = nullptr, *sb1 = nullptr;
    if (PAIR) {
        qb0 = Qb + ra * ldq + kg / 2 + 16 * q;
        qb1 = Qb + rb * ldq + kg / 2 + 16 * q;
        sb0 = Sb + ra * lds + kg / 32 + q;
        sb1 = Sb + rb * lds + kg / 32 + q;
    }
    const int ubase = kofs / 8 + 4 * q, flip = q >> 1;
#pragma unroll 2
    for (int r = 0; r < nrounds; ++r) {
        const uint4 ca0 = ldg_weights(qa0 + 64 * r), ca1 = ldg_weights(qa1 + 64 * r);
        const uint32_t fa0 = e8m0_to_f16x2(ldg_weight_byte(sa0 + 4 * r)), fa1 = e8m0_to_f16x2(ldg_weight_byte(sa1 + 4 * r));
        uint4 cb0 = make_uint4(0u, 0u, 0u, 0u), cb1 = cb0;
        uint32_t fb0 = 0u, fb1 = 0u;
        if (PAIR) {
            cb0 = ldg_weights(qb0 + 64 * r);
            cb1 = ldg_weights(qb1 + 64 * r);
            fb0 = e8m0_to_f16x2(ldg_weight_byte(sb0 + 4 * r));
            fb1 = e8m0_to_f16x2(ldg_weight_byte(sb1 + 4 * r));
        }
        const uint32_t wa0[4] = {ca0.x, ca0.y, ca0.z, ca0.w}, wa1[4] = {ca1.x, ca1.y, ca1.z, ca1.w};
        const uint32_t wb0[4] = {cb0.x, cb0.y, cb0.z, cb0.w}, wb1[4] = {cb1.x, cb1.y, cb1.z, cb1.w};
        // word w of the lane's 16-byte block holds MMA steps 2w and 2w+1; the matching token
        // values are unit w of the lane's 64-byte activation slice.
        const int u = (ubase + 16 * r) ;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint32_t d0[4], d1[4], e0[4], e1[4];
            e2m1x8_to_f16x2(wa0[w], d0);
            e2m1x8_to_f16x2(wa1[w], d1);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                d0[i] = hmul2(d0[i], fa0);
                d1[i] = hmul2(d1[i], fa1);
            }
            if (PAIR) {
                e2m1x8_to_f16x2(wb0[w], e0);
                e2m1x8_to_f16x2(wb1[w], e1);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    e0[i] = hmul2(e0[i], fb0);
                    e1[i] = hmul2(e1[i], fb1);
                }
            }
            const int uw = (u + w) ^ flip;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int col = nt * 8 + g;
                uint4 v = *reinterpret_cast<const uint4 *>(xs + (size_t)col * pitch + 8 * uw);
                if (col >= ncols) v = make_uint4(0u, 0u, 0u, 0u);
                mma_f16(acc[nt], d0[0], d1[0], d0[1], d1[1], v.x, v.y);
                mma_f16(acc[nt], d0[2], d1[2], d0[3], d1[3], v.z, v.w);
                if (PAIR) {
                    mma_f16(acc2[nt], e0[0], e1[0], e0[1], e1[1], v.x, v.y);
                    mma_f16(acc2[nt], e0[2], e1[2], e0[3], e1[3], v.z, v.w);
                }
            }
        }
    }
}

// Column value of accumulator tile entry: SPLIT columns (2i, 2i+1) are token i's hi and lo parts.
// Calls fn(token, row_in_tile, value) for every (token < ntok, row) this lane holds.
template <int NT, bool SPLIT, class F>
DEVI void tile_foreach(const float (&acc)[NT][4], int ntok, F fn) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        if (SPLIT) {
            const int t = nt * 4 + q;
            if (t < ntok) {
                fn(t, g, acc[nt][0] + acc[nt][1]);
                fn(t, g + 8, acc[nt][2] + acc[nt][3]);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int t = nt * 8 + 2 * q + j;
                if (t < ntok) {
                    fn(t, g, acc[nt][j]);
                    fn(t, g + 8, acc[nt][2 + j]);
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------------------
// staging

// bf16 tokens x[b][k0 .. k0+kc) -> xs[col b][0..kc) (bf16 layout), columns [ntok, ncols_pad) zero.
DEVI void stage_bf16(uint16_t *xs, int pitch, const uint16_t *x, size_t ldx, int ntok, int ncols_pad, int k0, int kc) {
    const int units = kc / 8;
    for (int i = threadIdx.x; i < ncols_pad * units; i += blockDim.x) {
        const int col = i / units, u = i % units;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (col < ntok) v = *reinterpret_cast<const uint4 *>(x + (size_t)col * ldx + k0 + 8 * u);
        *reinterpret_cast<uint4 *>(xs + (size_t)col * pitch + 8 * u) = v;
    }
}

// fp32 vectors src[rowof(i)][k0 .. k0+kc) * 2^-shift[i] -> fp16 columns (fp16 layout, swizzled).
// SPLIT: column 2i = fp16(v), 2i+1 = fp16(v - fp16(v)).  Reads with L1-bypassing loads.
template <bool SPLIT, class RowOf>
DEVI void stage_f16_from_f32(uint16_t *xs, int pitch, const float *src, size_t lds, int ntok, RowOf rowof,
                             const int *shift, int k0, int kc) {
    const int units = kc / 8;
    for (int i = threadIdx.x; i < ntok * units; i += blockDim.x) {
        const int t = i / units, u = i % units;
        const float *p = src + (size_t)rowof(t) * lds + k0 + 8 * u;
        const float4 v0 = __ldcg(reinterpret_cast<const float4 *>(p));
        const float4 v1 = __ldcg(reinterpret_cast<const float4 *>(p) + 1);
        const float sc = exp2i(-shift[t]);
        const float v[8] = {v0.x * sc, v0.y * sc, v0.z * sc, v0.w * sc, v1.x * sc, v1.y * sc, v1.z * sc, v1.w * sc};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            hi[j] = pack_f16x2(v[2 * j], v[2 * j + 1]);
            if (SPLIT) lo[j] = pack_f16x2(v[2 * j] - f16_lo(hi[j]), v[2 * j + 1] - f16_hi(hi[j]));
        }
        const int col = SPLIT ? 2 * t : t;
        *reinterpret_cast<uint4 *>(xs + (size_t)col * pitch + 8 * swz(u)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        if (SPLIT)
            *reinterpret_cast<uint4 *>(xs + (size_t)(col + 1) * pitch + 8 * swz(u)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// bf16 tokens * 2^-shift -> fp16 columns (exact in fp16 for all but values 2^-38 below the
// column's maximum), fp16 layout, swizzled.
DEVI void stage_f16_from_bf16(uint16_t *xs, int pitch, const uint16_t *x, size_t ldx, int ntok, const int *shift,
                              int k0, int kc) {
    const int units = kc / 8;
    for (int i = threadIdx.x; i < ntok * units; i += blockDim.x) {
        const int t = i / units, u = i % units;
        const uint4 v = *reinterpret_cast<const uint4 *>(x + (size_t)t * ldx + k0 + 8 * u);
        const float sc = exp2i(-shift[t]);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = pack_f16x2(bf16_lo(w[j]) * sc, bf16_hi(w[j]) * sc);
        *reinterpret_cast<uint4 *>(xs + (size_t)t * pitch + 8 * swz(u)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// fp32 vectors -> bf16 hi/lo column pairs (bf16 layout): column 2i = bf16(v), 2i+1 = bf16(v - hi).
DEVI void stage_bf16split_from_f32(uint16_t *xs, int pitch, const float *src, size_t lds, int ntok, int k0, int kc) {
    const int units = kc / 8;
    for (int i = threadIdx.x; i < ntok * units; i += blockDim.x) {
        const int t = i / units, u = i % units;
        const float *p = src + (size_t)t * lds + k0 + 8 * u;
        const float4 v0 = __ldcg(reinterpret_cast<const float4 *>(p));
        const float4 v1 = __ldcg(reinterpret_cast<const float4 *>(p) + 1);
        const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            hi[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
            lo[j] = pack_bf16x2(v[2 * j] - bf16_lo(hi[j]), v[2 * j + 1] - bf16_hi(hi[j]));
        }
        *reinterpret_cast<uint4 *>(xs + (size_t)(2 * t) * pitch + 8 * u) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(xs + (size_t)(2 * t + 1) * pitch + 8 * u) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// ---------------------------------------------------------------------------------------------
// K1: router logits (fp64) and h = W_dn x, one grid.  Blocks [0, rt.blocks*rt.splits) are router
// blocks (64 rows, one K range), the rest W_dn blocks (128 rows, one K range).

template <int NT>
DEVI void dn_block(const StepArgs &a, int bid, unsigned char *smem, unsigned *s_flag) {
    const int L = a.d.L, H = a.d.H, B = a.B, maxB = a.d.max_batch;
    const int rb = bid / a.p.dn.splits, ks = bid % a.p.dn.splits;
    const int KR = a.p.dn.krange, k0 = ks * KR;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    const int pitch = bf16_pitch(KR);
    stage_bf16(xs, pitch, a.x, H, B, 8 * NT, k0, KR);
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    const int row0 = rb * kDenseRows + warp * 16;
    if (row0 < L) {
        float acc[NT][4] = {};
        tile_bf16<NT>(a.w.w_dn, H, row0, k0, KR / 32, xs, pitch, 0, B, acc);
        float *part = a.ws.dn_part + (size_t)ks * maxB * L;
        tile_foreach<NT, false>(acc, B, [&](int t, int r, float v) { part[(size_t)t * L + row0 + r] = v; });
    }
    if (cta_ticket_last(a.ws.tickets + a.p.ticket_dn + rb, a.p.dn.splits, s_flag)) {
        for (int i = threadIdx.x; i < kDenseRows * B; i += blockDim.x) {
            const int r = rb * kDenseRows + (i % kDenseRows), b = i / kDenseRows;
            if (r >= L) continue;
            float s = 0.0f;
            for (int k = 0; k < a.p.dn.splits; ++k) s += __ldcg(a.ws.dn_part + ((size_t)k * maxB + b) * L + r);
            a.ws.h[(size_t)b * L + r] = s;
        }
    }
}

template <int NT>
__global__ void __launch_bounds__(256) k_router_dn(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ unsigned s_flag;
    const int nrt = a.p.rt.blocks * a.p.rt.splits;
    if ((int)blockIdx.x < nrt)
        router_block(a, blockIdx.x, smem, &s_flag);
    else
        dn_block<NT>(a, blockIdx.x - nrt, smem, &s_flag);
}

// ---------------------------------------------------------------------------------------------
// top-k: one CTA per token, one thread per expert.

__global__ void __launch_bounds__(1024) k_topk(StepArgs a) {
    const int E = a.d.E, K = a.d.k, B = a.B, L = a.d.L;
    const int b = blockIdx.x, e = threadIdx.x;
    __shared__ int s_warp[32];
    __shared__ unsigned s_key[kMaxTopK];
    __shared__ int s_e[kMaxTopK];
    __shared__ float s_rank_s[kMaxTopK];
    __shared__ int s_rank_e[kMaxTopK];
    __shared__ float s_red[32];
    __shared__ unsigned s_flag;
    __shared__ unsigned long long s_mask[kMaxExperts];
    __shared__ int s_off[kMaxExperts];

    const bool valid = e < E;
    float score = 0.0f;
    if (valid) {
        const float lg = __ldcg(a.ws.logits + (size_t)b * E + e);
        score = (float)(1.0 / (1.0 + exp(-(double)lg)));
    }
    // Non-negative fp32 scores order like their bit patterns.
    const uint32_t key = (valid && score >= 0.0f) ? __float_as_uint(score) : 0u;
    // T = largest t with #{key >= t} >= K  (the K-th largest key)
    uint32_t lo = 0u, hi = 0x3f800001u;
    while (hi - lo > 1u) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (__syncthreads_count(valid && key >= mid) >= K) lo = mid; else hi = mid;
    }
    const uint32_t T = lo;
    const bool gt = valid && key > T, eq = valid && key == T;
    const int n_gt = __syncthreads_count(gt);
    int tot;
    const int eq_rank = block_exclusive_scan(eq ? 1 : 0, s_warp, &tot);
    const bool sel = gt || (eq && eq_rank < K - n_gt);
    const int pos = block_exclusive_scan(sel ? 1 : 0, s_warp, &tot);
    if (sel) {
        s_key[pos] = key;
        s_e[pos] = e;
    }
    __syncthreads();
    if (e < K) {
        const uint32_t mk = s_key[e];
        const int me = s_e[e];
        int rank = 0;
        for (int j = 0; j < K; ++j) rank += (s_key[j] > mk) || (s_key[j] == mk && s_e[j] < me);
        s_rank_e[rank] = me;
        s_rank_s[rank] = __uint_as_float(mk);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float S = 0.0f;
        for (int r = 0; r < K; ++r) S += s_rank_s[r];
        for (int r = 0; r < K; ++r) {
            a.ws.idx[(size_t)b * K + r] = s_rank_e[r];
            a.ws.wts[(size_t)b * K + r] = s_rank_s[r] / S;
        }
    }
    // fp16 staging exponent of h for this token
    float m = 0.0f;
    for (int l = threadIdx.x; l < L; l += blockDim.x) m = fmaxf(m, fabsf(__ldcg(a.ws.h + (size_t)b * L + l)));
    m = block_max(m, s_red);
    if (threadIdx.x == 0) a.ws.h_shift[b] = prescale_shift(m);

    // the last token's CTA groups the B*K selections by expert
    if (!cta_ticket_last(a.ws.tickets + a.p.ticket_topk, (unsigned)B, &s_flag)) return;
    for (int i = threadIdx.x; i < E; i += blockDim.x) s_mask[i] = 0ull;
    __syncthreads();
    for (int i = threadIdx.x; i < B * K; i += blockDim.x) {
        const int ex = __ldcg(a.ws.idx + i);
        if (ex >= 0 && ex < E) atomicOr(&s_mask[ex], 1ull << (i / K));
        else atomicOr(a.ws.err, kErrBucket);
        a.ws.a_amax[i] = 0u;
    }
    __syncthreads();
    const unsigned long long mk = valid ? s_mask[e] : 0ull;
    const int cnt = __popcll(mk);
    int n_act, n_ent;
    const int j = block_exclusive_scan(cnt > 0 ? 1 : 0, s_warp, &n_act);
    const int off = block_exclusive_scan(cnt, s_warp, &n_ent);
    if (valid) s_off[e] = off;
    if (cnt > 0) {
        a.ws.active_e[j] = e;
        a.ws.active_cnt[j] = cnt;
        a.ws.active_off[j] = off;
    }
    if (threadIdx.x == 0) *a.ws.n_active = n_act;
    __syncthreads();
    for (int i = threadIdx.x; i < B * K; i += blockDim.x) {
        const int ex = __ldcg(a.ws.idx + i), tb = i / K;
        if (ex < 0 || ex >= E) continue;
        const int p = s_off[ex] + __popcll(s_mask[ex] & ((1ull << tb) - 1ull));
        a.ws.entries[p] = i;
    }
}

// ---------------------------------------------------------------------------------------------
// routed experts.  Work items are (active expert, 64-row block); a CTA owns a contiguous range
// of items, its 4 warps take 16 rows each, and the expert's tokens are staged once per K chunk.

template <int NT, bool SPLIT>
DEVI void expert_gu_item(const StepArgs &a, uint16_t *xs, int e, int row_blk, const int *ent, int ntok, int *s_shift) {
    const int L = a.d.L, I = a.d.I, K = a.d.k;
    const int ncols = SPLIT ? 2 * ntok : ntok;
    const int pitch = f16_pitch(kKChunk);
    const int warp = threadIdx.x >> 5;
    const int row0 = row_blk * kExpertRows + warp * 16;
    const size_t eq = (size_t)e * I * (L / 2), es = (size_t)e * I * (L / 32);
    float accg[NT][4] = {}, accu[NT][4] = {};
    for (int kc0 = 0; kc0 < L; kc0 += kKChunk) {
        const int kc = min(kKChunk, L - kc0);
        __syncthreads();
        stage_f16_from_f32<SPLIT>(xs, pitch, a.ws.h, L, ntok, [&](int t) { return ent[t] / K; }, s_shift, kc0, kc);
        __syncthreads();
        tile_fp4<NT, true>(a.w.gate_q + eq, a.w.gate_s + es, a.w.up_q + eq, a.w.up_s + es, L / 2, L / 32, row0, kc0,
                           kc / 128, xs, pitch, 0, ncols, accg, accu);
    }
    // epilogue: a = silu(g) * u (gate and up accumulators hold the same (token, row) in the same
    // lane), then the per-token max |a| over this tile's 16 rows feeds the down kernel's staging.
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    constexpr int PER_NT = SPLIT ? 1 : 2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int j = 0; j < PER_NT; ++j) {
            const int t = SPLIT ? nt * 4 + q : nt * 8 + 2 * q + j;
            const bool ok = t < ntok;
            const float sc = ok ? exp2i(s_shift[t]) : 0.0f;
            float g0, g1, u0, u1;
            if (SPLIT) {
                g0 = accg[nt][0] + accg[nt][1]; g1 = accg[nt][2] + accg[nt][3];
                u0 = accu[nt][0] + accu[nt][1]; u1 = accu[nt][2] + accu[nt][3];
            } else {
                g0 = accg[nt][j]; g1 = accg[nt][2 + j];
                u0 = accu[nt][j]; u1 = accu[nt][2 + j];
            }
            g0 *= sc; g1 *= sc; u0 *= sc; u1 *= sc;
            const float a0 = g0 / (1.0f + expf(-g0)) * u0, a1 = g1 / (1.0f + expf(-g1)) * u1;
            float m = ok ? fmaxf(fabsf(a0), fabsf(a1)) : 0.0f;
            if (ok) {
                float *dst = a.ws.a + (size_t)ent[t] * I + row0;
                dst[g] = a0;
                dst[g + 8] = a1;
            }
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
            if (ok && g == 0) atomicMax(a.ws.a_amax + ent[t], __float_as_uint(m));
        }
    }
}

template <int NT, bool SPLIT>
DEVI void expert_down_item(const StepArgs &a, uint16_t *xs, int e, int row_blk, const int *ent, int ntok, int *s_shift) {
    const int L = a.d.L, I = a.d.I;
    const int ncols = SPLIT ? 2 * ntok : ntok;
    const int pitch = f16_pitch(kKChunk);
    const int warp = threadIdx.x >> 5;
    const int row0 = row_blk * kExpertRows + warp * 16;
    const size_t eq = (size_t)e * L * (I / 2), es = (size_t)e * L * (I / 32);
    float acc[NT][4] = {}, dummy[NT][4];
    for (int kc0 = 0; kc0 < I; kc0 += kKChunk) {
        const int kc = min(kKChunk, I - kc0);
        __syncthreads();
        stage_f16_from_f32<SPLIT>(xs, pitch, a.ws.a, I, ntok, [&](int t) { return ent[t]; }, s_shift, kc0, kc);
        __syncthreads();
        tile_fp4<NT, false>(a.w.down_q + eq, a.w.down_s + es, nullptr, nullptr, I / 2, I / 32, row0, kc0, kc / 128, xs,
                            pitch, 0, ncols, acc, dummy);
    }
    tile_foreach<NT, SPLIT>(acc, ntok, [&](int t, int r, float v) {
        a.ws.y[(size_t)ent[t] * L + row0 + r] = v * exp2i(s_shift[t]);
    });
}

template <bool DOWN>
__global__ void __launch_bounds__(kExpertWarps * 32) k_expert(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    __shared__ int s_ent[32];
    __shared__ int s_shift[32];
    const int rows = DOWN ? a.d.L : a.d.I;
    const int blocks = rows / kExpertRows;
    const int n_active = __ldcg(a.ws.n_active);
    const int n_items = n_active * blocks;
    const int i0 = (int)((long long)blockIdx.x * n_items / gridDim.x);
    const int i1 = (int)((long long)(blockIdx.x + 1) * n_items / gridDim.x);
    for (int item = i0; item < i1; ++item) {
        const int j = item / blocks, blk = item % blocks;
        const int e = __ldcg(a.ws.active_e + j), cnt = __ldcg(a.ws.active_cnt + j), off = __ldcg(a.ws.active_off + j);
        for (int t0 = 0; t0 < cnt; t0 += 32) {
            const int ntok = min(32, cnt - t0);
            __syncthreads();  // previous users of s_ent / s_shift are done
            if (threadIdx.x < ntok) {
                const int ent = __ldcg(a.ws.entries + off + t0 + threadIdx.x);
                s_ent[threadIdx.x] = ent;
                if (DOWN) s_shift[threadIdx.x] = prescale_shift(__uint_as_float(__ldcg(a.ws.a_amax + ent)));
                else s_shift[threadIdx.x] = __ldcg(a.ws.h_shift + ent / a.d.k);
            }
            __syncthreads();
            if (DOWN) {
                if (ntok <= 4) expert_down_item<1, true>(a, xs, e, blk, s_ent, ntok, s_shift);
                else if (ntok <= 8) expert_down_item<1, false>(a, xs, e, blk, s_ent, ntok, s_shift);
                else if (ntok <= 16) expert_down_item<2, false>(a, xs, e, blk, s_ent, ntok, s_shift);
                else expert_down_item<4, false>(a, xs, e, blk, s_ent, ntok, s_shift);
            } else {
                if (ntok <= 4) expert_gu_item<1, true>(a, xs, e, blk, s_ent, ntok, s_shift);
                else if (ntok <= 8) expert_gu_item<1, false>(a, xs, e, blk, s_ent, ntok, s_shift);
                else if (ntok <= 16) expert_gu_item<2, false>(a, xs, e, blk, s_ent, ntok, s_shift);
                else expert_gu_item<4, false>(a, xs, e, blk, s_ent, ntok, s_shift);
            }
        }
    }
}

// ---------------------------------------------------------------------------------------------
// combine: ylat[b][l] = sum_r w[b][r] y[b*K + r][l], slots in rank order.

__global__ void __launch_bounds__(256) k_combine(StepArgs a) {
    const int L = a.d.L, K = a.d.k;
    const int b = blockIdx.y, l = blockIdx.x * blockDim.x + threadIdx.x;
    if (l >= L) return;
    float s = 0.0f;
    for (int r = 0; r < K; ++r)
        s += __ldcg(a.ws.wts + (size_t)b * K + r) * __ldcg(a.ws.y + ((size_t)b * K + r) * L + l);
    a.ws.ylat[(size_t)b * L + l] = s;
}

// ---------------------------------------------------------------------------------------------
// up-projection: out = bf16(W_up ylat + sh).  ylat enters as bf16 hi/lo column pairs.

template <int NT>
__global__ void __launch_bounds__(256) k_up(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ unsigned s_flag;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    const int H = a.d.H, L = a.d.L, B = a.B, maxB = a.d.max_batch;
    const int rb = blockIdx.x / a.p.up.splits, ks = blockIdx.x % a.p.up.splits;
    const int KR = a.p.up.krange, k0 = ks * KR;
    const int kc = up_chunk(NT, KR);
    const int pitch = bf16_pitch(kc);
    const int warp = threadIdx.x >> 5;
    const int row0 = rb * kDenseRows + warp * 16;
    float acc[NT][4] = {};
    for (int c0 = k0; c0 < k0 + KR; c0 += kc) {
        __syncthreads();
        stage_bf16split_from_f32(xs, pitch, a.ws.ylat, L, B, c0, kc);
        for (int i = threadIdx.x; i < (8 * NT - 2 * B) * (kc / 8); i += blockDim.x) {  // zero unused columns
            const int col = 2 * B + i / (kc / 8), u = i % (kc / 8);
            *reinterpret_cast<uint4 *>(xs + (size_t)col * pitch + 8 * u) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncthreads();
        if (row0 < H) tile_bf16<NT>(a.w.w_up, L, row0, c0, kc / 32, xs, pitch, 0, 2 * B, acc);
    }
    if (row0 < H) {
        float *part = a.ws.up_part + (size_t)ks * maxB * H;
        tile_foreach<NT, true>(acc, B, [&](int t, int r, float v) { part[(size_t)t * H + row0 + r] = v; });
    }
    if (cta_ticket_last(a.ws.tickets + a.p.ticket_up + rb, a.p.up.splits, &s_flag)) {
        for (int i = threadIdx.x; i < kDenseRows * B; i += blockDim.x) {
            const int r = rb * kDenseRows + (i % kDenseRows), b = i / kDenseRows;
            if (r >= H) continue;
            float s = 0.0f;
            for (int k = 0; k < a.p.up.splits; ++k) s += __ldcg(a.ws.up_part + ((size_t)k * maxB + b) * H + r);
            if (a.ws.up_tap) a.ws.up_tap[(size_t)b * H + r] = s;
            const float shv = a.d.n_shared ? __ldcg(a.ws.sh + (size_t)b * H + r) : 0.0f;
            a.out[(size_t)b * H + r] = f32_to_bf16_rne(s + shv);
        }
    }
}

// ---------------------------------------------------------------------------------------------
// shared expert (side stream).  gate/up: rows of I_s in pairs, K = H; down: rows of H, K = I_s.

template <int NT>
__global__ void __launch_bounds__(256) k_shared_gu(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ unsigned s_flag;
    __shared__ int s_shift[kMaxBatch];
    __shared__ unsigned s_amax[kMaxBatch];
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    const int H = a.d.H, Is = a.d.Is, B = a.B, maxB = a.d.max_batch;
    const int rb = blockIdx.x / a.p.sgu.splits, ks = blockIdx.x % a.p.sgu.splits;
    const int KR = a.p.sgu.krange, k0 = ks * KR;
    const int pitch = f16_pitch(KR);
    // per-token staging exponent over this K range
    for (int t = threadIdx.x; t < B; t += blockDim.x) s_amax[t] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < B * (KR / 8); i += blockDim.x) {
        const int t = i / (KR / 8), u = i % (KR / 8);
        const uint4 v = *reinterpret_cast<const uint4 *>(a.x + (size_t)t * H + k0 + 8 * u);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
        atomicMax(s_amax + t, __float_as_uint(m));
    }
    __syncthreads();
    for (int t = threadIdx.x; t < B; t += blockDim.x) s_shift[t] = prescale_shift(__uint_as_float(s_amax[t]));
    __syncthreads();
    stage_f16_from_bf16(xs, pitch, a.x, H, B, s_shift, k0, KR);
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    const int row0 = rb * kDenseRows + warp * 16;
    if (row0 < Is) {
        float accg[NT][4] = {}, accu[NT][4] = {};
        tile_fp4<NT, true>(a.w.sh_gate_q, a.w.sh_gate_s, a.w.sh_up_q, a.w.sh_up_s, H / 2, H / 32, row0, k0, KR / 128, xs,
                           pitch, 0, B, accg, accu);
        float *part = a.ws.sgu_part + (size_t)ks * maxB * 2 * Is;
        tile_foreach<NT, false>(accg, B, [&](int t, int r, float v) {
            part[(size_t)t * 2 * Is + row0 + r] = v * exp2i(s_shift[t]);
        });
        tile_foreach<NT, false>(accu, B, [&](int t, int r, float v) {
            part[(size_t)t * 2 * Is + Is + row0 + r] = v * exp2i(s_shift[t]);
        });
    }
    if (cta_ticket_last(a.ws.tickets + a.p.ticket_sgu + rb, a.p.sgu.splits, &s_flag)) {
        for (int i = threadIdx.x; i < kDenseRows * B; i += blockDim.x) {
            const int r = rb * kDenseRows + (i % kDenseRows), b = i / kDenseRows;
            if (r >= Is) continue;
            float gs = 0.0f, us = 0.0f;
            for (int k = 0; k < a.p.sgu.splits; ++k) {
                const float *p = a.ws.sgu_part + ((size_t)k * maxB + b) * 2 * Is;
                gs += __ldcg(p + r);
                us += __ldcg(p + Is + r);
            }
            a.ws.sh_a[(size_t)b * Is + r] = gs / (1.0f + expf(-gs)) * us;
        }
    }
}

template <int NT, bool SPLIT>
__global__ void __launch_bounds__(256) k_shared_down(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ unsigned s_flag;
    __shared__ int s_shift[kMaxBatch];
    __shared__ unsigned s_amax[kMaxBatch];
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    const int H = a.d.H, Is = a.d.Is, B = a.B, maxB = a.d.max_batch;
    const int rb = blockIdx.x / a.p.sd.splits, ks = blockIdx.x % a.p.sd.splits;
    const int KR = a.p.sd.krange, k0 = ks * KR;
    const int pitch = f16_pitch(KR);
    for (int t = threadIdx.x; t < B; t += blockDim.x) s_amax[t] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < B * (KR / 4); i += blockDim.x) {
        const int t = i / (KR / 4), u = i % (KR / 4);
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.ws.sh_a + (size_t)t * Is + k0) + u);
        atomicMax(s_amax + t, __float_as_uint(fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)))));
    }
    __syncthreads();
    for (int t = threadIdx.x; t < B; t += blockDim.x) s_shift[t] = prescale_shift(__uint_as_float(s_amax[t]));
    __syncthreads();
    stage_f16_from_f32<SPLIT>(xs, pitch, a.ws.sh_a, Is, B, [](int t) { return t; }, s_shift, k0, KR);
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    const int row0 = rb * kDenseRows + warp * 16;
    const int ncols = SPLIT ? 2 * B : B;
    if (row0 < H) {
        float acc[NT][4] = {}, dummy[NT][4];
        tile_fp4<NT, false>(a.w.sh_down_q, a.w.sh_down_s, nullptr, nullptr, Is / 2, Is / 32, row0, k0, KR / 128, xs,
                            pitch, 0, ncols, acc, dummy);
        float *part = a.ws.sd_part + (size_t)ks * maxB * H;
        tile_foreach<NT, SPLIT>(acc, B, [&](int t, int r, float v) {
            part[(size_t)t * H + row0 + r] = v * exp2i(s_shift[t]);
        });
    }
    if (cta_ticket_last(a.ws.tickets + a.p.ticket_sd + rb, a.p.sd.splits, &s_flag)) {
        for (int i = threadIdx.x; i < kDenseRows * B; i += blockDim.x) {
            const int r = rb * kDenseRows + (i % kDenseRows), b = i / kDenseRows;
            if (r >= H) continue;
            float s = 0.0f;
            for (int k = 0; k < a.p.sd.splits; ++k) s += __ldcg(a.ws.sd_part + ((size_t)k * maxB + b) * H + r);
            a.ws.sh[(size_t)b * H + r] = s;
        }
    }
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
// host launchers

static int nt_for_cols(int cols) { return cols <= 8 ? 1 : cols <= 16 ? 2 : cols <= 32 ? 4 : cols <= 64 ? 8 : 16; }

static size_t router_smem(const StepArgs &a) { return (size_t)8 * (a.p.rt.krange + 4) * sizeof(double); }

template <int NT>
static cudaError_t launch_router_dn_nt(const StepArgs &a, cudaStream_t s) {
    const size_t dn_smem = (size_t)8 * NT * bf16_pitch(a.p.dn.krange) * 2;
    const size_t sm = router_smem(a) > dn_smem ? router_smem(a) : dn_smem;
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
    int threads = ((a.d.E + 31) / 32) * 32;
    if (threads < 64) threads = 64;
    k_topk<<<a.B, threads, 0, s>>>(a);
    return cudaGetLastError();
}

static size_t expert_smem(const StepArgs &a) {
    const int cols = a.B <= 4 ? 2 * a.B : (a.B < 32 ? a.B : 32);
    const int pad_cols = 8 * nt_for_cols(cols < 8 ? 8 : cols);
    return (size_t)pad_cols * f16_pitch(kKChunk) * 2;
}

static cudaError_t launch_expert(const StepArgs &a, cudaStream_t s, int n_sm, bool down) {
    const size_t sm = expert_smem(a);
    auto kern = down ? k_expert<true> : k_expert<false>;
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kExpertWarps * 32, sm);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    kern<<<n_sm * per_sm, kExpertWarps * 32, sm, s>>>(a);
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
        (const void *)k_router_dn<1>, (const void *)k_router_dn<2>, (const void *)k_router_dn<4>,
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
