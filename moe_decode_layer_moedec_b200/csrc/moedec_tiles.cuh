// moedec_tiles.cuh -- warp-level MMA tiles and activation staging shared by the step kernels.
#pragma once

#include "moedec_device.cuh"
#include "moedec_internal.h"

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

// Sum of n (<= 16) split-K partials p[0], p[stride], ... in split order.  All loads are issued
// before the first add (one L2 round trip instead of n); L1-bypassing, since other CTAs wrote them.
template <class T, int W = 8>
DEVI T sum_splits(const T *p, size_t stride, int n) {
    T s = T(0);
    for (int k0 = 0; k0 < n; k0 += W) {  // W loads in flight, then W adds in split order
        T v[W];
#pragma unroll
        for (int k = 0; k < W; ++k) v[k] = k0 + k < n ? __ldcg(p + (size_t)(k0 + k) * stride) : T(0);
#pragma unroll
        for (int k = 0; k < W; ++k)
            if (k0 + k < n) s += v[k];
    }
    return s;
}

// NP such sums at once: out[i] = sum over k < n of p[i][k * stride], each in split order (the
// same additions as sum_splits, so the same bits).  The loads of all NP sums for W splits are
// issued before the first add: a thread that reduces several rows pays one L2 round trip per 16
// W splits for all of them instead of one per row.  valid[i] false gives out[i] = 0, no loads.
template <int NP, int W = 16, class T>
DEVI void sum_splits_batch(const T *const (&p)[NP], const bool (&valid)[NP], size_t stride, int n, T (&out)[NP]) {
#pragma unroll
    for (int i = 0; i < NP; ++i) out[i] = T(0);
    for (int k0 = 0; k0 < n; k0 += W) {
        T v[NP][W];
#pragma unroll
        for (int i = 0; i < NP; ++i)
#pragma unroll
            for (int k = 0; k < W; ++k) v[i][k] = (valid[i] && k0 + k < n) ? __ldcg(p[i] + (size_t)(k0 + k) * stride) : T(0);
#pragma unroll
        for (int i = 0; i < NP; ++i)
#pragma unroll
            for (int k = 0; k < W; ++k)
                if (k0 + k < n) out[i] += v[i][k];
    }
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
// The weight stream is software-pipelined: the loads of the next D rounds are in flight while
// a round is multiplied (D rounds x 32 bytes per lane).
// Rounds in flight per lane: more token columns mean more MMAs per byte, so fewer rounds cover
// the load latency (and the accumulators need the registers).
constexpr int depth_bf16(int nt) { return nt <= 2 ? 8 : nt <= 4 ? 6 : nt <= 8 ? 4 : 2; }
constexpr int depth_fp4(int nt, bool pair) { return pair ? (nt <= 1 ? 4 : nt <= 2 ? 3 : 2) : (nt <= 2 ? 8 : nt <= 4 ? 4 : 2); }

template <int NT, int D = depth_bf16(NT)>
DEVI void tile_bf16(const uint16_t *__restrict__ W, size_t ldw, int row0, int kg, int nrounds,
                    const uint16_t *xs, int pitch, int kofs, int ncols, float (&acc)[NT][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const uint16_t *wa = W + (size_t)(row0 + g) * ldw + kg + 8 * q;
    const uint16_t *wb = wa + 8 * ldw;
    const uint16_t *xr = xs + kofs + 8 * q;
    float acc2[NT][4] = {};  // second MMA step of each round: an independent accumulator chain
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
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int col = nt * 8 + g;
                    uint4 xb = *reinterpret_cast<const uint4 *>(xr + (size_t)col * pitch + 32 * r);
                    if (col >= ncols) xb = make_uint4(0u, 0u, 0u, 0u);
                    mma_bf16(acc[nt], a.x, b.x, a.y, b.y, xb.x, xb.y);
                    mma_bf16(acc2[nt], a.z, b.z, a.w, b.w, xb.z, xb.w);
                }
            }
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[nt][j] += acc2[nt][j];
}

// MXFP4 rows: codes Q[row][k/2], scales S[row][k/32]; lane quad q owns 32-element block
// (kg/32 + 4r + q) of each round.  PAIR = gate and up rows share the token operand.
// The E8M0 scale is folded into the fp16 weights (exact for scale bytes 104..140).
// Software-pipelined like tile_bf16: D rounds of codes and scales in flight per lane.
struct Fp4Round {
    uint4 c0, c1;      // 16-byte blocks of rows g and g+8
    uint32_t s0, s1;   // the round's four scale bytes of rows g and g+8 (byte q is this lane's)
};

DEVI void fp4_load(Fp4Round &f, const uint8_t *q0, const uint8_t *q1, const uint8_t *s0, const uint8_t *s1, int r) {
    f.c0 = ldg_weights(q0 + 64 * r);
    f.c1 = ldg_weights(q1 + 64 * r);
    f.s0 = ldg_weights_u32(s0 + 4 * r);
    f.s1 = ldg_weights_u32(s1 + 4 * r);
}

DEVI void fp4_decode_word(uint32_t codes, uint32_t scale_f16x2, uint32_t (&d)[4]) {
    e2m1x8_to_f16x2(codes, d);
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = hmul2(d[i], scale_f16x2);
}

// Independent accumulator sets per token tile: consecutive MMA steps alternate between them so
// that the MMAs of a round do not wait on one another (with one accumulator the eight MMAs of an
// FP4 round form a dependency chain that bounds a warp's streaming rate).
constexpr int chains_fp4(int nt) { return nt <= 1 ? 4 : nt <= 2 ? 2 : 1; }

template <int NT, bool PAIR, int D = depth_fp4(NT, PAIR)>
DEVI void tile_fp4(const uint8_t *__restrict__ Qa, const uint8_t *__restrict__ Sa, const uint8_t *__restrict__ Qb,
                   const uint8_t *__restrict__ Sb, size_t ldq, size_t lds, int row0, int kg, int nrounds,
                   const uint16_t *xs, int pitch, int kofs, int ncols, float (&acc)[NT][4], float (&acc2)[NT][4]) {
    constexpr int C = PAIR ? 1 : chains_fp4(NT);
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
    const int ubase = kofs / 8 + 4 * q, flip = q >> 1, sh = 8 * q;
    float ch[C][NT][4];
#pragma unroll
    for (int c = 0; c < C; ++c)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) ch[c][nt][j] = c == 0 ? acc[nt][j] : 0.0f;
    Fp4Round fa[D], fb[PAIR ? D : 1];
#pragma unroll
    for (int s = 0; s < D; ++s)
        if (s < nrounds) {
            fp4_load(fa[s], qa0, qa1, sa0, sa1, s);
            if (PAIR) fp4_load(fb[PAIR ? s : 0], qb0, qb1, sb0, sb1, s);
        }
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
                // word w of the lane's 16-byte block holds MMA steps 2w and 2w+1; the matching
                // token values are unit w of the lane's 64-byte activation slice.
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
                    constexpr int c0 = 0;
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
                    (void)c0;
                }
            }
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float t = ch[0][nt][j];
#pragma unroll
            for (int c = 1; c < C; ++c) t += ch[c][nt][j];
            acc[nt][j] = t;
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

// Every staging helper issues a batch of its thread's loads before the first store, so that a call
// costs about one L2 round trip per batch rather than one per element of its loop.
constexpr int kStageBatch = 4;   // 16-byte loads (bf16 sources)
constexpr int kStageBatchF = 2;  // 32-byte loads (fp32 sources)

// bf16 tokens x[b][k0 .. k0+kc) -> xs[col b][0..kc) (bf16 layout), columns [ntok, ncols_pad) zero.
DEVI void stage_bf16(uint16_t *xs, int pitch, const uint16_t *x, size_t ldx, int ntok, int ncols_pad, int k0, int kc,
                      int tid = threadIdx.x, int nthr = blockDim.x) {
    const int units = kc / 8, total = ncols_pad * units;
    for (int i0 = tid; i0 < total; i0 += kStageBatch * nthr) {
        uint4 v[kStageBatch];
#pragma unroll
        for (int j = 0; j < kStageBatch; ++j) {
            const int i = i0 + j * nthr, col = i / units, u = i % units;
            v[j] = make_uint4(0u, 0u, 0u, 0u);
            if (i < total && col < ntok) v[j] = *reinterpret_cast<const uint4 *>(x + (size_t)col * ldx + k0 + 8 * u);
        }
#pragma unroll
        for (int j = 0; j < kStageBatch; ++j) {
            const int i = i0 + j * nthr, col = i / units, u = i % units;
            if (i < total) *reinterpret_cast<uint4 *>(xs + (size_t)col * pitch + 8 * u) = v[j];
        }
    }
}

// fp32 vectors src[rowof(i)][k0 .. k0+kc) * 2^-shift[i] -> fp16 columns (fp16 layout, swizzled).
// SPLIT: column 2i = fp16(v), 2i+1 = fp16(v - fp16(v)).  Reads with L1-bypassing loads.
template <bool SPLIT, class RowOf>
DEVI void stage_f16_from_f32(uint16_t *xs, int pitch, const float *src, size_t lds, int ntok, RowOf rowof,
                             const int *shift, int k0, int kc, int tid = threadIdx.x, int nthr = blockDim.x) {
    const int units = kc / 8, total = ntok * units;
    for (int i0 = tid; i0 < total; i0 += kStageBatchF * nthr) {
        float4 v0[kStageBatchF], v1[kStageBatchF];
#pragma unroll
        for (int j = 0; j < kStageBatchF; ++j) {
            const int i = i0 + j * nthr;
            if (i < total) {
                const int t = i / units, u = i % units;
                const float *p = src + (size_t)rowof(t) * lds + k0 + 8 * u;
                v0[j] = __ldcg(reinterpret_cast<const float4 *>(p));
                v1[j] = __ldcg(reinterpret_cast<const float4 *>(p) + 1);
            }
        }
#pragma unroll
        for (int j = 0; j < kStageBatchF; ++j) {
            const int i = i0 + j * nthr;
            if (i < total) {
                const int t = i / units, u = i % units;
                const float sc = exp2i(-shift[t]);
                const float v[8] = {v0[j].x * sc, v0[j].y * sc, v0[j].z * sc, v0[j].w * sc,
                                    v1[j].x * sc, v1[j].y * sc, v1[j].z * sc, v1[j].w * sc};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    hi[q] = pack_f16x2(v[2 * q], v[2 * q + 1]);
                    if (SPLIT) lo[q] = pack_f16x2(v[2 * q] - f16_lo(hi[q]), v[2 * q + 1] - f16_hi(hi[q]));
                }
                const int col = SPLIT ? 2 * t : t;
                *reinterpret_cast<uint4 *>(xs + (size_t)col * pitch + 8 * swz(u)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                if (SPLIT)
                    *reinterpret_cast<uint4 *>(xs + (size_t)(col + 1) * pitch + 8 * swz(u)) =
                        make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
    }
}

// bf16 tokens * 2^-shift -> fp16 columns (exact in fp16 for all but values 2^-38 below the
// column's maximum), fp16 layout, swizzled.
DEVI void stage_f16_from_bf16(uint16_t *xs, int pitch, const uint16_t *x, size_t ldx, int ntok, const int *shift,
                              int k0, int kc, int tid = threadIdx.x, int nthr = blockDim.x) {
    const int units = kc / 8, total = ntok * units;
    for (int i0 = tid; i0 < total; i0 += kStageBatch * nthr) {
        uint4 v[kStageBatch];
#pragma unroll
        for (int j = 0; j < kStageBatch; ++j) {
            const int i = i0 + j * nthr, t = i / units, u = i % units;
            v[j] = i < total ? *reinterpret_cast<const uint4 *>(x + (size_t)t * ldx + k0 + 8 * u) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < kStageBatch; ++j) {
            const int i = i0 + j * nthr, t = i / units, u = i % units;
            if (i < total) {
                const float sc = exp2i(-shift[t]);
                const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
                uint32_t o[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) o[q] = pack_f16x2(bf16_lo(w[q]) * sc, bf16_hi(w[q]) * sc);
                *reinterpret_cast<uint4 *>(xs + (size_t)t * pitch + 8 * swz(u)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
}

// fp32 vectors -> bf16 hi/lo column pairs (bf16 layout): column 2i = bf16(v), 2i+1 = bf16(v - hi).
DEVI void stage_bf16split_from_f32(uint16_t *xs, int pitch, const float *src, size_t lds, int ntok, int k0, int kc,
                                   int tid = threadIdx.x, int nthr = blockDim.x) {
    const int units = kc / 8, total = ntok * units;
    for (int i0 = tid; i0 < total; i0 += kStageBatchF * nthr) {
        float4 v0[kStageBatchF], v1[kStageBatchF];
#pragma unroll
        for (int j = 0; j < kStageBatchF; ++j) {
            const int i = i0 + j * nthr;
            if (i < total) {
                const int t = i / units, u = i % units;
                const float *p = src + (size_t)t * lds + k0 + 8 * u;
                v0[j] = __ldcg(reinterpret_cast<const float4 *>(p));
                v1[j] = __ldcg(reinterpret_cast<const float4 *>(p) + 1);
            }
        }
#pragma unroll
        for (int j = 0; j < kStageBatchF; ++j) {
            const int i = i0 + j * nthr;
            if (i < total) {
                const int t = i / units, u = i % units;
                const float v[8] = {v0[j].x, v0[j].y, v0[j].z, v0[j].w, v1[j].x, v1[j].y, v1[j].z, v1[j].w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    hi[q] = pack_bf16x2(v[2 * q], v[2 * q + 1]);
                    lo[q] = pack_bf16x2(v[2 * q] - bf16_lo(hi[q]), v[2 * q + 1] - bf16_hi(hi[q]));
                }
                *reinterpret_cast<uint4 *>(xs + (size_t)(2 * t) * pitch + 8 * u) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(xs + (size_t)(2 * t + 1) * pitch + 8 * u) =
                    make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
    }
}

}  // namespace moedec
