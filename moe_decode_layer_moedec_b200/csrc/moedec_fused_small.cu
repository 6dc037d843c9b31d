// moedec_fused_small.cu -- the decode layer step for batches of at most 4 tokens, one persistent
// kernel.
//
// This is the small-matrix variant of the step: the Kimi K3 decode work picks a small-matrix
// kernel shape at batch 1-2 and split-K above ("快是可以生成的，可信只能证明（vLLM 重写 Kimi K3
// 解码路径…）", section 他们换掉了什么).  With at most 4 tokens the whole activation of a part fits
// in shared memory, so every work item covers full K: the CTA's 8 warps split K (or rows x K)
// between them and add their accumulators in shared memory in a fixed order.  There are no
// split-K partials in global memory and no tickets; an item's result is final when the item ends.
//
// Queues, drained in this order by every CTA (one CTA per SM, cooperative launch), each item
// claimed one ahead so that its weights are prefetched into L2 while the previous one runs:
//   router       8 rows x K=H       fp64 MMAs, warps split K               -> logits rows
//   top-k        one per token      waits: all router items                -> routing, buckets
//   W_dn         16 rows x K=H      warps split K                          -> h rows, max |h|
//   shared g/u   32 rows x K=H      2 row tiles x 4 K quarters, gate+up    -> sh_a rows
//   expert g/u   128 rows of one    waits: buckets, all of h               -> a rows
//                expert, K=L        one 16-row tile per warp
//   shared down  64 rows x K=I_s    4 row tiles x 2 K halves               -> sh rows
//   expert down  128 rows of one    waits: the expert's g/u items          -> y rows; the item that
//                expert, K=I        one 16-row tile per warp                 completes a token's 128
//                                                                            rows combines them to ylat
//   W_up         64 rows x K=L      4 row tiles x 2 K halves; waits: ylat, sh -> out rows
#include "moedec_items.cuh"

namespace moedec {

constexpr int kFsRouterRows = 8, kFsDnRows = 16, kFsSguRows = 32, kFsExpRows = 128, kFsSdRows = 64, kFsUpRows = 64;
enum SmallQueue { Q_ROUTER_S = 0, Q_TOPK_S, Q_DN_S, Q_SGU_S, Q_EGU_S, Q_SD_S, Q_EDOWN_S, Q_UP_S };

struct FsSmem {
    double rd[8][32][2];  // router partials of the 8 warps
    float rf[8][32][8];   // tile accumulators of the 8 warps (gate and up)
    int ent[8];
    int shift[8];
    int xshift[8];
    int flag[8];
    int ok;
    int item;
};

// prefetch `bytes` (multiple of 16) starting at p into L2, 32 KB per thread
DEVI void fs_prefetch(const void *p, size_t bytes) {
    const size_t piece = 32768;
    const size_t n = (bytes + piece - 1) / piece;
    for (size_t i = threadIdx.x; i < n; i += blockDim.x) {
        const size_t off = i * piece;
        const size_t len = bytes - off < piece ? bytes - off : piece;
        prefetch_l2(static_cast<const uint8_t *>(p) + off, (uint32_t)len);
    }
}

// ---- router: 8 rows, full K; warp w sums k in [w*H/8, (w+1)*H/8) ---------------------------------

DEVI void fs_router(const StepArgs &a, int item, const uint16_t *xs, FsSmem &f) {
    const int E = a.d.E, H = a.d.H, B = a.B;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int row = item * kFsRouterRows + g;
    const bool row_ok = row < E;
    const int KW = H / 8, k0 = warp * KW, nch = KW / 32;
    const int pitch = bf16_pitch(H);
    const uint16_t *rrow = a.w.router + (size_t)(row_ok ? row : 0) * H + k0 + 8 * q;
    const uint16_t *xr = xs + (size_t)g * pitch + k0 + 8 * q;
    double c0 = 0.0, c1 = 0.0, d0 = 0.0, d1 = 0.0;
    constexpr int D = 8;
    uint4 A[D];
#pragma unroll
    for (int s = 0; s < D; ++s) A[s] = (row_ok && s < nch) ? ldg_weights(rrow + 32 * s) : make_uint4(0u, 0u, 0u, 0u);
    for (int c0i = 0; c0i < nch; c0i += D) {
#pragma unroll
        for (int s = 0; s < D; ++s) {
            const int c = c0i + s;
            if (c < nch) {
                const uint4 Ac = A[s];
                if (c + D < nch) A[s] = row_ok ? ldg_weights(rrow + 32 * (c + D)) : make_uint4(0u, 0u, 0u, 0u);
                const uint4 xb = *reinterpret_cast<const uint4 *>(xr + 32 * c);
                const double av[8] = {bf16_lo(Ac.x), bf16_hi(Ac.x), bf16_lo(Ac.y), bf16_hi(Ac.y),
                                      bf16_lo(Ac.z), bf16_hi(Ac.z), bf16_lo(Ac.w), bf16_hi(Ac.w)};
                const double xv[8] = {bf16_lo(xb.x), bf16_hi(xb.x), bf16_lo(xb.y), bf16_hi(xb.y),
                                      bf16_lo(xb.z), bf16_hi(xb.z), bf16_lo(xb.w), bf16_hi(xb.w)};
                // m8n8k4 step s of chunk c: slot q holds k = 32c + 8q + s
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    mma_f64(c0, c1, av[2 * s2], xv[2 * s2]);
                    mma_f64(d0, d1, av[2 * s2 + 1], xv[2 * s2 + 1]);
                }
            }
        }
    }
    f.rd[warp][lane][0] = c0 + d0;
    f.rd[warp][lane][1] = c1 + d1;
    __syncthreads();
    if (warp == 0 && row_ok) {
        double s0 = 0.0, s1 = 0.0;
        for (int w = 0; w < 8; ++w) {
            s0 += f.rd[w][lane][0];
            s1 += f.rd[w][lane][1];
        }
        if (2 * q < B) a.ws.logits[(size_t)(2 * q) * E + row] = (float)s0;
        if (2 * q + 1 < B) a.ws.logits[(size_t)(2 * q + 1) * E + row] = (float)s1;
    }
    if (!(a.flags & kFlagTestStall)) cta_signal_add(a.ws.ctl + CTL_RT_DONE, 1u);
    else __syncthreads();
}

// ---- reduction of per-warp accumulators in shared memory -----------------------------------------

// Sum the accumulators (n floats per lane) of warps w0, w0+ws, ..., (cnt warps) in that order.
DEVI void fs_sum(const FsSmem &f, int w0, int wstride, int cnt, int n, float *out) {
    const int lane = threadIdx.x & 31;
    for (int i = 0; i < n; ++i) out[i] = 0.0f;
    for (int k = 0; k < cnt; ++k)
        for (int i = 0; i < n; ++i) out[i] += f.rf[w0 + k * wstride][lane][i];
}

// ---- W_dn: 16 rows, full K; warp w sums k in [w*H/8, (w+1)*H/8) ----------------------------------

DEVI void fs_dn(const StepArgs &a, int item, const uint16_t *xs, FsSmem &f) {
    const int L = a.d.L, H = a.d.H, B = a.B;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int row0 = item * kFsDnRows, KW = H / 8, k0 = warp * KW;
    float acc[1][4] = {};
    tile_bf16<1>(a.w.w_dn, H, row0, k0, KW / 32, xs, bf16_pitch(H), k0, B, acc);
    for (int j = 0; j < 4; ++j) f.rf[warp][lane][j] = acc[0][j];
    __syncthreads();
    if (warp == 0) {
        float v[4];
        fs_sum(f, 0, 1, 8, 4, v);
        // lane holds rows g, g+8 for tokens 2q, 2q+1
        for (int j = 0; j < 2; ++j) {
            const int t = 2 * q + j;
            float m = 0.0f;
            if (t < B) {
                a.ws.h[(size_t)t * L + row0 + g] = v[j];
                a.ws.h[(size_t)t * L + row0 + g + 8] = v[2 + j];
                m = fmaxf(fabsf(v[j]), fabsf(v[2 + j]));
            }
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
            if (t < B && g == 0) atomicMax(a.ws.ctl + a.p.ctl_hamax + t, __float_as_uint(m));
        }
    }
    cta_signal_add(a.ws.ctl + CTL_DN_DONE, 1u);
}

// ---- shared gate/up: 32 rows (2 tiles) x full K (4 quarters), gate and up together ----------------

DEVI void fs_sgu(const StepArgs &a, int item, const uint16_t *xs16, FsSmem &f) {
    const int H = a.d.H, Is = a.d.Is, B = a.B;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int tile = warp >> 2, kq = warp & 3;
    const int row0 = item * kFsSguRows + tile * 16, KW = H / 4, k0 = kq * KW;
    float accg[1][4] = {}, accu[1][4] = {};
    tile_fp4<1, true>(a.w.sh_gate_q, a.w.sh_gate_s, a.w.sh_up_q, a.w.sh_up_s, H / 2, H / 32, row0, k0, KW / 128, xs16,
                      f16_pitch(H), k0, B, accg, accu);
    for (int j = 0; j < 4; ++j) {
        f.rf[warp][lane][j] = accg[0][j];
        f.rf[warp][lane][4 + j] = accu[0][j];
    }
    __syncthreads();
    if (kq == 0) {
        float v[8];
        fs_sum(f, warp, 1, 4, 8, v);
        for (int j = 0; j < 2; ++j) {
            const int t = 2 * q + j;
            float m = 0.0f;
            if (t < B) {
                const float sc = exp2i(f.xshift[t]);
                for (int h2 = 0; h2 < 2; ++h2) {
                    const float gg = v[j + 2 * h2] * sc, uu = v[4 + j + 2 * h2] * sc;
                    const float av = gg / (1.0f + expf(-gg)) * uu;
                    a.ws.sh_a[(size_t)t * Is + row0 + g + 8 * h2] = av;
                    m = fmaxf(m, fabsf(av));
                }
            }
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
            if (t < B && g == 0) atomicMax(a.ws.ctl + a.p.ctl_shamax + t, __float_as_uint(m));
        }
    }
    cta_signal_add(a.ws.ctl + CTL_SGU_DONE, 1u);
}

// ---- expert gate/up: 128 rows of one active expert, full K, one 16-row tile per warp --------------

DEVI void fs_egu(const StepArgs &a, int item, uint16_t *xs, FsSmem &f) {
    const int L = a.d.L, I = a.d.I, K = a.d.k;
    const int blocks = I / kFsExpRows, j = item / blocks, blk = item % blocks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int e = __ldcg(a.ws.active_e + j), cnt = __ldcg(a.ws.active_cnt + j), off = __ldcg(a.ws.active_off + j);
    __syncthreads();  // the previous item is done with xs and f.ent
    if (threadIdx.x < cnt) {
        const int en = __ldcg(a.ws.entries + off + threadIdx.x);
        f.ent[threadIdx.x] = en;
        f.shift[threadIdx.x] = prescale_shift(__uint_as_float(__ldcg(a.ws.ctl + a.p.ctl_hamax + en / K)));
    }
    __syncthreads();
    stage_f16_from_f32<true>(xs, f16_pitch(L), a.ws.h, L, cnt, [&](int t) { return f.ent[t] / K; }, f.shift, 0, L);
    __syncthreads();
    const int row0 = blk * kFsExpRows + warp * 16;
    const size_t eq = (size_t)e * I * (L / 2), es = (size_t)e * I * (L / 32);
    float accg[1][4] = {}, accu[1][4] = {};
    tile_fp4<1, true>(a.w.gate_q + eq, a.w.gate_s + es, a.w.up_q + eq, a.w.up_s + es, L / 2, L / 32, row0, 0, L / 128, xs,
                      f16_pitch(L), 0, 2 * cnt, accg, accu);
    // hi/lo columns: token q's values are (acc[0]+acc[1]) for row g and (acc[2]+acc[3]) for row g+8
    const int t = q;
    const bool ok = t < cnt;
    const float sc = ok ? exp2i(f.shift[t]) : 0.0f;
    const float g0 = (accg[0][0] + accg[0][1]) * sc, g1 = (accg[0][2] + accg[0][3]) * sc;
    const float u0 = (accu[0][0] + accu[0][1]) * sc, u1 = (accu[0][2] + accu[0][3]) * sc;
    const float a0 = g0 / (1.0f + expf(-g0)) * u0, a1 = g1 / (1.0f + expf(-g1)) * u1;
    float m = ok ? fmaxf(fabsf(a0), fabsf(a1)) : 0.0f;
    if (ok) {
        float *dst = a.ws.a + (size_t)f.ent[t] * I + row0;
        dst[g] = a0;
        dst[g + 8] = a1;
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
    if (ok && g == 0) atomicMax(a.ws.a_amax + f.ent[t], __float_as_uint(m));
    cta_signal_add(a.ws.ctl + a.p.ctl_gu + j, 1u);
}

// ---- shared down: 64 rows x full K (2 halves); sh_a staged once per CTA ----------------------------

DEVI void fs_sd(const StepArgs &a, int item, const uint16_t *xs, FsSmem &f) {
    const int H = a.d.H, Is = a.d.Is, B = a.B;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int tile = warp & 3, kh = warp >> 2;
    const int row0 = item * kFsSdRows + tile * 16, KW = Is / 2, k0 = kh * KW;
    float acc[1][4] = {};
    tile_fp4<1, false>(a.w.sh_down_q, a.w.sh_down_s, nullptr, nullptr, Is / 2, Is / 32, row0, k0, KW / 128, xs,
                       f16_pitch(Is), k0, 2 * B, acc, acc);
    for (int j = 0; j < 4; ++j) f.rf[warp][lane][j] = acc[0][j];
    __syncthreads();
    if (kh == 0) {
        float v[4];
        fs_sum(f, warp, 4, 2, 4, v);
        const int t = q;
        if (t < B) {
            const float sc = exp2i(f.shift[t]);
            a.ws.sh[(size_t)t * H + row0 + g] = (v[0] + v[1]) * sc;
            a.ws.sh[(size_t)t * H + row0 + g + 8] = (v[2] + v[3]) * sc;
        }
    }
    cta_signal_add(a.ws.ctl + CTL_SD_DONE, 1u);
}

// ---- expert down: 128 rows of L for one active expert, full K; combine completed tokens ------------

DEVI bool fs_edown(const StepArgs &a, int item, uint16_t *xs, FsSmem &f) {
    const int L = a.d.L, I = a.d.I, K = a.d.k;
    const int blocks = L / kFsExpRows, j = item / blocks, blk = item % blocks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    if (!cta_wait_geq(a, a.ws.ctl + a.p.ctl_gu + j, (unsigned)(I / kFsExpRows), &f.ok)) return false;
    const int e = __ldcg(a.ws.active_e + j), cnt = __ldcg(a.ws.active_cnt + j), off = __ldcg(a.ws.active_off + j);
    if (threadIdx.x < cnt) {
        const int en = __ldcg(a.ws.entries + off + threadIdx.x);
        f.ent[threadIdx.x] = en;
        f.shift[threadIdx.x] = prescale_shift(__uint_as_float(__ldcg(a.ws.a_amax + en)));
    }
    __syncthreads();
    stage_f16_from_f32<true>(xs, f16_pitch(I), a.ws.a, I, cnt, [&](int t) { return f.ent[t]; }, f.shift, 0, I);
    __syncthreads();
    const int row0 = blk * kFsExpRows + warp * 16;
    const size_t eq = (size_t)e * L * (I / 2), es = (size_t)e * L * (I / 32);
    float acc[1][4] = {};
    tile_fp4<1, false>(a.w.down_q + eq, a.w.down_s + es, nullptr, nullptr, I / 2, I / 32, row0, 0, I / 128, xs,
                       f16_pitch(I), 0, 2 * cnt, acc, acc);
    if (q < cnt) {
        const float sc = exp2i(f.shift[q]);
        float *dst = a.ws.y + (size_t)f.ent[q] * L + row0;
        dst[g] = (acc[0][0] + acc[0][1]) * sc;
        dst[g + 8] = (acc[0][2] + acc[0][3]) * sc;
    }
    // count this block's rows for every token; the item that completes a token's K slots combines
    __threadfence();
    __syncthreads();
    const int nb = L / kFsExpRows;
    if (threadIdx.x < cnt) {
        const int b = f.ent[threadIdx.x] / K;
        f.flag[threadIdx.x] = (atomicAdd(a.ws.ctl + a.p.ctl_comb + b * nb + blk, 1u) == (unsigned)(K - 1)) ? 1 : 0;
    }
    __syncthreads();
    int done = 0;
    for (int t = 0; t < cnt; ++t) {
        if (!f.flag[t]) continue;
        ++done;
        __threadfence();  // acquire: every slot's y rows of this block are visible
        const int b = f.ent[t] / K;
        for (int r = threadIdx.x; r < kFsExpRows; r += blockDim.x)
            a.ws.ylat[(size_t)b * L + blk * kFsExpRows + r] = combine_value(a, b, blk * kFsExpRows + r);
    }
    if (done) cta_signal_add(a.ws.ctl + a.p.ctl_ylat + blk, (unsigned)done);
    return true;
}

// ---- W_up: 64 rows x full K (2 halves); ylat staged once per CTA; out = bf16(W_up ylat + sh) ------

DEVI void fs_up(const StepArgs &a, int item, const uint16_t *xs, FsSmem &f) {
    const int H = a.d.H, L = a.d.L, B = a.B;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int tile = warp & 3, kh = warp >> 2;
    const int row0 = item * kFsUpRows + tile * 16, KW = L / 2, k0 = kh * KW;
    float acc[1][4] = {};
    tile_bf16<1>(a.w.w_up, L, row0, k0, KW / 32, xs, bf16_pitch(L), k0, 2 * B, acc);
    for (int j = 0; j < 4; ++j) f.rf[warp][lane][j] = acc[0][j];
    __syncthreads();
    if (kh == 0) {
        float v[4];
        fs_sum(f, warp, 4, 2, 4, v);
        const int t = q;
        if (t < B) {
            for (int h2 = 0; h2 < 2; ++h2) {
                const int r = row0 + g + 8 * h2;
                const float s = v[2 * h2] + v[2 * h2 + 1];
                if (a.ws.up_tap) a.ws.up_tap[(size_t)t * H + r] = s;
                const float shv = a.d.n_shared ? __ldcg(a.ws.sh + (size_t)t * H + r) : 0.0f;
                a.out[(size_t)t * H + r] = f32_to_bf16_rne(s + shv);
            }
        }
    }
    __syncthreads();
}

// ---- the kernel ---------------------------------------------------------------------------------------

__host__ __device__ inline size_t fused_small_smem(const StepArgs &a) {
    size_t m = (size_t)8 * bf16_pitch(a.d.H) * 2;                    // x, bf16
    auto mx = [&](size_t v) { m = v > m ? v : m; };
    mx((size_t)8 * f16_pitch(a.d.H) * 2);                              // x, fp16 (shared gate/up)
    mx((size_t)8 * f16_pitch(a.d.L) * 2);                              // h (expert gate/up)
    mx((size_t)8 * f16_pitch(a.d.I) * 2);                              // a (expert down)
    mx((size_t)8 * f16_pitch(a.d.Is) * 2);                             // sh_a (shared down)
    mx((size_t)8 * bf16_pitch(a.d.L) * 2);                             // ylat (W_up)
    return m;
}

__global__ void __launch_bounds__(256, 1) k_fused_small(StepArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ TopkSmem topk;
    __shared__ FsSmem f;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    unsigned *ctl = a.ws.ctl;
    const int H = a.d.H, L = a.d.L, I = a.d.I, Is = a.d.Is, B = a.B, E = a.d.E;
    bool alive = true;
    unsigned long long *trace = a.ws.trace ? a.ws.trace + (size_t)blockIdx.x * kTraceStamps : nullptr;
    auto stamp = [&](int i) {
        if (trace && threadIdx.x == 0) trace[i] = global_ns();
    };
    stamp(0);
    const int n_rt = (E + kFsRouterRows - 1) / kFsRouterRows, n_dn = L / kFsDnRows;
    const int n_sgu = a.d.n_shared ? Is / kFsSguRows : 0, n_sd = a.d.n_shared ? H / kFsSdRows : 0;
    const int n_up = H / kFsUpRows;

    // one item ahead: claim the next index when the current item starts, prefetch its weights
    auto queue = [&](int qi, int n, auto prefetch, auto body) {
        if (threadIdx.x == 0) f.item = (int)atomicAdd(ctl + CTL_QHEAD + qi, 1u);
        __syncthreads();
        int it = f.item;
        __syncthreads();
        if (it < n) prefetch(it);
        while (alive && it < n) {
            if (threadIdx.x == 0) f.item = (int)atomicAdd(ctl + CTL_QHEAD + qi, 1u);
            __syncthreads();
            const int nxt = f.item;
            __syncthreads();
            if (nxt < n) prefetch(nxt);
            alive = body(it);
            it = nxt;
        }
    };

    // x as bf16, 8 columns (zeros beyond B), for the router and W_dn
    stage_bf16(xs, bf16_pitch(H), a.x, H, B, 8, 0, H);
    __syncthreads();
    queue(Q_ROUTER_S, n_rt,
          [&](int it) {
              const int rows = min(kFsRouterRows, E - it * kFsRouterRows);
              if (rows > 0) fs_prefetch(a.w.router + (size_t)it * kFsRouterRows * H, (size_t)rows * H * 2);
          },
          [&](int it) { fs_router(a, it, xs, f); return true; });
    stamp(1);
    queue(Q_TOPK_S, B, [](int) {}, [&](int it) { return item_topk<true>(a, it, topk); });
    stamp(2);
    queue(Q_DN_S, n_dn, [&](int it) { fs_prefetch(a.w.w_dn + (size_t)it * kFsDnRows * H, (size_t)kFsDnRows * H * 2); },
          [&](int it) { fs_dn(a, it, xs, f); return true; });
    stamp(3);
    if (alive && n_sgu) {
        // x as fp16 with a per-token exponent (over all of H), no hi/lo split: bf16 fits in fp16
        __syncthreads();
        if (threadIdx.x < 8) f.flag[threadIdx.x] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < B * (H / 8); i += blockDim.x) {
            const int t = i / (H / 8), u = i % (H / 8);
            const uint4 v = *reinterpret_cast<const uint4 *>(a.x + (size_t)t * H + 8 * u);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
            atomicMax(reinterpret_cast<unsigned *>(&f.flag[t]), __float_as_uint(m));
        }
        __syncthreads();
        if (threadIdx.x < 8) f.xshift[threadIdx.x] = prescale_shift(__uint_as_float((unsigned)f.flag[threadIdx.x]));
        __syncthreads();
        stage_f16_from_bf16(xs, f16_pitch(H), a.x, H, B, f.xshift, 0, H);
        for (int i = threadIdx.x; i < (8 - B) * (H / 8); i += blockDim.x) {  // unused columns
            const int col = B + i / (H / 8), u = i % (H / 8);
            *reinterpret_cast<uint4 *>(xs + (size_t)col * f16_pitch(H) + 8 * u) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncthreads();
        queue(Q_SGU_S, n_sgu,
              [&](int it) {
                  const size_t r0 = (size_t)it * kFsSguRows;
                  fs_prefetch(a.w.sh_gate_q + r0 * (H / 2), (size_t)kFsSguRows * (H / 2));
                  fs_prefetch(a.w.sh_up_q + r0 * (H / 2), (size_t)kFsSguRows * (H / 2));
                  fs_prefetch(a.w.sh_gate_s + r0 * (H / 32), (size_t)kFsSguRows * (H / 32));
                  fs_prefetch(a.w.sh_up_s + r0 * (H / 32), (size_t)kFsSguRows * (H / 32));
              },
              [&](int it) { fs_sgu(a, it, xs, f); return true; });
    }
    stamp(4);
    if (alive) alive = cta_wait_geq(a, ctl + CTL_ROUTE_READY, 1u, &f.ok);
    if (alive) alive = cta_wait_geq(a, ctl + CTL_DN_DONE, (unsigned)n_dn, &f.ok);
    stamp(5);
    if (alive) {
        const int blocks = I / kFsExpRows;
        const int n = __ldcg(a.ws.n_active) * blocks;
        queue(Q_EGU_S, n,
              [&](int it) {
                  const int e = __ldcg(a.ws.active_e + it / blocks);
                  const size_t r0 = (size_t)e * I + (size_t)(it % blocks) * kFsExpRows;
                  fs_prefetch(a.w.gate_q + r0 * (L / 2), (size_t)kFsExpRows * (L / 2));
                  fs_prefetch(a.w.up_q + r0 * (L / 2), (size_t)kFsExpRows * (L / 2));
                  fs_prefetch(a.w.gate_s + r0 * (L / 32), (size_t)kFsExpRows * (L / 32));
                  fs_prefetch(a.w.up_s + r0 * (L / 32), (size_t)kFsExpRows * (L / 32));
              },
              [&](int it) { fs_egu(a, it, xs, f); return true; });
    }
    stamp(6);
    if (alive && n_sd) {
        alive = cta_wait_geq(a, ctl + CTL_SGU_DONE, (unsigned)n_sgu, &f.ok);
        if (alive) {
            if (threadIdx.x < B) f.shift[threadIdx.x] = prescale_shift(__uint_as_float(__ldcg(ctl + a.p.ctl_shamax + threadIdx.x)));
            __syncthreads();
            stage_f16_from_f32<true>(xs, f16_pitch(Is), a.ws.sh_a, Is, B, [](int t) { return t; }, f.shift, 0, Is);
            __syncthreads();
            queue(Q_SD_S, n_sd,
                  [&](int it) {
                      const size_t r0 = (size_t)it * kFsSdRows;
                      fs_prefetch(a.w.sh_down_q + r0 * (Is / 2), (size_t)kFsSdRows * (Is / 2));
                      fs_prefetch(a.w.sh_down_s + r0 * (Is / 32), (size_t)kFsSdRows * (Is / 32));
                  },
                  [&](int it) { fs_sd(a, it, xs, f); return true; });
        }
    }
    stamp(7);
    if (alive) {
        const int blocks = L / kFsExpRows;
        const int n = __ldcg(a.ws.n_active) * blocks;
        queue(Q_EDOWN_S, n,
              [&](int it) {
                  const int e = __ldcg(a.ws.active_e + it / blocks);
                  const size_t r0 = (size_t)e * L + (size_t)(it % blocks) * kFsExpRows;
                  fs_prefetch(a.w.down_q + r0 * (I / 2), (size_t)kFsExpRows * (I / 2));
                  fs_prefetch(a.w.down_s + r0 * (I / 32), (size_t)kFsExpRows * (I / 32));
              },
              [&](int it) { return fs_edown(a, it, xs, f); });
    }
    stamp(8);
    if (alive) {
        // ylat (every token, every row) and sh must be final; each thread polls one ylat block
        __syncthreads();
        int ok = 1;
        for (int blk = threadIdx.x; blk < L / kFsExpRows; blk += blockDim.x)
            ok &= wait_geq(a, ctl + a.p.ctl_ylat + blk, (unsigned)B) ? 1 : 0;
        if (threadIdx.x == 0 && a.d.n_shared) ok &= wait_geq(a, ctl + CTL_SD_DONE, (unsigned)n_sd) ? 1 : 0;
        __threadfence();
        alive = __syncthreads_and(ok) != 0;
        if (alive) {
            stage_bf16split_from_f32(xs, bf16_pitch(L), a.ws.ylat, L, B, 0, L);
            for (int i = threadIdx.x; i < (8 - 2 * B) * (L / 8); i += blockDim.x) {  // unused columns
                const int col = 2 * B + i / (L / 8), u = i % (L / 8);
                *reinterpret_cast<uint4 *>(xs + (size_t)col * bf16_pitch(L) + 8 * u) = make_uint4(0u, 0u, 0u, 0u);
            }
            __syncthreads();
            queue(Q_UP_S, n_up,
                  [&](int it) { fs_prefetch(a.w.w_up + (size_t)it * kFsUpRows * L, (size_t)kFsUpRows * L * 2); },
                  [&](int it) { fs_up(a, it, xs, f); return true; });
        }
    }
    stamp(9);
    // leave; the last CTA out clears the control block for the next step
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        f.ok = (atomicAdd(ctl + CTL_EXIT, 1u) == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    stamp(10);
    if (f.ok) {
        __threadfence();
        for (int i = threadIdx.x; i < CTL_FIXED; i += blockDim.x) ctl[i] = 0u;
        for (int i = threadIdx.x; i < E; i += blockDim.x) ctl[a.p.ctl_gu + i] = 0u;
        for (int i = threadIdx.x; i < B * (L / kFsExpRows); i += blockDim.x) ctl[a.p.ctl_comb + i] = 0u;
        for (int i = threadIdx.x; i < L / kFsExpRows; i += blockDim.x) ctl[a.p.ctl_ylat + i] = 0u;
        for (int i = threadIdx.x; i < B; i += blockDim.x) {
            ctl[a.p.ctl_hamax + i] = 0u;
            ctl[a.p.ctl_shamax + i] = 0u;
        }
    }
}

bool fused_small_supports(const Dims &d, int B) {
    // full-K items: H/8 and H/4 split evenly into bf16 (32) and MXFP4 (128) rounds, I_s/2 into
    // MXFP4 rounds; at most 4 tokens so that hi/lo columns of every part fit one 8-column tile
    return B <= 4 && d.H % 512 == 0 && d.L % 128 == 0 && d.I % 128 == 0 && (d.n_shared == 0 || d.Is % 256 == 0);
}

cudaError_t launch_fused_small(const StepArgs &a, cudaStream_t s, int n_sm) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_sm);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = fused_small_smem(a);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_fused_small, a);
}

cudaError_t init_fused_small_attributes() {
    return cudaFuncSetAttribute(k_fused_small, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
}

}  // namespace moedec
