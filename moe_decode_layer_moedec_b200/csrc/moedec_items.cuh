// moedec_items.cuh -- the work items of one decode layer step.
//
// Each item is one unit of the step: a router row block x K range, one token's top-k, a W_dn /
// shared-expert / W_up row block x K range (whole CTA), or 16 rows of one routed expert (one
// warp).  The same items run in two schedules:
//   FUSED = false  one kernel per part, ordered by the stream (moedec_kernels.cu);
//   FUSED = true   one persistent kernel whose CTAs pull items from in-order queues and wait on
//                  completion counters (moedec_fused.cu).
// The fused schedule is this library's form of the "megakernel" of the Kimi K3 decode work: the
// parts of the step no longer wait for one another at kernel boundaries, and the weights of an
// item are streamed before its inputs are ready ("NVIDIA uses a 12,000-line Megakernel to
// optimize Kimi K3 inference…", section 一个工程师、1.2万行代码、AI辅助开发; "快是可以生成的，可信
// 只能证明", section 他们换掉了什么, where every technique removes waiting).
#pragma once

#include "moedec_router.cuh"
#include "moedec_tiles.cuh"

namespace moedec {

constexpr unsigned kFlagTestStall = 4u;           // MOEDEC_FLAG_TEST_STALL (see include/moedec.h)
constexpr unsigned kFlagTestStallExperts = 128u;  // MOEDEC_FLAG_TEST_STALL_EXPERTS

// ---------------------------------------------------------------------------------------------
// device-side synchronisation of the fused step

DEVI unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

DEVI unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Thread-level bounded wait for *p >= target.  Gives up when another CTA has aborted the step,
// or after a.p.wait_limit_ns, in which case it records kErrTimeout and sets the abort word.
DEVI bool wait_geq(const StepArgs &a, const unsigned *p, unsigned target) {
    if (ld_acquire(p) >= target) return true;
    unsigned *ctl = a.ws.ctl;
    const unsigned long long t0 = global_ns();
    unsigned ns = 32;
    for (;;) {
        __nanosleep(ns);
        if (ns < 256) ns <<= 1;
        if (ld_acquire(p) >= target) return true;
        if (ld_acquire(ctl + CTL_ABORT)) return false;
        if ((long long)(global_ns() - t0) > a.p.wait_limit_ns) {
            atomicOr(a.ws.err, kErrTimeout);
            atomicExch(ctl + CTL_ABORT, 1u);
            return false;
        }
    }
}

// CTA-wide wait (thread 0 waits; every thread returns the outcome).
DEVI bool cta_wait_geq(const StepArgs &a, const unsigned *p, unsigned target, int *s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        *s_ok = wait_geq(a, p, target) ? 1 : 0;
        __threadfence();
    }
    __syncthreads();
    return *s_ok != 0;
}

DEVI bool warp_wait_geq(const StepArgs &a, const unsigned *p, unsigned target) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) {
        ok = wait_geq(a, p, target) ? 1 : 0;
        __threadfence();
    }
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Publish every prior write of the CTA, then add v to *counter (all threads call it).
DEVI void cta_signal_add(unsigned *counter, unsigned v) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) atomicAdd(counter, v);
}

DEVI void warp_signal_add(unsigned *counter, unsigned v) {
    __threadfence();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) atomicAdd(counter, v);
}

// ---------------------------------------------------------------------------------------------
// Work claiming.  Items of a queue are uniform, and every queue's length is known when a CTA
// reaches it, so CTA c owns the contiguous range [n*c/G, n*(c+1)/G) of each queue and its warps
// take items from it with a shared-memory counter: no global atomic (a queue head is one L2
// address that thousands of warps would otherwise serialise on) and no lock.

struct CtaTake {
    int next[8];
};

// by every thread of the CTA before the first take (a __syncthreads must follow)
DEVI void cta_take_init(CtaTake &t) {
    for (int i = threadIdx.x; i < 8; i += blockDim.x) t.next[i] = 0;
}

// next item of queue q (n items) of the range [n c / G, n (c + 1) / G) that CTA c of a group of
// G CTAs owns, for the calling thread (one lane per warp), or -1 once the range is used up
DEVI int cta_take(CtaTake &t, int q, int n, int c, int G) {
    const int lo = (int)((long long)n * c / G), hi = (int)((long long)n * (c + 1) / G);
    const int k = atomicAdd(t.next + q, 1);
    return lo + k < hi ? lo + k : -1;
}

// the same over the whole grid
DEVI int cta_take(CtaTake &t, int q, int n) { return cta_take(t, q, n, (int)blockIdx.x, (int)gridDim.x); }

// ---------------------------------------------------------------------------------------------
// router: one router row block x K range (fp64 MMAs); the block's last CTA publishes logits

template <bool FUSED>
DEVI void item_router(const StepArgs &a, int bid, unsigned char *smem, unsigned *s_flag) {
    const bool last = router_block(a, bid, smem, s_flag);
    if (FUSED && last && !(a.flags & kFlagTestStall)) cta_signal_add(a.ws.ctl + CTL_RT_DONE, 1u);
}

// ---------------------------------------------------------------------------------------------
// h = W_dn x: one 128-row block x K range (bf16 MMAs); the block's last CTA publishes h rows and
// folds their per-token max |h| into the token's staging exponent

// MAXB: tokens per step at most (sizes the per-token shared arrays of the dense items)
template <bool FUSED, int NT, int MAXB = kMaxBatch>
DEVI void item_dn(const StepArgs &a, int bid, unsigned char *smem, unsigned *s_flag) {
    __shared__ unsigned s_amax[MAXB];
    const int L = a.d.L, H = a.d.H, B = a.B, maxB = a.d.max_batch;
    const int rb = bid / a.p.dn.splits, ks = bid % a.p.dn.splits;
    const int KR = a.p.dn.krange, k0 = ks * KR;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    const int pitch = bf16_pitch(KR);
    const int warp = threadIdx.x >> 5;
    const int row0 = rb * kDenseRows + warp * 16;
    float *part = a.ws.dn_part + (size_t)ks * maxB * L;
    // token groups of 8 NT columns (one group up to 64 tokens; larger batches re-read the rows)
    for (int tg = 0; tg < B; tg += 8 * NT) {
        const int nb = min(8 * NT, B - tg);
        __syncthreads();
        stage_bf16(xs, pitch, a.x + (size_t)tg * H, H, nb, 8 * NT, k0, KR);
        __syncthreads();
        if (row0 < L) {
            float acc[NT][4] = {};
            tile_bf16<NT>(a.w.w_dn, H, row0, k0, KR / 32, xs, pitch, 0, nb, acc);
            tile_foreach<NT, false>(acc, nb, [&](int t, int r, float v) { part[(size_t)(tg + t) * L + row0 + r] = v; });
        }
    }
    if (cta_ticket_last(a.ws.tickets + a.p.ticket_dn + rb, a.p.dn.splits, s_flag)) {
        for (int t = threadIdx.x; t < B; t += blockDim.x) s_amax[t] = 0u;
        __syncthreads();
        constexpr int NP = 4;  // (row, token) sums per thread and pass, their loads in flight together
        for (int i0 = threadIdx.x; i0 < kDenseRows * B; i0 += NP * blockDim.x) {
            const float *pp[NP];
            bool ok[NP];
            size_t o[NP];
            float sum[NP];
            int bb[NP];
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                const int i = i0 + j * blockDim.x, r = rb * kDenseRows + (i % kDenseRows);
                bb[j] = i / kDenseRows;
                ok[j] = i < kDenseRows * B && r < L;
                o[j] = ok[j] ? (size_t)bb[j] * L + r : 0;
                pp[j] = a.ws.dn_part + o[j];
            }
            sum_splits_batch<NP, 8>(pp, ok, (size_t)maxB * L, a.p.dn.splits, sum);
#pragma unroll
            for (int j = 0; j < NP; ++j)
                if (ok[j]) {
                    a.ws.h[o[j]] = sum[j];
                    atomicMax(s_amax + bb[j], __float_as_uint(fabsf(sum[j])));
                }
        }
        __syncthreads();
        for (int t = threadIdx.x; t < B; t += blockDim.x) atomicMax(a.ws.ctl + a.p.ctl_hamax + t, s_amax[t]);
        if (FUSED) cta_signal_add(a.ws.ctl + CTL_DN_DONE, 1u);
    }
}

// ---------------------------------------------------------------------------------------------
// top-k of one token (any block size >= 256, up to 4 experts per thread), then, in the last
// token's CTA, the per-expert token buckets

struct TopkSmem {
    unsigned hist[256];
    int warp[32];
    unsigned key[kMaxTopK];
    int e[kMaxTopK];
    int rank_e[kMaxTopK];
    float rank_s[kMaxTopK];
    unsigned digit, want;
    int ok;
    unsigned flag;
};

// Shared memory of item_topk's candidate and bucket lists (bytes): max(E ceil(B / 64), 256) words
// of selection masks (the warps' candidates first), then E offsets.  Callers place it in dynamic
// shared memory that is free while the top-k runs.
__host__ __device__ inline size_t topk_lists_smem(int E, int B) {
    const size_t w = (size_t)E * ((B + 63) / 64);
    return (w > 256 ? w : 256) * 8 + (size_t)E * 4;
}

// Warp maximum of the lanes' N packed words; the lane holding it clears it (words are unique
// apart from 0, which only ever ties with another 0).  Returns the maximum to every lane.  Two
// warp reductions (high halves, then the low halves of the lanes that hold the highest high
// half) instead of a shuffle tree: the rounds of a selection are a dependent chain.
template <int N>
DEVI unsigned long long warp_take_best(unsigned long long (&w)[N]) {
    unsigned long long m = w[0];
#pragma unroll
    for (int i = 1; i < N; ++i) m = w[i] > m ? w[i] : m;
    const unsigned hi = __reduce_max_sync(0xffffffffu, (unsigned)(m >> 32));
    const unsigned lo = __reduce_max_sync(0xffffffffu, (unsigned)(m >> 32) == hi ? (unsigned)m : 0u);
    const unsigned long long best = ((unsigned long long)hi << 32) | lo;
#pragma unroll
    for (int i = 0; i < N; ++i)
        if (w[i] == best) w[i] = 0ull;
    return best;
}

// FUSED: first wait until CTL_RT_DONE reaches rt_done (the schedule's count of router signals).
// zero_rows: when given, the token's row of it ([B][L]) is zeroed before the routing is
// published (the small-batch step adds the expert outputs into ylat).
// acc64: when given, the logits are the fp64 sums there ([B][E]): they are rounded to fp32 into
// ws.logits and the accumulator is cleared; otherwise ws.logits already holds them.
// lists: topk_lists_smem(E, B) bytes of shared memory (16-byte aligned) for the warps' candidates,
// the bucket builder's token masks (ceil(B / 64) words per expert) and the experts' offsets.
template <bool FUSED>
DEVI bool item_topk(const StepArgs &a, int b, TopkSmem &t, unsigned char *lists, unsigned rt_done = 0u,
                    unsigned long long *stamps = nullptr, float *zero_rows = nullptr, double *acc64 = nullptr) {
    const int E = a.d.E, K = a.d.k, B = a.B;
    unsigned long long *masks = reinterpret_cast<unsigned long long *>(lists);
    int *offs = reinterpret_cast<int *>(lists + topk_lists_smem(E, B) - (size_t)E * 4);
    if (FUSED && !cta_wait_geq(a, a.ws.ctl + CTL_RT_DONE, rt_done, &t.ok)) return false;
    // optional trace (global ns): logits complete, keys, warp candidates, ranked, routing
    // written, expert masks, buckets written, buckets published
    auto stamp = [&](int i) {
        if (stamps && threadIdx.x == 0) stamps[i] = global_ns();
    };
    stamp(0);
    const int tid = threadIdx.x;
    // thread tid owns experts 4*tid .. 4*tid+3 (index order follows thread order); all four
    // logits are loaded before the first score is computed (one memory round trip, not four)
    unsigned key[4];
    bool valid[4];
    float lg[4];
    if (acc64) {
        double v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            valid[i] = 4 * tid + i < E;
            v[i] = valid[i] ? __ldcg(acc64 + (size_t)b * E + 4 * tid + i) : 0.0;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            lg[i] = (float)v[i];
            if (valid[i]) {
                a.ws.logits[(size_t)b * E + 4 * tid + i] = lg[i];
                acc64[(size_t)b * E + 4 * tid + i] = 0.0;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            valid[i] = 4 * tid + i < E;
            lg[i] = valid[i] ? __ldcg(a.ws.logits + (size_t)b * E + 4 * tid + i) : 0.0f;
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float sc = router_score(lg[i]);
        key[i] = valid[i] && sc >= 0.0f ? __float_as_uint(sc) : 0u;  // non-negative fp32 orders like its bits
    }
    stamp(1);
    // Selection on packed words (score bits << 32 | ~expert): a larger word ranks first (higher
    // score, then lower expert index), 0 is no expert.  Each warp takes its K best by K rounds of
    // a warp maximum whose holder drops the word; the warps' candidates are then ranked by
    // counting, which yields the top K in rank order.
    const int lane = tid & 31, warp = tid >> 5, nw = (int)(blockDim.x >> 5);
    unsigned long long P[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        P[i] = valid[i] ? ((unsigned long long)key[i] << 32) | (0xffffffffu - (unsigned)(4 * tid + i)) : 0ull;
    unsigned long long *cand = masks;  // nw * K candidates; the expert masks are built after
    for (int r = 0; r < K; ++r) {
        const unsigned long long m = warp_take_best(P);
        if (lane == 0) cand[warp * K + r] = m;
    }
    __syncthreads();
    stamp(2);
    // The warps' candidates ranked at once: a candidate's rank is the number of larger candidates
    // (the packed words are unique, 0 is none), so the K best land in rank order.  (Selecting
    // them by K more rounds of a warp maximum costs K dependent shuffle chains.)
    const int nc = nw * K;
    for (int c = tid; c < nc; c += blockDim.x) {
        const unsigned long long m = cand[c];
        int rank = 0;
        for (int j = 0; j < nc; ++j) rank += cand[j] > m ? 1 : 0;
        if (rank < K && m != 0ull) {
            t.rank_e[rank] = (int)(0xffffffffu - (unsigned)(m & 0xffffffffull));
            t.rank_s[rank] = __uint_as_float((unsigned)(m >> 32));
        }
    }
    __syncthreads();
    stamp(3);
    if (warp == 0) {
        float S = 0.0f;  // sum of the selected scores in rank order
        for (int r = 0; r < K; ++r) S += t.rank_s[r];
        if (lane < K) {
            a.ws.idx[(size_t)b * K + lane] = t.rank_e[lane];
            a.ws.wts[(size_t)b * K + lane] = t.rank_s[lane] / S;
        }
    }
    if (zero_rows)
        for (int i = tid; i < a.d.L / 4; i += blockDim.x)
            reinterpret_cast<float4 *>(zero_rows + (size_t)b * a.d.L)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();
    stamp(4);
    // A shard of an expert-parallel layer keeps only the selections of its own experts
    // [e0, e0 + ne) (bucketed by local index e - e0); the W_up items still wait for B K counts per
    // ylat block, so the selections of other shards' experts are counted here at once.
    const int e0 = a.d.e0, e1 = a.d.e0 + a.d.ne;
    if (B == 1) {
        // one token: its K distinct experts are the buckets (one entry each), in expert order
        if (warp == 0) {
            const int er = lane < K ? t.rank_e[lane] : -1;
            const bool local = er >= e0 && er < e1;
            const int e = local ? er : 0x7fffffff;
            int pos = 0;
            for (int j = 0; j < K; ++j) pos += __shfl_sync(0xffffffffu, e, j) < e ? 1 : 0;
            const int n_local = __popc(__ballot_sync(0xffffffffu, local));
            if (local) {
                a.ws.active_e[pos] = e - e0;
                a.ws.active_cnt[pos] = 1;
                a.ws.active_off[pos] = pos;
                a.ws.entries[pos] = lane;
            }
            if (lane < K) a.ws.a_amax[lane] = 0u;
            if (lane == 0) *a.ws.n_active = n_local;
            if (FUSED && n_local < K)
                for (int i = lane; i < a.d.L / 16; i += 32) atomicAdd(a.ws.ctl + a.p.ctl_ylat + i, (unsigned)(K - n_local));
        }
        stamp(6);
        if (FUSED) cta_signal_add(a.ws.ctl + CTL_ROUTE_READY, 1u);
        stamp(7);
        return true;
    }
    // the last token's CTA groups the B*K selections by expert: one bit per (expert, token) in W
    // words per expert, so that an expert's entries come out token-ascending (the position of a
    // selection is the number of lower tokens of its expert)
    if (!cta_ticket_last(a.ws.tickets + a.p.ticket_topk, (unsigned)B, &t.flag)) return true;
    const int W = (B + 63) / 64;
    unsigned long long *mk = masks;  // [E][W]
    auto sel_e = [&](int i) { return __ldcg(a.ws.idx + i); };
    for (int i = tid; i < E * W; i += blockDim.x) mk[i] = 0ull;
    __syncthreads();
    for (int i = tid; i < B * K; i += blockDim.x) {
        const int ex = sel_e(i), tb = i / K;
        if (ex < 0 || ex >= E) atomicOr(a.ws.err, kErrBucket);
        else if (ex >= e0 && ex < e1) atomicOr(&mk[ex * W + tb / 64], 1ull << (tb % 64));
        a.ws.a_amax[i] = 0u;
    }
    __syncthreads();
    stamp(5);
    int cnt[4], n_act_t = 0, n_ent_t = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = 4 * tid + i;
        cnt[i] = 0;
        if (e < E)
            for (int w = 0; w < W; ++w) cnt[i] += __popcll(mk[e * W + w]);
        n_act_t += cnt[i] > 0 ? 1 : 0;
        n_ent_t += cnt[i];
    }
    int n_act, n_ent;
    int j = block_exclusive_scan(n_act_t, t.warp, &n_act);
    int off = block_exclusive_scan(n_ent_t, t.warp, &n_ent);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = 4 * tid + i;
        if (e < E) offs[e] = off;
        if (cnt[i] > 0) {
            a.ws.active_e[j] = e - e0;
            a.ws.active_cnt[j] = cnt[i];
            a.ws.active_off[j] = off;
            ++j;
        }
        off += cnt[i];
    }
    if (tid == 0) *a.ws.n_active = n_act;
    if (FUSED && n_ent < B * K)
        for (int i = tid; i < a.d.L / 16; i += blockDim.x) atomicAdd(a.ws.ctl + a.p.ctl_ylat + i, (unsigned)(B * K - n_ent));
    __syncthreads();
    for (int i = tid; i < B * K; i += blockDim.x) {
        const int ex = sel_e(i), tb = i / K;
        if (ex < e0 || ex >= e1) continue;
        const unsigned long long *m = mk + ex * W;
        int pos = offs[ex] + __popcll(m[tb / 64] & ((1ull << (tb % 64)) - 1ull));
        for (int w = 0; w < tb / 64; ++w) pos += __popcll(m[w]);
        a.ws.entries[pos] = i;
    }
    stamp(6);
    if (FUSED) cta_signal_add(a.ws.ctl + CTL_ROUTE_READY, 1u);
    stamp(7);
    return true;
}

// ylat[b][l] = sum_r w[b][r] y[b*K + r][l] in slot order (all loads issued before the sum); a
// shard of an expert-parallel layer sums the slots of its own experts only
DEVI float combine_value(const StepArgs &a, int b, int l) {
    const int L = a.d.L, K = a.d.k;
    const bool all = a.d.ne == a.d.E;
    float wv[kMaxTopK], yv[kMaxTopK];
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r)
        if (r < K) {
            const int e = all ? 0 : __ldcg(a.ws.idx + (size_t)b * K + r) - a.d.e0;
            const bool local = all || (e >= 0 && e < a.d.ne);
            wv[r] = local ? __ldcg(a.ws.wts + (size_t)b * K + r) : 0.0f;
            yv[r] = local ? __ldcg(a.ws.y + ((size_t)b * K + r) * L + l) : 0.0f;
        }
    float s = 0.0f;
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r)
        if (r < K) s += wv[r] * yv[r];
    return s;
}

// ---------------------------------------------------------------------------------------------
// The step's expert buckets, copied into shared memory once per CTA when the routing is out, so
// that the routed items of the fused schedules read them from there instead of paying a global
// round trip each.  NEXP >= active experts (min(E, B k)), NENT >= entries (B k).
template <int NEXP, int NENT>
struct RouteTables {
    int n_active;
    int e[NEXP], cnt[NEXP], off[NEXP];
    int ent[NENT];
    float w[NENT];  // routing weight of each entry
};

// all threads; every load is issued before the first use (one round trip); a barrier must follow
template <int NEXP, int NENT>
DEVI void cta_load_routing(const StepArgs &a, RouteTables<NEXP, NENT> &r) {
    const int n = a.B * a.d.k, n_exp = n < a.d.E ? n : a.d.E;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        int e = 0, c = 0, o = 0;
        if (i < n_exp) {
            e = __ldcg(a.ws.active_e + i);
            c = __ldcg(a.ws.active_cnt + i);
            o = __ldcg(a.ws.active_off + i);
        }
        const int en = __ldcg(a.ws.entries + i);
        const float w = __ldcg(a.ws.wts + i);
        if (i < n_exp) {
            r.e[i] = e;
            r.cnt[i] = c;
            r.off[i] = o;
        }
        r.ent[i] = en;
        r.w[i] = w;
    }
    if (threadIdx.x == 0) r.n_active = __ldcg(a.ws.n_active);
}

using SplitKRoute = RouteTables<kMaxExperts, kMaxEntries>;

// ---------------------------------------------------------------------------------------------
// routed experts: one warp = 16 rows of one active expert for up to 16 of its tokens

template <int NT, bool SPLIT>
DEVI void warp_expert_gu(const StepArgs &a, uint16_t *xs, int e, int tile, const int *ent, const int *shift, int ntok) {
    const int L = a.d.L, I = a.d.I, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int ncols = SPLIT ? 2 * ntok : ntok;
    const int pitch = f16_pitch(kKChunk);
    const int row0 = tile * 16;
    const size_t eq = (size_t)e * I * (L / 2), es = (size_t)e * I * (L / 32);
    float accg[NT][4] = {}, accu[NT][4] = {};
    const int K = a.d.k;
    for (int kc0 = 0; kc0 < L; kc0 += kKChunk) {
        const int kc = min(kKChunk, L - kc0);
        __syncwarp();
        stage_f16_from_f32<SPLIT>(xs, pitch, a.ws.h, L, ntok, [&](int t) { return ent[t] / K; }, shift, kc0, kc, lane, 32);
        __syncwarp();
        // gate rows then up rows through one copy of the tile code (one weight stream live at a time)
#pragma unroll 1
        for (int m = 0; m < 2; ++m) {
            float acc[NT][4];
#pragma unroll
            for (int i = 0; i < NT; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = m ? accu[i][j] : accg[i][j];
            tile_fp4<NT, false>(m ? a.w.up_q + eq : a.w.gate_q + eq, m ? a.w.up_s + es : a.w.gate_s + es, nullptr, nullptr,
                                L / 2, L / 32, row0, kc0, kc / 128, xs, pitch, 0, ncols, acc, acc);
#pragma unroll
            for (int i = 0; i < NT; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (m) accu[i][j] = acc[i][j];
                    else accg[i][j] = acc[i][j];
                }
        }
    }
    // a = silu(g) * u; the per-token max |a| over these 16 rows feeds the down item's staging
    constexpr int PER_NT = SPLIT ? 1 : 2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int j = 0; j < PER_NT; ++j) {
            const int tk = SPLIT ? nt * 4 + q : nt * 8 + 2 * q + j;
            const bool ok = tk < ntok;
            const float sc = ok ? exp2i(shift[tk]) : 0.0f;
            float g0, g1, u0, u1;
            if (SPLIT) {
                g0 = accg[nt][0] + accg[nt][1];
                g1 = accg[nt][2] + accg[nt][3];
                u0 = accu[nt][0] + accu[nt][1];
                u1 = accu[nt][2] + accu[nt][3];
            } else {
                g0 = accg[nt][j];
                g1 = accg[nt][2 + j];
                u0 = accu[nt][j];
                u1 = accu[nt][2 + j];
            }
            g0 *= sc;
            g1 *= sc;
            u0 *= sc;
            u1 *= sc;
            const float a0 = g0 / (1.0f + expf(-g0)) * u0, a1 = g1 / (1.0f + expf(-g1)) * u1;
            float m = ok ? fmaxf(fabsf(a0), fabsf(a1)) : 0.0f;
            if (ok) {
                float *dst = a.ws.a + (size_t)ent[tk] * I + row0;
                dst[g] = a0;
                dst[g + 8] = a1;
            }
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
            if (ok && g == 0) atomicMax(a.ws.a_amax + ent[tk], __float_as_uint(m));
        }
    }
}

// y rows of 16-row block `tile` for the warp's tokens.  FUSED folds the combine in: each
// token's rows, times its routing weight (ent_w), are added into ylat with fp32 reductions and
// the block's ylat count grows by the number of tokens (complete at B k).
template <bool FUSED, int NT, bool SPLIT>
DEVI void warp_expert_down(const StepArgs &a, uint16_t *xs, int e, int tile, const int *ent, const int *shift, int ntok,
                           const float *ent_w = nullptr) {
    const int L = a.d.L, I = a.d.I, K = a.d.k, lane = threadIdx.x & 31;
    const int ncols = SPLIT ? 2 * ntok : ntok;
    const int pitch = f16_pitch(kKChunk);
    const int row0 = tile * 16;
    const size_t eq = (size_t)e * L * (I / 2), es = (size_t)e * L * (I / 32);
    float acc[NT][4] = {};
    for (int kc0 = 0; kc0 < I; kc0 += kKChunk) {
        const int kc = min(kKChunk, I - kc0);
        __syncwarp();
        stage_f16_from_f32<SPLIT>(xs, pitch, a.ws.a, I, ntok, [&](int t) { return ent[t]; }, shift, kc0, kc, lane, 32);
        __syncwarp();
        tile_fp4<NT, false>(a.w.down_q + eq, a.w.down_s + es, nullptr, nullptr, I / 2, I / 32, row0, kc0, kc / 128, xs,
                            pitch, 0, ncols, acc, acc);
    }
    if (FUSED) {
        tile_foreach<NT, SPLIT>(acc, ntok, [&](int t, int r, float v) {
            atomicAdd(a.ws.ylat + (size_t)(ent[t] / K) * L + row0 + r, v * exp2i(shift[t]) * ent_w[t]);
        });
        warp_signal_add(a.ws.ctl + a.p.ctl_ylat + tile, (unsigned)ntok);
        return;
    }
    tile_foreach<NT, SPLIT>(acc, ntok, [&](int t, int r, float v) {
        a.ws.y[(size_t)ent[t] * L + row0 + r] = v * exp2i(shift[t]);
    });
}

// One warp item: 16 rows (`tile`) of active expert slot j, all its tokens in groups of 16.
// Returns false if the fused step was aborted while waiting.
// rt (FUSED): the routing tables in shared memory; w_ent / w_shift / w_w: the warp's scratch
// for a group's entries, exponents and (down) routing weights.
template <bool FUSED, bool DOWN>
DEVI bool warp_expert_item(const StepArgs &a, uint16_t *xs, int item, int *w_ent, int *w_shift,
                           const SplitKRoute *rt = nullptr, float *w_w = nullptr) {
    const int tiles = (DOWN ? a.d.L : a.d.I) / 16;
    const int j = item / tiles, tile = item % tiles, lane = threadIdx.x & 31, K = a.d.k;
    if (FUSED && DOWN && !warp_wait_geq(a, a.ws.ctl + a.p.ctl_gu + j, (unsigned)(a.d.I / 16))) return false;
    int e, cnt, off;
    if (FUSED) {
        e = rt->e[j];
        cnt = rt->cnt[j];
        off = rt->off[j];
    } else {
        e = __ldcg(a.ws.active_e + j);
        cnt = __ldcg(a.ws.active_cnt + j);
        off = __ldcg(a.ws.active_off + j);
    }
    for (int t0 = 0; t0 < cnt; t0 += kExpertTokGroup) {
        const int ntok = min(kExpertTokGroup, cnt - t0);
        __syncwarp();
        if (lane < ntok) {
            const int ent = FUSED ? rt->ent[off + t0 + lane] : __ldcg(a.ws.entries + off + t0 + lane);
            w_ent[lane] = ent;
            if (FUSED && DOWN) w_w[lane] = rt->w[ent];
            const unsigned amax = DOWN ? __ldcg(a.ws.a_amax + ent) : __ldcg(a.ws.ctl + a.p.ctl_hamax + ent / K);
            w_shift[lane] = prescale_shift(__uint_as_float(amax));
        }
        __syncwarp();
        if (DOWN) {
            if (ntok <= 4) warp_expert_down<FUSED, 1, true>(a, xs, e, tile, w_ent, w_shift, ntok, w_w);
            else if (ntok <= 8) warp_expert_down<FUSED, 1, false>(a, xs, e, tile, w_ent, w_shift, ntok, w_w);
            else warp_expert_down<FUSED, 2, false>(a, xs, e, tile, w_ent, w_shift, ntok, w_w);
        } else {
            if (ntok <= 4) warp_expert_gu<1, true>(a, xs, e, tile, w_ent, w_shift, ntok);
            else if (ntok <= 8) warp_expert_gu<1, false>(a, xs, e, tile, w_ent, w_shift, ntok);
            else warp_expert_gu<2, false>(a, xs, e, tile, w_ent, w_shift, ntok);
        }
    }
    if (FUSED && !DOWN) warp_signal_add(a.ws.ctl + a.p.ctl_gu + j, 1u);
    return true;
}

// smem per warp of the expert items: staged columns x (kKChunk + pad) halfs
__host__ __device__ __forceinline__ int expert_warp_cols(int B) { return B <= 8 ? 8 : 16; }
__host__ __device__ __forceinline__ size_t expert_warp_smem(int B) {
    return (size_t)expert_warp_cols(B) * f16_pitch(kKChunk) * 2;
}

// ---------------------------------------------------------------------------------------------
// combine for the multi-kernel schedule: ylat[b][l] = sum_r w[b][r] y[b*K + r][l]

DEVI void combine_rows(const StepArgs &a, int b, int l) { a.ws.ylat[(size_t)b * a.d.L + l] = combine_value(a, b, l); }

// ---------------------------------------------------------------------------------------------
// up-projection: one 128-row block of W_up x K range; the block's last CTA writes
// out = bf16(W_up ylat + sh).  ylat enters as bf16 hi/lo column pairs.

template <bool FUSED, int NT>
DEVI bool item_up(const StepArgs &a, int bid, unsigned char *smem, unsigned *s_flag, int *s_ok) {
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    const int H = a.d.H, L = a.d.L, B = a.B, maxB = a.d.max_batch;
    const int rb = bid / a.p.up.splits, ks = bid % a.p.up.splits;
    const int KR = a.p.up.krange, k0 = ks * KR;
    const int kc = up_chunk(NT, KR);
    const int pitch = bf16_pitch(kc);
    const int warp = threadIdx.x >> 5;
    const int row0 = rb * kDenseRows + warp * 16;
    if (FUSED) {
        // ylat rows k0 .. k0+KR of every token must be final: one thread per 16-row block waits
        // (they all poll at once), then the CTA agrees on the outcome
        const int nblk = KR / 16;
        int ok = 1;
        if (threadIdx.x < nblk) {
            ok = wait_geq(a, a.ws.ctl + a.p.ctl_ylat + k0 / 16 + threadIdx.x, (unsigned)(B * a.d.k)) ? 1 : 0;
            __threadfence();
        }
        if (!__syncthreads_and(ok)) return false;
    }
    // token groups of 4 NT tokens (hi/lo column pairs fill the 8 NT columns)
    for (int tg = 0; tg < B; tg += 4 * NT) {
        const int nb = min(4 * NT, B - tg);
        float acc[NT][4] = {};
        for (int c0 = k0; c0 < k0 + KR; c0 += kc) {
            __syncthreads();
            stage_bf16split_from_f32(xs, pitch, a.ws.ylat + (size_t)tg * L, L, nb, c0, kc);
            for (int i = threadIdx.x; i < (8 * NT - 2 * nb) * (kc / 8); i += blockDim.x) {  // unused columns
                const int col = 2 * nb + i / (kc / 8), u = i % (kc / 8);
                *reinterpret_cast<uint4 *>(xs + (size_t)col * pitch + 8 * u) = make_uint4(0u, 0u, 0u, 0u);
            }
            __syncthreads();
            if (row0 < H) tile_bf16<NT>(a.w.w_up, L, row0, c0, kc / 32, xs, pitch, 0, 2 * nb, acc);
        }
        if (row0 < H) {
            float *part = a.ws.up_part + (size_t)ks * maxB * H;
            tile_foreach<NT, true>(acc, nb, [&](int t, int r, float v) { part[(size_t)(tg + t) * H + row0 + r] = v; });
        }
    }
    if (cta_ticket_last(a.ws.tickets + a.p.ticket_up + rb, a.p.up.splits, s_flag)) {
        if (FUSED && a.d.n_shared && !cta_wait_geq(a, a.ws.ctl + CTL_SD_DONE, (unsigned)a.p.sd.blocks, s_ok)) return false;
        constexpr int NP = 4;
        for (int i0 = threadIdx.x; i0 < kDenseRows * B; i0 += NP * blockDim.x) {
            const float *pp[NP];
            bool ok[NP];
            size_t o[NP];
            float sum[NP], shv[NP];
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                const int i = i0 + j * blockDim.x, r = rb * kDenseRows + (i % kDenseRows), b = i / kDenseRows;
                ok[j] = i < kDenseRows * B && r < H;
                o[j] = ok[j] ? (size_t)b * H + r : 0;
                pp[j] = a.ws.up_part + o[j];
                shv[j] = (ok[j] && a.d.n_shared) ? __ldcg(a.ws.sh + o[j]) : 0.0f;
            }
            sum_splits_batch<NP, 8>(pp, ok, (size_t)maxB * H, a.p.up.splits, sum);
#pragma unroll
            for (int j = 0; j < NP; ++j)
                if (ok[j]) {
                    if (a.ws.up_tap) a.ws.up_tap[o[j]] = sum[j];
                    if (a.out_f32) a.out_f32[o[j]] = sum[j] + shv[j];
                    else a.out[o[j]] = f32_to_bf16_rne(sum[j] + shv[j]);
                }
        }
    }
    return true;
}

// ---------------------------------------------------------------------------------------------
// shared expert.  gate/up: 128 rows of I_s (gate, then up) x K range of H; down: 128 rows of H
// x K range of I_s.  Tokens are staged as fp16 with a per-token exponent over the K range.

template <bool FUSED, int NT, int MAXB = kMaxBatch>
DEVI void item_sgu(const StepArgs &a, int bid, unsigned char *smem, unsigned *s_flag) {
    __shared__ int s_shift[MAXB];
    __shared__ unsigned s_amax[MAXB];
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    const int H = a.d.H, Is = a.d.Is, B = a.B, maxB = a.d.max_batch;
    const int rb = bid / a.p.sgu.splits, ks = bid % a.p.sgu.splits;
    const int KR = a.p.sgu.krange, k0 = ks * KR;
    const int pitch = f16_pitch(KR);
    __syncthreads();
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
    const int warp = threadIdx.x >> 5;
    const int row0 = rb * kDenseRows + warp * 16;
    float *part = a.ws.sgu_part + (size_t)ks * maxB * 2 * Is;
    for (int tg = 0; tg < B; tg += 8 * NT) {
        const int nb = min(8 * NT, B - tg);
        __syncthreads();
        stage_f16_from_bf16(xs, pitch, a.x + (size_t)tg * H, H, nb, s_shift + tg, k0, KR);
        __syncthreads();
        if (row0 < Is) {
#pragma unroll 1
            for (int m = 0; m < 2; ++m) {
                float acc[NT][4] = {};
                tile_fp4<NT, false>(m ? a.w.sh_up_q : a.w.sh_gate_q, m ? a.w.sh_up_s : a.w.sh_gate_s, nullptr, nullptr,
                                    H / 2, H / 32, row0, k0, KR / 128, xs, pitch, 0, nb, acc, acc);
                tile_foreach<NT, false>(acc, nb, [&](int t, int r, float v) {
                    part[(size_t)(tg + t) * 2 * Is + m * Is + row0 + r] = v * exp2i(s_shift[tg + t]);
                });
            }
        }
    }
    if (cta_ticket_last(a.ws.tickets + a.p.ticket_sgu + rb, a.p.sgu.splits, s_flag)) {
        constexpr int NR = 2;  // (row, token) pairs per thread and pass: gate and up sums of each
        for (int i0 = threadIdx.x; i0 < kDenseRows * B; i0 += NR * blockDim.x) {
            const float *pp[2 * NR];
            bool ok[2 * NR];
            size_t o[NR];
            float sum[2 * NR];
#pragma unroll
            for (int j = 0; j < NR; ++j) {
                const int i = i0 + j * blockDim.x, r = rb * kDenseRows + (i % kDenseRows), b = i / kDenseRows;
                ok[2 * j] = ok[2 * j + 1] = i < kDenseRows * B && r < Is;
                o[j] = ok[2 * j] ? (size_t)b * Is + r : 0;
                pp[2 * j] = a.ws.sgu_part + (ok[2 * j] ? (size_t)b * 2 * Is + r : 0);
                pp[2 * j + 1] = pp[2 * j] + Is;
            }
            sum_splits_batch<2 * NR, 8>(pp, ok, (size_t)maxB * 2 * Is, a.p.sgu.splits, sum);
#pragma unroll
            for (int j = 0; j < NR; ++j)
                if (ok[2 * j]) {
                    const float gs = sum[2 * j], us = sum[2 * j + 1];
                    a.ws.sh_a[o[j]] = gs / (1.0f + expf(-gs)) * us;
                }
        }
        if (FUSED) cta_signal_add(a.ws.ctl + CTL_SGU_DONE, 1u);
    }
}

template <bool FUSED, int NT, bool SPLIT, int MAXB = kMaxBatch>
DEVI bool item_sd(const StepArgs &a, int bid, unsigned char *smem, unsigned *s_flag, int *s_ok) {
    __shared__ int s_shift[MAXB];
    __shared__ unsigned s_amax[MAXB];
    if (FUSED && !cta_wait_geq(a, a.ws.ctl + CTL_SGU_DONE, (unsigned)a.p.sgu.blocks, s_ok)) return false;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);
    const int H = a.d.H, Is = a.d.Is, B = a.B, maxB = a.d.max_batch;
    const int rb = bid / a.p.sd.splits, ks = bid % a.p.sd.splits;
    const int KR = a.p.sd.krange, k0 = ks * KR;
    const int pitch = f16_pitch(KR);
    __syncthreads();
    for (int t = threadIdx.x; t < B; t += blockDim.x) s_amax[t] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < B * (KR / 4); i += blockDim.x) {
        const int t = i / (KR / 4), u = i % (KR / 4);
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.ws.sh_a + (size_t)t * Is + k0) + u);
        atomicMax(s_amax + t, __float_as_uint(fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)))));
    }
    __syncthreads();
    for (int t = threadIdx.x; t < B; t += blockDim.x) s_shift[t] = prescale_shift(__uint_as_float(s_amax[t]));
    const int warp = threadIdx.x >> 5;
    const int row0 = rb * kDenseRows + warp * 16;
    float *part = a.ws.sd_part + (size_t)ks * maxB * H;
    constexpr int GT = SPLIT ? 4 * NT : 8 * NT;  // tokens per group
    for (int tg = 0; tg < B; tg += GT) {
        const int nb = min(GT, B - tg);
        __syncthreads();
        stage_f16_from_f32<SPLIT>(xs, pitch, a.ws.sh_a + (size_t)tg * Is, Is, nb, [](int t) { return t; }, s_shift + tg, k0,
                                  KR);
        __syncthreads();
        if (row0 < H) {
            float acc[NT][4] = {};
            tile_fp4<NT, false>(a.w.sh_down_q, a.w.sh_down_s, nullptr, nullptr, Is / 2, Is / 32, row0, k0, KR / 128, xs,
                                pitch, 0, SPLIT ? 2 * nb : nb, acc, acc);
            tile_foreach<NT, SPLIT>(acc, nb, [&](int t, int r, float v) {
                part[(size_t)(tg + t) * H + row0 + r] = v * exp2i(s_shift[tg + t]);
            });
        }
    }
    if (cta_ticket_last(a.ws.tickets + a.p.ticket_sd + rb, a.p.sd.splits, s_flag)) {
        constexpr int NP = 4;
        for (int i0 = threadIdx.x; i0 < kDenseRows * B; i0 += NP * blockDim.x) {
            const float *pp[NP];
            bool ok[NP];
            size_t o[NP];
            float sum[NP];
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                const int i = i0 + j * blockDim.x, r = rb * kDenseRows + (i % kDenseRows), b = i / kDenseRows;
                ok[j] = i < kDenseRows * B && r < H;
                o[j] = ok[j] ? (size_t)b * H + r : 0;
                pp[j] = a.ws.sd_part + o[j];
            }
            sum_splits_batch<NP, 8>(pp, ok, (size_t)maxB * H, a.p.sd.splits, sum);
#pragma unroll
            for (int j = 0; j < NP; ++j)
                if (ok[j]) a.ws.sh[o[j]] = sum[j];
        }
        if (FUSED) cta_signal_add(a.ws.ctl + CTL_SD_DONE, 1u);
    }
    return true;
}

// ---------------------------------------------------------------------------------------------
// L2 prefetch for the cross-layer hint

// Router rows [E c / G, E (c+1) / G) of the layer that steps next (a.next_router), one row per
// thread: the cross-layer hint, issued by CTAs that have no work left in this step.
DEVI void prefetch_next_router(const StepArgs &a, int c, int G) {
    if (!a.next_router) return;
    const int E = a.d.E, lo = (int)((long long)E * c / G), hi = (int)((long long)E * (c + 1) / G);
    for (int r = lo + (int)threadIdx.x; r < hi; r += blockDim.x)
        prefetch_l2(a.next_router + (size_t)r * a.d.H, (uint32_t)a.d.H * 2);
}

// ---------------------------------------------------------------------------------------------
// token-column tiles of each dense part for batch B

__host__ __device__ __forceinline__ int nt_for_cols(int cols) {
    return cols <= 8 ? 1 : cols <= 16 ? 2 : cols <= 32 ? 4 : cols <= 64 ? 8 : 16;
}

}  // namespace moedec
