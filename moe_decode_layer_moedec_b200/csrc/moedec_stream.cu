// moedec_stream.cu -- the decode layer step for 1-2 tokens as four launches of a kernel of
// streaming warps.
//
// Batch 1-2 is the pages' small-matrix range of the Kimi K3 decode path ("快是可以生成的，可信
// 只能证明（vLLM 重写 Kimi K3 解码路径…）", section 他们换掉了什么), and there the step is pure
// weight streaming: 148 MB per full-size layer step at batch 1.  A loaded HBM access on B200 takes
// about 2 us, so each SM must keep ~100 KB of weights in flight at all times.
//
// Each warp owns a ring of 3 shared-memory slots and streams its work items through it with bulk
// copies (cp.async.bulk, the tensor memory accelerator's 1-D form): a slot holds one stage of one
// item, 16 weight rows of 256 bytes (128 bf16 or 512 MXFP4 elements) plus, for MXFP4, the rows'
// 16 E8M0 scale bytes, and completes on its own mbarrier.  One lane per row issues the copy, so a
// stage costs the warp a handful of instructions; the warp issues the next stages (of its next
// items) before it computes the current one, so its copies never drain between items.
//
// The step is four launches; each runs only work whose inputs earlier launches finished, so no
// warp ever waits on another's results:
//   1  router (16 rows x K range, fp64 MMAs; the warp that completes the last row group ranks the
//      experts and builds the expert buckets), W_dn, shared gate/up        (x)
//   2  shared down, expert gate/up of the active experts                  (sh_a, h)
//   3  expert down; completing a token's 16 latent rows combines them      (a)
//   4  W_up and the output                                                 (ylat, sh)
// A launch stages the activation it reads in every CTA once, as MMA operands (bf16, or fp16 hi/lo
// columns scaled by a power of two per token or expert entry), while its first copies fly.
#include <algorithm>

#include "moedec_items.cuh"

namespace moedec {

namespace {

constexpr int kStWarps = 12;
constexpr int kStStages = 3;
constexpr int kStMaxBatch = 2;
constexpr int kSlotSc = 4096, kSlotBytes = 4352;  // 16 rows x 256 B, then 16 rows x 16 scale bytes
constexpr int kRingBytes = kStWarps * kStStages * kSlotBytes;
constexpr int kMaxActive = 64;       // active experts at <= 2 tokens x <= 32 slots
constexpr int kMaxEdownExperts = 2;  // experts of one CTA's expert-down range (see stream_supports)

enum StQueue { SQ_RT = 0, SQ_DN, SQ_SGU, SQ_SD, SQ_EGU, SQ_EDOWN, SQ_UP, SQ_N };

struct SlotMeta {
    int q, item, c, n;  // queue, item, stage within the item, stages of the item
};

struct StSmem {
    unsigned long long bar[kStWarps][kStStages];  // one mbarrier per slot
    SlotMeta meta[kStWarps][kStStages];
    int route_state;  // 0 not loaded, 1 loading, 2 loaded, 3 aborted
    int n_active;
    int act_e[kMaxActive], act_cnt[kMaxActive], act_off[kMaxActive], ent[kMaxActive];
    int tk_idx[kMaxActive], srt_e[kMaxActive], srt_i[kMaxActive], first_pos[kMaxActive + 1];
    int shift[2 * kMaxEdownExperts * kStMaxBatch];  // staging exponents of the launch's columns
    unsigned amax[2 * kMaxEdownExperts * kStMaxBatch];
    int ed_j0;  // expert-down launch: first active slot staged by this CTA
    int exit_last;
    CtaTake claim;
};

// ---------------------------------------------------------------------------------------------
// bulk copies and their barriers

DEVI uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

DEVI void mbar_init(unsigned long long *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
// one arrival that also announces `bytes` of copies completing on the barrier
DEVI void mbar_arrive_expect_tx(unsigned long long *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
DEVI bool mbar_test(unsigned long long *bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// global -> shared bulk copy (16-byte aligned, size a multiple of 16) completing on `bar`
DEVI void bulk_copy(uint32_t dst, const void *src, unsigned bytes, unsigned long long *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// Bounded wait for phase `parity` of a slot's barrier (all lanes).  The copies always complete;
// the limit only bounds a broken run.
DEVI bool slot_wait(const StepArgs &a, unsigned long long *bar, unsigned parity) {
    if (mbar_test(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        if (mbar_test(bar, parity)) return true;
        if ((long long)(global_ns() - t0) > a.p.wait_limit_ns) {
            if ((threadIdx.x & 31) == 0) {
                atomicOr(a.ws.err, kErrTimeout);
                atomicExch(a.ws.ctl + CTL_ABORT, 1u);
            }
            return false;
        }
    }
}

// ---------------------------------------------------------------------------------------------
// the step's geometry

struct Geo {
    int H, L, E, K, I, Is, B, ns;  // ns: 1 with a shared expert
};

DEVI Geo geo(const StepArgs &a) {
    Geo g;
    g.H = a.d.H; g.L = a.d.L; g.E = a.d.E; g.K = a.d.k; g.I = a.d.I; g.Is = a.d.Is; g.B = a.B;
    g.ns = a.d.n_shared ? 1 : 0;
    return g;
}

DEVI int queue_len(const StepArgs &a, const Geo &g, int q, int n_active) {
    const StreamPlan &p = a.p.st;
    switch (q) {
        case SQ_RT: return g.E / 16 * p.s_rt;
        case SQ_DN: return g.L / 16 * p.s_dn;
        case SQ_SGU: return g.ns ? g.Is / 16 * p.s_sgu : 0;
        case SQ_EGU: return n_active * (g.I / 16) * p.s_egu;
        case SQ_SD: return g.ns ? g.H / 16 * p.s_sd : 0;
        case SQ_EDOWN: return n_active * (g.L / 16);
        case SQ_UP: return g.H / 16 * p.s_up;
    }
    return 0;
}

struct Item {
    int a, b, ks;  // row tile (or active slot j and tile b), K split
};

// item it of queue q; stages: bf16 128 k each, MXFP4 512 k each (gate and up alternate in pairs)
DEVI Item decode_item(const StepArgs &a, const Geo &g, int q, int it, int *n_stages) {
    const StreamPlan &p = a.p.st;
    Item r = {0, 0, 0};
    switch (q) {
        case SQ_RT: r.a = it / p.s_rt; r.ks = it % p.s_rt; *n_stages = p.kr_rt / 128; break;
        case SQ_DN: r.a = it / p.s_dn; r.ks = it % p.s_dn; *n_stages = p.kr_dn / 128; break;
        case SQ_SGU: r.a = it / p.s_sgu; r.ks = it % p.s_sgu; *n_stages = 2 * (p.kr_sgu / 512); break;
        case SQ_EGU: {
            const int jt = it / p.s_egu, tiles = g.I / 16;
            r.ks = it % p.s_egu; r.a = jt / tiles; r.b = jt % tiles; *n_stages = 2 * (p.kr_egu / 512);
            break;
        }
        case SQ_SD: r.a = it / p.s_sd; r.ks = it % p.s_sd; *n_stages = p.kr_sd / 512; break;
        case SQ_EDOWN: r.a = it / (g.L / 16); r.b = it % (g.L / 16); *n_stages = g.I / 512; break;
        case SQ_UP: r.ks = it / (g.H / 16); r.a = it % (g.H / 16); *n_stages = p.kr_up / 128; break;  // K major
        default: *n_stages = 0; break;
    }
    return r;
}

// ---------------------------------------------------------------------------------------------
// stage issue: lane r < 16 copies weight row r of the stage (256 B); for MXFP4, lane 16 + r copies
// the row's 16 scale bytes.  The per-lane sources are computed once per item.

struct IssuePlan {
    const unsigned char *src;  // this lane's copy source at stage 0 (matrix 0)
    long long dmat;            // MXFP4 gate/up pairs: offset of the up matrix's matching source
    int step;                  // bytes the source advances per stage of one matrix
    unsigned bytes;            // bytes of this lane's copy
    uint32_t dst;              // its offset in a slot
    unsigned expect;           // bytes of one stage
    bool pair;
};

DEVI IssuePlan make_plan(const StepArgs &a, const Geo &g, const StSmem &sm, int q, const Item &t) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, r = lane & 15;
    IssuePlan P;
    P.dmat = 0;
    P.pair = (q == SQ_SGU || q == SQ_EGU);
    if (q == SQ_RT || q == SQ_DN || q == SQ_UP) {
        const uint16_t *W = q == SQ_RT ? a.w.router : q == SQ_DN ? a.w.w_dn : a.w.w_up;
        const int ld = q == SQ_UP ? g.L : g.H;
        const int k0 = t.ks * (q == SQ_RT ? p.kr_rt : q == SQ_DN ? p.kr_dn : p.kr_up);
        P.src = reinterpret_cast<const unsigned char *>(W + (size_t)(16 * t.a + r) * ld + k0);
        P.step = 256;
        P.bytes = lane < 16 ? 256u : 0u;
        P.dst = r * 256;
        P.expect = 16 * 256;
        return P;
    }
    const uint8_t *Q, *S;
    size_t ldq, lds, row0;
    int k0;
    if (q == SQ_SGU) {
        Q = a.w.sh_gate_q; S = a.w.sh_gate_s; ldq = g.H / 2; lds = g.H / 32; row0 = (size_t)16 * t.a;
        k0 = t.ks * p.kr_sgu;
        P.dmat = lane < 16 ? (long long)(a.w.sh_up_q - a.w.sh_gate_q) : (long long)(a.w.sh_up_s - a.w.sh_gate_s);
    } else if (q == SQ_EGU) {
        Q = a.w.gate_q; S = a.w.gate_s; ldq = g.L / 2; lds = g.L / 32;
        row0 = (size_t)sm.act_e[t.a] * g.I + 16 * t.b;
        k0 = t.ks * p.kr_egu;
        P.dmat = lane < 16 ? (long long)(a.w.up_q - a.w.gate_q) : (long long)(a.w.up_s - a.w.gate_s);
    } else if (q == SQ_SD) {
        Q = a.w.sh_down_q; S = a.w.sh_down_s; ldq = g.Is / 2; lds = g.Is / 32; row0 = (size_t)16 * t.a;
        k0 = t.ks * p.kr_sd;
    } else {  // SQ_EDOWN
        Q = a.w.down_q; S = a.w.down_s; ldq = g.I / 2; lds = g.I / 32;
        row0 = (size_t)sm.act_e[t.a] * g.L + 16 * t.b;
        k0 = 0;
    }
    if (lane < 16) {
        P.src = Q + (row0 + r) * ldq + k0 / 2;
        P.step = 256;
        P.bytes = 256;
        P.dst = r * 256;
    } else {
        P.src = S + (row0 + r) * lds + k0 / 32;
        P.step = 16;
        P.bytes = 16;
        P.dst = kSlotSc + r * 16;
    }
    P.expect = 16 * 256 + 16 * 16;
    return P;
}

DEVI void issue_stage(const IssuePlan &P, unsigned char *slot, unsigned long long *bar, int c) {
    const int kk = P.pair ? (c >> 1) : c;
    if ((threadIdx.x & 31) == 0) mbar_arrive_expect_tx(bar, P.expect);
    __syncwarp();
    if (P.bytes) {
        const unsigned char *src = P.src + (P.pair && (c & 1) ? P.dmat : 0) + (long long)P.step * kk;
        bulk_copy(smem_addr(slot) + P.dst, src, P.bytes, bar);
    }
}

// ---------------------------------------------------------------------------------------------
// stage compute (weights from the slot, activation columns from the CTA's staging)

// bf16: 16 rows x 128 k; B column g is staged column col (or zero when col < 0)
DEVI void mma_stage_bf16(const unsigned char *slot, const uint16_t *xs, int pitch, int kofs, int col,
                         float (&acc0)[4], float (&acc1)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const unsigned char *ra = slot + g * 256 + 16 * q, *rb = ra + 8 * 256;
    const uint16_t *xr = xs + (size_t)(col >= 0 ? col : 0) * pitch + kofs + 8 * q;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const uint4 A = *reinterpret_cast<const uint4 *>(ra + 64 * r);
        const uint4 Bm = *reinterpret_cast<const uint4 *>(rb + 64 * r);
        uint4 xb = *reinterpret_cast<const uint4 *>(xr + 32 * r);
        if (col < 0) xb = make_uint4(0u, 0u, 0u, 0u);
        mma_bf16(acc0, A.x, Bm.x, A.y, Bm.y, xb.x, xb.y);
        mma_bf16(acc1, A.z, Bm.z, A.w, Bm.w, xb.z, xb.w);
    }
}

// router: 16 rows (two 8-row groups) x 128 k in fp64 (slot q of step s of a 32-k chunk holds
// k = 8q + s); column g is token g
DEVI void mma_stage_router(const unsigned char *slot, const uint16_t *xs, int pitch, int kofs, int B,
                           double (&c)[2][2], double (&d)[2][2]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const uint16_t *xr = xs + (size_t)(g < B ? g : 0) * pitch + kofs + 8 * q;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        uint4 xb = *reinterpret_cast<const uint4 *>(xr + 32 * r);
        if (g >= B) xb = make_uint4(0u, 0u, 0u, 0u);
        const double xv[8] = {bf16_lo(xb.x), bf16_hi(xb.x), bf16_lo(xb.y), bf16_hi(xb.y),
                              bf16_lo(xb.z), bf16_hi(xb.z), bf16_lo(xb.w), bf16_hi(xb.w)};
#pragma unroll
        for (int G = 0; G < 2; ++G) {
            const uint4 A = *reinterpret_cast<const uint4 *>(slot + (8 * G + g) * 256 + 64 * r + 16 * q);
            const double av[8] = {bf16_lo(A.x), bf16_hi(A.x), bf16_lo(A.y), bf16_hi(A.y),
                                  bf16_lo(A.z), bf16_hi(A.z), bf16_lo(A.w), bf16_hi(A.w)};
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                mma_f64(c[G][0], c[G][1], av[2 * s], xv[2 * s]);
                mma_f64(d[G][0], d[G][1], av[2 * s + 1], xv[2 * s + 1]);
            }
        }
    }
}

// MXFP4: 16 rows x 512 k (4 rounds of 128 k); lane quad q owns 32-element block 4r + q of each
// row; word w of its 16 code bytes holds MMA steps 2w, 2w+1 against staged unit kofs/8 + 16r +
// 4q + w (fp16 staging layout, swizzled); two accumulator chains
DEVI void mma_stage_fp4(const unsigned char *slot, const uint16_t *xs, int pitch, int kofs, int col,
                        float (&acc0)[4], float (&acc1)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, sh = 8 * q;
    const uint16_t *xc = xs + (size_t)(col >= 0 ? col : 0) * pitch;
    const int ubase = kofs / 8 + 4 * q, flip = q >> 1;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const uint4 c0 = *reinterpret_cast<const uint4 *>(slot + g * 256 + 64 * r + 16 * q);
        const uint4 c1 = *reinterpret_cast<const uint4 *>(slot + (g + 8) * 256 + 64 * r + 16 * q);
        const uint32_t s0 = *reinterpret_cast<const uint32_t *>(slot + kSlotSc + g * 16 + 4 * r);
        const uint32_t s1 = *reinterpret_cast<const uint32_t *>(slot + kSlotSc + (g + 8) * 16 + 4 * r);
        const uint32_t f0 = e8m0_to_f16x2((s0 >> sh) & 0xffu), f1 = e8m0_to_f16x2((s1 >> sh) & 0xffu);
        const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w}, w1[4] = {c1.x, c1.y, c1.z, c1.w};
        const int u = ubase + 16 * r;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint4 v = *reinterpret_cast<const uint4 *>(xc + 8 * ((u + w) ^ flip));
            if (col < 0) v = make_uint4(0u, 0u, 0u, 0u);
            uint32_t d0[4], d1[4];
            fp4_decode_word(w0[w], f0, d0);
            fp4_decode_word(w1[w], f1, d1);
            mma_f16(acc0, d0[0], d1[0], d0[1], d1[1], v.x, v.y);
            mma_f16(acc1, d0[2], d1[2], d0[3], d1[3], v.z, v.w);
        }
    }
}

// ---------------------------------------------------------------------------------------------
// tickets and flags

DEVI bool warp_last_of(unsigned *counter, unsigned expected) {
    __threadfence();
    __syncwarp();
    unsigned last = 0;
    if ((threadIdx.x & 31) == 0) {
        last = (atomicAdd(counter, 1u) == expected - 1u) ? 1u : 0u;
        if (last) *counter = 0u;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) __threadfence();
    return last != 0;
}

// add 1 to *counter after this warp's writes; true in every lane for the warp that made it `target`
DEVI bool warp_count_reaches(unsigned *counter, unsigned target) {
    __threadfence();
    __syncwarp();
    unsigned hit = 0;
    if ((threadIdx.x & 31) == 0) hit = (atomicAdd(counter, 1u) == target - 1u) ? 1u : 0u;
    hit = __shfl_sync(0xffffffffu, hit, 0);
    if (hit) __threadfence();
    return hit != 0;
}

DEVI void warp_publish(unsigned *flag, unsigned v) {
    __threadfence();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) atomicExch(flag, v);
}

// ---------------------------------------------------------------------------------------------
// routing: top-k per token and the expert buckets (one warp, after every logit is final)

// lane-local best of 32 keys, skipping the ones marked in `gone`: largest key, the lowest index
// among equal keys (tree, ties keep the left = lower index)
DEVI void best_of32(const unsigned (&key)[32], unsigned gone, unsigned &bk, int &bi) {
    unsigned k[16];
    int ix[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const unsigned k0 = (gone >> (2 * j) & 1u) ? 0u : key[2 * j];
        const unsigned k1 = (gone >> (2 * j + 1) & 1u) ? 0u : key[2 * j + 1];
        const bool r = k1 > k0;
        k[j] = r ? k1 : k0;
        ix[j] = r ? 2 * j + 1 : 2 * j;
    }
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) {
            const bool r = k[2 * j + 1] > k[2 * j];
            k[j] = r ? k[2 * j + 1] : k[2 * j];
            ix[j] = r ? ix[2 * j + 1] : ix[2 * j];
        }
    bk = k[0];
    bi = ix[0];
}

// top-k of token b: K rounds of a warp argmax over the keys (score desc, expert index asc), so the
// experts come out in rank order; weights = score / (fp32 sum of the scores in rank order)
DEVI void st_topk_token(const StepArgs &a, const Geo &g, StSmem &sm, int b) {
    const int lane = threadIdx.x & 31, E = g.E, K = g.K;
    // key = fp32 score bits + 1 (non-negative floats order like their bits), written with the
    // logits; 0 marks "no expert".  Expert e = lane + 32 i sits in key[i] of lane e % 32.
    unsigned key[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? __ldcg(a.ws.st_key + (size_t)b * E + e) : 0u;
    }
    unsigned bk, gone = 0u;
    int bi;
    best_of32(key, gone, bk, bi);
    float S = 0.0f, my_s = 0.0f;
    int my_e = 0;
    for (int r = 0; r < K; ++r) {
        const unsigned mk = __reduce_max_sync(0xffffffffu, bk);
        const unsigned me = __reduce_min_sync(0xffffffffu, bk == mk ? (unsigned)(lane + 32 * bi) : 0xffffffffu);
        const float sc = __uint_as_float(mk - 1u);
        S += sc;
        if (lane == r) {
            my_e = (int)me;
            my_s = sc;
        }
        if (lane == (int)(me & 31u)) {
            gone |= 1u << (me >> 5);
            best_of32(key, gone, bk, bi);
        }
    }
    if (lane < K) {
        a.ws.idx[(size_t)b * K + lane] = my_e;
        a.ws.wts[(size_t)b * K + lane] = my_s / S;
        sm.tk_idx[b * K + lane] = my_e;
    }
    __syncwarp();
}

// expert buckets of the B*K (<= 64) selections: entries i = b*K + r sorted by (expert, i)
DEVI void st_buckets(const StepArgs &a, const Geo &g, StSmem &sm) {
    const int lane = threadIdx.x & 31, N = g.B * g.K;
    // keys (expert << 6 | i) are distinct; lane holds entries lane and lane + 32
    const unsigned k0 = lane < N ? ((unsigned)sm.tk_idx[lane] << 6 | (unsigned)lane) : 0xffffffffu;
    const unsigned k1 = lane + 32 < N ? ((unsigned)sm.tk_idx[lane + 32] << 6 | (unsigned)(lane + 32)) : 0xffffffffu;
    int r0 = 0, r1 = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const unsigned a0 = __shfl_sync(0xffffffffu, k0, j), a1 = __shfl_sync(0xffffffffu, k1, j);
        r0 += (a0 < k0) + (a1 < k0);
        r1 += (a0 < k1) + (a1 < k1);
    }
    if (lane < N) {
        sm.srt_e[r0] = (int)(k0 >> 6);
        sm.srt_i[r0] = lane;
    }
    if (lane + 32 < N) {
        sm.srt_e[r1] = (int)(k1 >> 6);
        sm.srt_i[r1] = lane + 32;
    }
    __syncwarp();
    int n_first = 0;
#pragma unroll
    for (int p0 = 0; p0 < 64; p0 += 32) {
        const int p = p0 + lane;
        const bool first = p < N && (p == 0 || sm.srt_e[p - 1] != sm.srt_e[p]);
        const unsigned m = __ballot_sync(0xffffffffu, first);
        if (first) sm.first_pos[n_first + __popc(m & ((1u << lane) - 1u))] = p;
        n_first += __popc(m);
    }
    if (lane == 0) sm.first_pos[n_first] = N;
    __syncwarp();
#pragma unroll
    for (int j0 = 0; j0 < 64; j0 += 32) {
        const int j = j0 + lane;
        if (j < n_first) {
            const int p = sm.first_pos[j];
            a.ws.active_e[j] = sm.srt_e[p];
            a.ws.active_off[j] = p;
            a.ws.active_cnt[j] = sm.first_pos[j + 1] - p;
        }
        if (j < N) a.ws.entries[j] = sm.srt_i[j];
    }
    if (lane == 0) *a.ws.n_active = n_first;
    warp_publish(a.ws.ctl + CTL_ROUTE_READY, 1u);
}

// the CTA's copy of the routing tables (first warp to need it loads it; an earlier launch made it)
DEVI bool ensure_routing(const StepArgs &a, StSmem &sm) {
    const int lane = threadIdx.x & 31;
    volatile int *state = &sm.route_state;
    if (*state == 2) return true;
    int mine = 0;
    if (lane == 0) mine = atomicCAS(&sm.route_state, 0, 1) == 0 ? 1 : 0;
    mine = __shfl_sync(0xffffffffu, mine, 0);
    if (mine) {
        if (!warp_wait_geq(a, a.ws.ctl + CTL_ROUTE_READY, 1u)) {
            if (lane == 0) atomicExch(&sm.route_state, 3);
            return false;
        }
        const int n = __ldcg(a.ws.n_active);
        for (int j = lane; j < n && j < kMaxActive; j += 32) {
            sm.act_e[j] = __ldcg(a.ws.active_e + j);
            sm.act_cnt[j] = __ldcg(a.ws.active_cnt + j);
            sm.act_off[j] = __ldcg(a.ws.active_off + j);
        }
        for (int p = lane; p < a.B * a.d.k && p < kMaxActive; p += 32) sm.ent[p] = __ldcg(a.ws.entries + p);
        if (lane == 0) sm.n_active = n;
        __threadfence_block();
        __syncwarp();
        if (lane == 0) atomicExch(&sm.route_state, 2);
        return true;
    }
    const unsigned long long t0 = global_ns();
    for (;;) {
        const int s = *state;
        if (s == 2) break;
        if (s == 3) return false;
        if (*(volatile unsigned *)(a.ws.ctl + CTL_ABORT)) return false;
        if ((long long)(global_ns() - t0) > a.p.wait_limit_ns) {
            if (lane == 0) {
                atomicOr(a.ws.err, kErrTimeout);
                atomicExch(a.ws.ctl + CTL_ABORT, 1u);
            }
            return false;
        }
        __nanosleep(64);
    }
    __threadfence_block();
    return true;
}

// ---------------------------------------------------------------------------------------------
// epilogues (after the last stage of an item); accumulator entry j of a lane is row g (j < 2) or
// g + 8 (j >= 2), MMA column 2q + (j & 1)

struct Acc {
    float f[2][2][4];  // [gate|up][chain][4]
    double c[2][2], d[2][2];
};

DEVI void acc_zero(Acc &r) {
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j) r.f[m][h][j] = 0.0f;
#pragma unroll
    for (int G = 0; G < 2; ++G) r.c[G][0] = r.c[G][1] = r.d[G][0] = r.d[G][1] = 0.0;
}

DEVI float accv(const Acc &r, int m, int j) { return r.f[m][0][j] + r.f[m][1][j]; }

DEVI void epi_router(const StepArgs &a, const Geo &g, StSmem &sm, const Item &t, Acc &r) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    double *part = a.ws.st_rt_part + (size_t)t.ks * 2 * g.E;
#pragma unroll
    for (int G = 0; G < 2; ++G) {
        const int row = 16 * t.a + 8 * G + gg;
        if (2 * q < g.B) part[(size_t)(2 * q) * g.E + row] = r.c[G][0] + r.d[G][0];
        if (2 * q + 1 < g.B) part[(size_t)(2 * q + 1) * g.E + row] = r.c[G][1] + r.d[G][1];
    }
    if (!warp_last_of(a.ws.ctl + p.c_rt_tk + t.a, (unsigned)p.s_rt)) return;
    for (int i = lane; i < 16 * g.B; i += 32) {
        const int b = i >> 4, row = 16 * t.a + (i & 15);
        const float lg = (float)sum_splits<double, 16>(a.ws.st_rt_part + (size_t)b * g.E + row, (size_t)2 * g.E, p.s_rt);
        a.ws.logits[(size_t)b * g.E + row] = lg;
        // top-k key: fp32 sigmoid score (computed in double) bits + 1; 0 marks "no expert"
        const float sc = router_score(lg);
        a.ws.st_key[(size_t)b * g.E + row] = (sc >= 0.0f ? __float_as_uint(sc) : 0u) + 1u;
    }
    if (a.flags & kFlagTestStall) return;  // the routing never completes: its waits must time out
    if (!warp_count_reaches(a.ws.ctl + CTL_RT_DONE, (unsigned)(g.E / 16))) return;
    unsigned long long *tr =
        a.ws.trace ? a.ws.trace + ((size_t)blockIdx.x * kTraceRowsPerSm + (threadIdx.x >> 5)) * kTraceStamps : nullptr;
    if (tr && lane == 0) tr[14] = global_ns();
    for (int b = 0; b < g.B; ++b) st_topk_token(a, g, sm, b);
    if (tr && lane == 0) tr[15] = global_ns();
    st_buckets(a, g, sm);
    if (tr && lane == 0) tr[11] = global_ns();
}

// 16-row split-K tile of B token columns (x columns are tokens: column 2q + j is token 2q + j)
DEVI void epi_dn(const StepArgs &a, const Geo &g, const Item &t, Acc &r) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    float *part = a.ws.st_dn_part + (size_t)t.ks * 2 * g.L;
    const int row = 16 * t.a + gg;
#pragma unroll
    for (int j = 0; j < 2; ++j)
        if (2 * q + j < g.B) {
            part[(size_t)(2 * q + j) * g.L + row] = accv(r, 0, j);
            part[(size_t)(2 * q + j) * g.L + row + 8] = accv(r, 0, 2 + j);
        }
    if (!warp_last_of(a.ws.ctl + p.c_dn_tk + t.a, (unsigned)p.s_dn)) return;
    for (int i = lane; i < 16 * g.B; i += 32) {
        const int b = i >> 4, rr = 16 * t.a + (i & 15);
        a.ws.h[(size_t)b * g.L + rr] = sum_splits(a.ws.st_dn_part + (size_t)b * g.L + rr, (size_t)2 * g.L, p.s_dn);
    }
}

// shared gate/up: x16 columns are tokens, scaled by 2^-shift[token]
DEVI void epi_sgu(const StepArgs &a, const Geo &g, const StSmem &sm, const Item &t, Acc &r) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    float *part = a.ws.st_sgu_part + (size_t)t.ks * 2 * 2 * g.Is;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int b = 2 * q + j;
        if (b < g.B) {
            const float sc = exp2i(sm.shift[b]);
            float *pg = part + (size_t)b * 2 * g.Is, *pu = pg + g.Is;
            const int row = 16 * t.a + gg;
            pg[row] = accv(r, 0, j) * sc;
            pg[row + 8] = accv(r, 0, 2 + j) * sc;
            pu[row] = accv(r, 1, j) * sc;
            pu[row + 8] = accv(r, 1, 2 + j) * sc;
        }
    }
    if (!warp_last_of(a.ws.ctl + p.c_sgu_tk + t.a, (unsigned)p.s_sgu)) return;
    const size_t st = (size_t)2 * 2 * g.Is;
    for (int i = lane; i < 16 * g.B; i += 32) {
        const int b = i >> 4, rr = 16 * t.a + (i & 15);
        const float *pb = a.ws.st_sgu_part + (size_t)b * 2 * g.Is;
        const float gs = sum_splits(pb + rr, st, p.s_sgu), us = sum_splits(pb + g.Is + rr, st, p.s_sgu);
        a.ws.sh_a[(size_t)b * g.Is + rr] = gs / (1.0f + expf(-gs)) * us;
    }
}

// expert gate/up: columns 2m, 2m+1 are entry m's hi and lo parts (h of its token)
DEVI void epi_egu(const StepArgs &a, const Geo &g, const StSmem &sm, const Item &t, Acc &r) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    const int cnt = sm.act_cnt[t.a], off = sm.act_off[t.a];
    const int nent = g.B * g.K;
    if (q < cnt) {
        const int ent = sm.ent[off + q];
        const float sc = exp2i(sm.shift[ent / g.K]);
        float *pg = a.ws.st_egu_part + ((size_t)t.ks * nent + ent) * 2 * g.I, *pu = pg + g.I;
        const int row = 16 * t.b + gg;
        pg[row] = (accv(r, 0, 0) + accv(r, 0, 1)) * sc;
        pg[row + 8] = (accv(r, 0, 2) + accv(r, 0, 3)) * sc;
        pu[row] = (accv(r, 1, 0) + accv(r, 1, 1)) * sc;
        pu[row + 8] = (accv(r, 1, 2) + accv(r, 1, 3)) * sc;
    }
    if (!warp_last_of(a.ws.ctl + p.c_egu_tk + t.a * (g.I / 16) + t.b, (unsigned)p.s_egu)) return;
    const size_t st = (size_t)nent * 2 * g.I;
    for (int i = lane; i < 16 * cnt; i += 32) {
        const int m = i >> 4, rr = 16 * t.b + (i & 15);
        const int ent = sm.ent[off + m];
        const float *pb = a.ws.st_egu_part + (size_t)ent * 2 * g.I;
        const float gs = sum_splits(pb + rr, st, p.s_egu), us = sum_splits(pb + g.I + rr, st, p.s_egu);
        a.ws.a[(size_t)ent * g.I + rr] = gs / (1.0f + expf(-gs)) * us;
    }
}

// shared down: columns 2q, 2q+1 are token q's hi and lo parts
DEVI void epi_sd(const StepArgs &a, const Geo &g, const StSmem &sm, const Item &t, Acc &r) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    float *part = a.ws.st_sd_part + (size_t)t.ks * 2 * g.H;
    if (q < g.B) {
        const float sc = exp2i(sm.shift[g.B + q]);
        const int row = 16 * t.a + gg;
        part[(size_t)q * g.H + row] = (accv(r, 0, 0) + accv(r, 0, 1)) * sc;
        part[(size_t)q * g.H + row + 8] = (accv(r, 0, 2) + accv(r, 0, 3)) * sc;
    }
    if (!warp_last_of(a.ws.ctl + p.c_sd_tk + t.a, (unsigned)p.s_sd)) return;
    for (int i = lane; i < 16 * g.B; i += 32) {
        const int b = i >> 4, rr = 16 * t.a + (i & 15);
        a.ws.sh[(size_t)b * g.H + rr] = sum_splits(a.ws.st_sd_part + (size_t)b * g.H + rr, (size_t)2 * g.H, p.s_sd);
    }
}

// expert down (full K): y rows of the slot's entries; the K-th entry of a (token, tile) combines
// the token's 16 latent rows in slot order
DEVI void epi_edown(const StepArgs &a, const Geo &g, const StSmem &sm, const Item &t, Acc &r) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    const int cnt = sm.act_cnt[t.a], off = sm.act_off[t.a];
    if (q < cnt) {
        const int ent = sm.ent[off + q];
        const float sc = exp2i(sm.shift[(t.a - sm.ed_j0) * g.B + q]);
        float *y = a.ws.y + (size_t)ent * g.L + 16 * t.b + gg;
        y[0] = (accv(r, 0, 0) + accv(r, 0, 1)) * sc;
        y[8] = (accv(r, 0, 2) + accv(r, 0, 3)) * sc;
    }
    __threadfence();
    __syncwarp();
    unsigned mine = 0;
    if (lane < cnt) {
        const int tok = sm.ent[off + lane] / g.K;
        mine = atomicAdd(a.ws.ctl + p.c_comb + tok * (g.L / 16) + t.b, 1u) == (unsigned)(g.K - 1) ? 1u : 0u;
    }
    unsigned todo = __ballot_sync(0xffffffffu, mine != 0);
    if (todo) __threadfence();
    while (todo) {
        const int m = __ffs(todo) - 1;
        todo &= todo - 1;
        const int tok = sm.ent[off + m] / g.K;
        // lane (row i, half h) adds the weighted slots of its parity in slot order
        const int l = 16 * t.b + (lane & 15), h = lane >> 4;
        float s = 0.0f;
        for (int r0 = h; r0 < g.K; r0 += 16) {
            float wv[8], yv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int rr = r0 + 2 * j;
                wv[j] = rr < g.K ? __ldcg(a.ws.wts + (size_t)tok * g.K + rr) : 0.0f;
                yv[j] = rr < g.K ? __ldcg(a.ws.y + ((size_t)tok * g.K + rr) * g.L + l) : 0.0f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) s += wv[j] * yv[j];
        }
        s += __shfl_xor_sync(0xffffffffu, s, 16);
        if (lane < 16) a.ws.ylat[(size_t)tok * g.L + l] = s;
    }
}

// W_up: ylat columns 2q, 2q+1 are token q's bf16 hi and lo parts; out = bf16(. + sh)
DEVI void epi_up(const StepArgs &a, const Geo &g, const Item &t, Acc &r) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    float *part = a.ws.st_up_part + (size_t)t.ks * 2 * g.H;
    const int row = 16 * t.a + gg;
    if (q < g.B) {
        part[(size_t)q * g.H + row] = accv(r, 0, 0) + accv(r, 0, 1);
        part[(size_t)q * g.H + row + 8] = accv(r, 0, 2) + accv(r, 0, 3);
    }
    if (!warp_last_of(a.ws.ctl + p.c_up_tk + t.a, (unsigned)p.s_up)) return;
    for (int i = lane; i < 16 * g.B; i += 32) {
        const int b = i >> 4, rr = 16 * t.a + (i & 15);
        const float s = sum_splits(a.ws.st_up_part + (size_t)b * g.H + rr, (size_t)2 * g.H, p.s_up);
        if (a.ws.up_tap) a.ws.up_tap[(size_t)b * g.H + rr] = s;
        const float shv = g.ns ? __ldcg(a.ws.sh + (size_t)b * g.H + rr) : 0.0f;
        a.out[(size_t)b * g.H + rr] = f32_to_bf16_rne(s + shv);
    }
}

// ---------------------------------------------------------------------------------------------
// activation staging of a launch (all threads of the CTA)

constexpr int kStageMax = 6;  // 16-byte units (4 fp32 or 8 bf16) each thread stages at most

// fp32 rows -> fp16 hi/lo column pairs: row r (n floats at rows[r]) becomes columns (2r, 2r+1) of the
// fp16 staging xs (swizzled units), scaled by 2^-shift[base + r] with the shift from the row's max
// |v|.  Every load is issued before the first use: one L2 round trip.
DEVI void cta_stage_f32_rows(uint16_t *xs, int pitch, const float *const *rows, int nrows, int n, StSmem &sm,
                             int base) {
    const int units = n / 4, total = nrows * units;
    if ((int)threadIdx.x < nrows) sm.amax[base + threadIdx.x] = 0u;
    float4 v[kStageMax];
#pragma unroll
    for (int j = 0; j < kStageMax; ++j) {
        const int u = threadIdx.x + j * blockDim.x;
        v[j] = u < total ? __ldcg(reinterpret_cast<const float4 *>(rows[u / units]) + u % units)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kStageMax; ++j) {
        const int u = threadIdx.x + j * blockDim.x;
        if (u < total) {
            const float m = fmaxf(fmaxf(fabsf(v[j].x), fabsf(v[j].y)), fmaxf(fabsf(v[j].z), fabsf(v[j].w)));
            atomicMax(sm.amax + base + u / units, __float_as_uint(m));
        }
    }
    __syncthreads();
    if ((int)threadIdx.x < nrows) sm.shift[base + threadIdx.x] = prescale_shift(__uint_as_float(sm.amax[base + threadIdx.x]));
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kStageMax; ++j) {
        const int u = threadIdx.x + j * blockDim.x;
        if (u < total) {
            const int r = u / units, k = 4 * (u % units);
            const float sc = exp2i(-sm.shift[base + r]);
            const float x0 = v[j].x * sc, x1 = v[j].y * sc, x2 = v[j].z * sc, x3 = v[j].w * sc;
            const uint32_t h01 = pack_f16x2(x0, x1), h23 = pack_f16x2(x2, x3);
            const uint32_t l01 = pack_f16x2(x0 - f16_lo(h01), x1 - f16_hi(h01));
            const uint32_t l23 = pack_f16x2(x2 - f16_lo(h23), x3 - f16_hi(h23));
            const int off = 8 * swz(k >> 3) + (k & 7);
            *reinterpret_cast<uint2 *>(xs + (size_t)(2 * r) * pitch + off) = make_uint2(h01, h23);
            *reinterpret_cast<uint2 *>(xs + (size_t)(2 * r + 1) * pitch + off) = make_uint2(l01, l23);
        }
    }
}

// x (B bf16 rows of H): bf16 columns t of xs, and (with a shared expert) fp16 columns t of x16
// scaled by 2^-shift[t] from the token's max |x|; one L2 round trip
DEVI void cta_stage_x(uint16_t *xs, uint16_t *x16, const StepArgs &a, const Geo &g, StSmem &sm) {
    const int units = g.H / 8, total = g.B * units;
    if ((int)threadIdx.x < g.B) sm.amax[threadIdx.x] = 0u;
    uint4 v[kStageMax];
#pragma unroll
    for (int j = 0; j < kStageMax; ++j) {
        const int u = threadIdx.x + j * blockDim.x;
        v[j] = u < total ? *reinterpret_cast<const uint4 *>(a.x + (size_t)u * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kStageMax; ++j) {
        const int u = threadIdx.x + j * blockDim.x;
        if (u < total) {
            const int t = u / units, k = 8 * (u % units);
            *reinterpret_cast<uint4 *>(xs + (size_t)t * bf16_pitch(g.H) + k) = v[j];
            if (g.ns) {
                const uint32_t w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
                float m = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w4[i])), fabsf(bf16_hi(w4[i]))));
                atomicMax(sm.amax + t, __float_as_uint(m));
            }
        }
    }
    if (!g.ns) return;
    __syncthreads();
    if ((int)threadIdx.x < g.B) sm.shift[threadIdx.x] = prescale_shift(__uint_as_float(sm.amax[threadIdx.x]));
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kStageMax; ++j) {
        const int u = threadIdx.x + j * blockDim.x;
        if (u < total) {
            const int t = u / units, k = 8 * (u % units);
            const float sc = exp2i(-sm.shift[t]);
            const uint32_t w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = pack_f16x2(bf16_lo(w4[i]) * sc, bf16_hi(w4[i]) * sc);
            *reinterpret_cast<uint4 *>(x16 + (size_t)t * f16_pitch(g.H) + 8 * swz(k >> 3)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// ylat (B fp32 rows of L) -> bf16 hi/lo columns (2t, 2t+1); one L2 round trip
DEVI void cta_stage_ylat(uint16_t *xs, const StepArgs &a, const Geo &g) {
    const int units = g.L / 4, total = g.B * units, pitch = bf16_pitch(g.L);
    float4 v[kStageMax];
#pragma unroll
    for (int j = 0; j < kStageMax; ++j) {
        const int u = threadIdx.x + j * blockDim.x;
        v[j] = u < total ? __ldcg(reinterpret_cast<const float4 *>(a.ws.ylat) + u) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < kStageMax; ++j) {
        const int u = threadIdx.x + j * blockDim.x;
        if (u < total) {
            const int t = u / units, k = 4 * (u % units);
            const uint32_t h01 = pack_bf16x2(v[j].x, v[j].y), h23 = pack_bf16x2(v[j].z, v[j].w);
            const uint32_t l01 = pack_bf16x2(v[j].x - bf16_lo(h01), v[j].y - bf16_hi(h01));
            const uint32_t l23 = pack_bf16x2(v[j].z - bf16_lo(h23), v[j].w - bf16_hi(h23));
            *reinterpret_cast<uint2 *>(xs + (size_t)(2 * t) * pitch + k) = make_uint2(h01, h23);
            *reinterpret_cast<uint2 *>(xs + (size_t)(2 * t + 1) * pitch + k) = make_uint2(l01, l23);
        }
    }
}

}  // namespace

// ---------------------------------------------------------------------------------------------
// the kernel

// Launch `ph` (0..3) of a step; the last one clears the control block for the next step.
__global__ void __launch_bounds__(kStWarps * 32, 1) k_stream(StepArgs a, int ph) {
    extern __shared__ __align__(128) unsigned char st_dyn[];
    __shared__ StSmem sm;
    const Geo g = geo(a);
    const StreamPlan &p = a.p.st;
    unsigned *ctl = a.ws.ctl;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *ring = st_dyn + (size_t)warp * kStStages * kSlotBytes;
    uint16_t *xs = reinterpret_cast<uint16_t *>(st_dyn + kRingBytes);  // the launch's activations
    const int q_lo = ph == 0 ? SQ_RT : ph == 1 ? SQ_SD : ph == 2 ? SQ_EDOWN : SQ_UP;
    const int q_hi = ph == 0 ? SQ_SD : ph == 1 ? SQ_EDOWN : ph == 2 ? SQ_UP : SQ_N;
    unsigned long long *trace =
        a.ws.trace ? a.ws.trace + ((size_t)blockIdx.x * kTraceRowsPerSm + warp) * kTraceStamps : nullptr;
    unsigned long long *launch_row =
        a.ws.trace ? a.ws.trace + ((size_t)blockIdx.x * kTraceRowsPerSm + 12) * kTraceStamps : nullptr;
    if (trace && lane < kTraceStamps && (ph == 0 || (lane != 11 && lane != 14 && lane != 15))) trace[lane] = 0ull;
    if (trace && lane == 0) trace[0] = global_ns();
    if (launch_row && threadIdx.x == 0) launch_row[2 * ph] = global_ns();
    if (a.ws.trace && ph == 0 && threadIdx.x < kTraceStamps)
        a.ws.trace[((size_t)blockIdx.x * kTraceRowsPerSm + 13) * kTraceStamps + threadIdx.x] = 0ull;

    if (lane < kStStages) mbar_init(&sm.bar[warp][lane], 1u);
    if (threadIdx.x == 0) {
        sm.route_state = 0;
        sm.n_active = 0;
        sm.ed_j0 = 0;
    }
    cta_take_init(sm.claim);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();

    // producer state (warp-uniform)
    int pq = q_lo, pit = -1, pc = 0, pn = 0;
    Item pitem = {0, 0, 0};
    IssuePlan pplan;
    int n_iss = 0, n_con = 0;
    bool alive = true;
    int n_active = -1;

    auto claim_next = [&](int q, int n) {
        int v = -1;
        if (lane == 0) v = cta_take(sm.claim, q, n);
        return __shfl_sync(0xffffffffu, v, 0);
    };
    auto next_item = [&](bool routed) -> bool {
        while (pq < q_hi) {
            if ((pq == SQ_EGU || pq == SQ_EDOWN) && n_active < 0) {
                if (!routed) return false;  // before the launch dependency resolves: no routing yet
                if (!ensure_routing(a, sm)) {
                    alive = false;
                    return false;
                }
                n_active = sm.n_active;
            }
            const int n = queue_len(a, g, pq, n_active < 0 ? 0 : n_active);
            const int it = n > 0 ? claim_next(pq, n) : -1;
            if (it >= 0) {
                pit = it;
                pitem = decode_item(a, g, pq, it, &pn);
                pc = 0;
                pplan = make_plan(a, g, sm, pq, pitem);
                return true;
            }
            ++pq;
        }
        return false;
    };
    auto top_up = [&](bool routed) {
        while (alive && n_iss - n_con < kStStages) {
            if (pit < 0 || pc == pn) {
                pit = -1;
                if (!next_item(routed)) return;
            }
            const int s = n_iss % kStStages;
            issue_stage(pplan, ring + (size_t)s * kSlotBytes, &sm.bar[warp][s], pc);
            if (lane == 0) {
                sm.meta[warp][s].q = pq;
                sm.meta[warp][s].item = pit;
                sm.meta[warp][s].c = pc;
                sm.meta[warp][s].n = pn;
            }
            __syncwarp();
            ++pc;
            ++n_iss;
        }
    };

    // The next launch may be scheduled onto SMs as this one's CTAs leave (its weight copies need
    // nothing of ours); it reads our results only after its griddepcontrol.wait.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // start the copies that need nothing of the previous launches (weights of the queues before
    // the routed ones), then wait for the previous launch, stage its results while they fly
    top_up(false);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (ph == 0) {
        // x as bf16 (router, W_dn) and as fp16 * 2^-shift[token] (shared gate/up)
        cta_stage_x(xs, xs + (size_t)g.B * bf16_pitch(g.H), a, g, sm);
    } else if (ph == 1) {
        // h (all tokens) and sh_a as fp16 hi/lo columns; shift[t] for h, shift[B + t] for sh_a
        const float *rows[2 * kStMaxBatch];
        for (int t = 0; t < g.B; ++t) {
            rows[t] = a.ws.h + (size_t)t * g.L;
            rows[g.B + t] = a.ws.sh_a + (size_t)t * g.Is;
        }
        cta_stage_f32_rows(xs, f16_pitch(g.L), rows, g.B, g.L, sm, 0);
        if (g.ns) cta_stage_f32_rows(xs + (size_t)2 * g.B * f16_pitch(g.L), f16_pitch(g.Is), rows + g.B, g.B, g.Is, sm, g.B);
    } else if (ph == 2) {
        // a of the entries of the (at most two) experts of this CTA's range, fp16 hi/lo; expert
        // j0 + e, entry m: columns 2(e B + m) + part, shift[e B + m]
        __shared__ int s_ok, s_rows[2 * kMaxEdownExperts * kStMaxBatch], s_nr;
        if (warp == 0) {
            const bool ok = ensure_routing(a, sm);
            if (lane == 0) s_ok = ok ? 1 : 0;
        }
        __syncthreads();
        alive = alive && s_ok;
        const int n = sm.n_active * (g.L / 16);
        const long long G = gridDim.x, cc = blockIdx.x;
        const int lo = (int)((long long)n * cc / G), hi = (int)((long long)n * (cc + 1) / G);
        if (s_ok && hi > lo) {
            const int j0 = lo / (g.L / 16), j1 = (hi - 1) / (g.L / 16);
            if (threadIdx.x == 0) {
                int nr = 0;
                for (int e = 0; e <= j1 - j0 && e < kMaxEdownExperts; ++e)
                    for (int m = 0; m < g.B; ++m) {
                        const int cnt = sm.act_cnt[j0 + e];
                        s_rows[e * g.B + m] = sm.ent[sm.act_off[j0 + e] + (m < cnt ? m : 0)];
                        nr = e * g.B + m + 1;
                    }
                s_nr = nr;
                sm.ed_j0 = j0;
            }
            __syncthreads();
            const float *rows[2 * kMaxEdownExperts * kStMaxBatch];
            for (int i = 0; i < s_nr; ++i) rows[i] = a.ws.a + (size_t)s_rows[i] * g.I;
            cta_stage_f32_rows(xs, f16_pitch(g.I), rows, s_nr, g.I, sm, 0);
        }
    } else {
        // ylat as bf16 hi/lo columns (2t, 2t+1)
        cta_stage_ylat(xs, a, g);
    }
    __syncthreads();
    if (trace && lane == 0) trace[1] = global_ns();
    const unsigned long long t_staged = a.ws.trace ? global_ns() : 0ull;
    unsigned long long *spread =
        a.ws.trace ? a.ws.trace + ((size_t)blockIdx.x * kTraceRowsPerSm + 14) * kTraceStamps + 4 * ph : nullptr;
    if (spread && threadIdx.x == 0) {
        spread[0] = t_staged - launch_row[2 * ph];  // launch start to activations staged
        spread[1] = 0ull;                           // latest warp finish after staging
        spread[2] = ~0ull;                          // earliest warp finish after staging
    }
    __syncthreads();

    Acc acc;
    acc_zero(acc);
    Item cit = {0, 0, 0};
    long long cyc_issue = 0, cyc_data = 0, cyc_compute = 0, cyc_epi = 0;
    for (;;) {
        const long long ti0 = trace ? clock64() : 0;
        top_up(true);
        const long long ti1 = trace ? clock64() : 0;
        cyc_issue += ti1 - ti0;
        if (!alive || n_con == n_iss) break;  // aborted, or every queue of this launch is drained
        const int s = n_con % kStStages;
        unsigned char *slot = ring + (size_t)s * kSlotBytes;
        if (!slot_wait(a, &sm.bar[warp][s], (unsigned)((n_con / kStStages) & 1))) {
            alive = false;
            break;
        }
        const long long td = trace ? clock64() : 0;
        cyc_data += td - ti1;
        const SlotMeta m = sm.meta[warp][s];
        if (m.c == 0) {
            int ns_;
            cit = decode_item(a, g, m.q, m.item, &ns_);
            acc_zero(acc);
        }
        const Item it = cit;
        const int gcol = lane >> 2;
        switch (m.q) {
            case SQ_RT:
                mma_stage_router(slot, xs, bf16_pitch(g.H), it.ks * p.kr_rt + 128 * m.c, g.B, acc.c, acc.d);
                break;
            case SQ_DN:
                mma_stage_bf16(slot, xs, bf16_pitch(g.H), it.ks * p.kr_dn + 128 * m.c, gcol < g.B ? gcol : -1,
                               acc.f[0][0], acc.f[0][1]);
                break;
            case SQ_UP:
                mma_stage_bf16(slot, xs, bf16_pitch(g.L), it.ks * p.kr_up + 128 * m.c, gcol < 2 * g.B ? gcol : -1,
                               acc.f[0][0], acc.f[0][1]);
                break;
            case SQ_SGU: {
                const uint16_t *x16 = xs + (size_t)g.B * bf16_pitch(g.H);
                const int kofs = it.ks * p.kr_sgu + 512 * (m.c >> 1), col = gcol < g.B ? gcol : -1;
                if (m.c & 1) mma_stage_fp4(slot, x16, f16_pitch(g.H), kofs, col, acc.f[1][0], acc.f[1][1]);
                else mma_stage_fp4(slot, x16, f16_pitch(g.H), kofs, col, acc.f[0][0], acc.f[0][1]);
                break;
            }
            case SQ_EGU: {
                // MMA column gcol: entry gcol/2 of the slot, hi (even) or lo (odd) part of its token's h
                const int cnt = sm.act_cnt[it.a];
                const int col = (gcol >> 1) < cnt ? 2 * (sm.ent[sm.act_off[it.a] + (gcol >> 1)] / g.K) + (gcol & 1) : -1;
                const int kofs = it.ks * p.kr_egu + 512 * (m.c >> 1);
                if (m.c & 1) mma_stage_fp4(slot, xs, f16_pitch(g.L), kofs, col, acc.f[1][0], acc.f[1][1]);
                else mma_stage_fp4(slot, xs, f16_pitch(g.L), kofs, col, acc.f[0][0], acc.f[0][1]);
                break;
            }
            case SQ_SD: {
                const uint16_t *s16 = xs + (size_t)2 * g.B * f16_pitch(g.L);
                mma_stage_fp4(slot, s16, f16_pitch(g.Is), it.ks * p.kr_sd + 512 * m.c, gcol < 2 * g.B ? gcol : -1,
                              acc.f[0][0], acc.f[0][1]);
                break;
            }
            case SQ_EDOWN: {
                const int cnt = sm.act_cnt[it.a];
                const int col = gcol < 2 * cnt ? 2 * (it.a - sm.ed_j0) * g.B + gcol : -1;
                mma_stage_fp4(slot, xs, f16_pitch(g.I), 512 * m.c, col, acc.f[0][0], acc.f[0][1]);
                break;
            }
        }
        __syncwarp();  // every lane is done with the slot before it is refilled
        const long long tc1 = trace ? clock64() : 0;
        cyc_compute += tc1 - td;
        if (m.c == m.n - 1) {
            switch (m.q) {
                case SQ_RT: epi_router(a, g, sm, it, acc); break;
                case SQ_DN: epi_dn(a, g, it, acc); break;
                case SQ_UP: epi_up(a, g, it, acc); break;
                case SQ_SGU: epi_sgu(a, g, sm, it, acc); break;
                case SQ_EGU: epi_egu(a, g, sm, it, acc); break;
                case SQ_SD: epi_sd(a, g, sm, it, acc); break;
                case SQ_EDOWN: epi_edown(a, g, sm, it, acc); break;
            }
            __syncwarp();
            if (trace) cyc_epi += clock64() - tc1;
        }
        ++n_con;
    }
    // an aborted warp still owns copies in flight: let them land before the CTA leaves
    for (; n_con < n_iss; ++n_con)
        if (!slot_wait(a, &sm.bar[warp][n_con % kStStages], (unsigned)((n_con / kStStages) & 1))) break;
    if (spread && lane == 0) {
        const unsigned long long dt = global_ns() - t_staged;
        atomicMax(spread + 1, dt);
        atomicMin(spread + 2, dt);
    }
    if (trace && lane == 0) {
        trace[2] = cyc_issue;
        trace[3] = cyc_data;
        trace[5] = cyc_compute;
        trace[6] = cyc_epi;
        trace[7] = n_iss;
        trace[9] = global_ns();
        // row 13 of the SM: this launch's cycle sums over the CTA's warps (issue, data, compute,
        // epilogue), 4 stamps per launch
        unsigned long long *sums = a.ws.trace + ((size_t)blockIdx.x * kTraceRowsPerSm + 13) * kTraceStamps + 4 * ph;
        atomicAdd(sums + 0, (unsigned long long)cyc_issue);
        atomicAdd(sums + 1, (unsigned long long)cyc_data);
        atomicAdd(sums + 2, (unsigned long long)cyc_compute);
        atomicAdd(sums + 3, (unsigned long long)cyc_epi);
    }

    // leave; the last CTA out of the last launch clears the control block for the next step
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        sm.exit_last = (atomicAdd(ctl + CTL_QHEAD + ph, 1u) == gridDim.x - 1) ? 1 : 0;  // per-launch exit count
    }
    __syncthreads();
    if (trace && lane == 0) trace[10] = global_ns();
    if (launch_row && threadIdx.x == 0) launch_row[2 * ph + 1] = global_ns();
    if (sm.exit_last) {
        __threadfence();
        if (ph == kStreamLaunches - 1) {
            for (int i = threadIdx.x; i < CTL_FIXED; i += blockDim.x) ctl[i] = 0u;
            for (int i = p.c_rt_tk + threadIdx.x; i < p.words; i += blockDim.x) ctl[i] = 0u;
        }
    }
}

// ---------------------------------------------------------------------------------------------
// host side

// dynamic shared memory: the rings, then the largest activation staging of the four launches
static size_t stream_smem(const Dims &d, int B) {
    size_t act = (size_t)B * bf16_pitch(d.H) * 2 + (d.n_shared ? (size_t)B * f16_pitch(d.H) * 2 : 0);
    act = std::max(act, (size_t)2 * B * f16_pitch(d.L) * 2 + (d.n_shared ? (size_t)2 * B * f16_pitch(d.Is) * 2 : 0));
    act = std::max(act, (size_t)2 * kMaxEdownExperts * B * f16_pitch(d.I) * 2);
    act = std::max(act, (size_t)2 * B * bf16_pitch(d.L) * 2);
    return (size_t)kRingBytes + act;
}

constexpr size_t kStSmemLimit = 216 * 1024;  // dynamic; the static part is a few KB

bool stream_supports(const Dims &d, int B) {
    if (B < 1 || B > kStMaxBatch || d.k > 32 || d.k > d.E || d.E > 1024 || B * d.k > kMaxActive) return false;
    // whole MXFP4 stages (512 k, 16-byte scale rows) and bf16 stages (128 k); 16-row tiles
    if (d.H % 512 || d.L % 512 || d.I % 512 || (d.n_shared && d.Is % 512) || d.E % 16) return false;
    // a CTA's expert-down range (n_active * L/16 items over the grid) spans at most two experts
    // as long as there are no more active experts than CTAs (>= 1 per SM, and n_active <= 64)
    // batched staging: at most kStageMax 16-byte units per thread in every launch
    const int cap = kStageMax * kStWarps * 32;
    if (B * d.H / 8 > cap || B * d.L / 4 > cap || (d.n_shared && B * d.Is / 4 > cap) ||
        kMaxEdownExperts * B * d.I / 4 > cap)
        return false;
    return stream_smem(d, B) <= kStSmemLimit;
}

// largest multiple of `unit` that is <= pref and divides K (K is a multiple of unit)
static int pick_range(int K, int pref, int unit) {
    for (int r = pref - pref % unit; r >= unit; r -= unit)
        if (K % r == 0) return r;
    return unit;
}

void stream_plan(const Dims &d, StreamPlan &sp, int ctl_base) {
    const int Is = d.n_shared ? d.Is : 512;
    sp.kr_rt = pick_range(d.H, 512, 128);
    sp.kr_dn = pick_range(d.H, 512, 128);
    sp.kr_sgu = pick_range(d.H, 512, 512);
    sp.kr_egu = pick_range(d.L, 512, 512);
    sp.kr_sd = pick_range(Is, 512, 512);
    sp.kr_up = pick_range(d.L, 256, 128);
    sp.s_rt = d.H / sp.kr_rt;
    sp.s_dn = d.H / sp.kr_dn;
    sp.s_sgu = d.H / sp.kr_sgu;
    sp.s_egu = d.L / sp.kr_egu;
    sp.s_sd = Is / sp.kr_sd;
    sp.s_up = d.L / sp.kr_up;
    int c = ctl_base;
    sp.c_rt_tk = c; c += (d.E + 15) / 16;
    sp.c_dn_tk = c; c += d.L / 16;
    sp.c_sgu_tk = c; c += Is / 16;
    sp.c_egu_tk = c; c += d.E * (d.I / 16);
    sp.c_sd_tk = c; c += d.H / 16;
    sp.c_comb = c; c += kStMaxBatch * (d.L / 16);
    sp.c_up_tk = c; c += d.H / 16;
    sp.words = c;
}

// The step as four launches, each of which only runs work whose inputs the previous launches
// finished (see the top of this file).
cudaError_t launch_stream(const StepArgs &a, cudaStream_t s, int n_sm) {
    cudaError_t e = cudaSuccess;
    const size_t smem = stream_smem(a.d, a.B);
    for (int ph = 0; ph < kStreamLaunches && e == cudaSuccess; ++ph) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(n_sm);
        cfg.blockDim = dim3(kStWarps * 32);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        // launches 2..4 may start as SMs free up (they wait for the previous launch's results on
        // the device); the first one waits for the previous step like any stream-ordered launch
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = ph > 0 ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, k_stream, a, ph);
    }
    return e;
}

cudaError_t init_stream_attributes() {
    return cudaFuncSetAttribute(k_stream, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStSmemLimit);
}

}  // namespace moedec
