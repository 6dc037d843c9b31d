// moedec_stream.cu -- the decode layer step for 1-2 tokens as one persistent kernel of streaming
// warps.
//
// Batch 1-2 is the pages' small-matrix range of the Kimi K3 decode path ("快是可以生成的，可信
// 只能证明（vLLM 重写 Kimi K3 解码路径…）", section 他们换掉了什么), and there the step is pure
// weight streaming: 148 MB per full-size layer step at batch 1.  A loaded HBM access on B200 takes
// about 2 us, so each SM must keep ~100 KB of weights in flight at all times, across work items
// and across the step's dependency points (routing, h, a, ylat).  The same page lists the
// techniques as ways of removing waiting; this kernel is built around exactly that.
//
// Each warp owns a ring of 3 shared-memory slots and streams its own sequence of work items
// through it with cp.async: a slot holds one stage of one item, 4 KB of weights (16 bf16 rows or
// 64 MXFP4 rows, 128 k each) plus the matching 128 k of activation columns.  The warp issues the
// next stages (of the next items, claimed one ahead) before it computes the current one, so its
// loads never drain between items.  Weights never depend on anything but routing; when a stage's
// activation block is not final yet, its weights are loaded anyway and the activation part is
// copied when the stage is consumed.
//
// Work queues, in order (every warp drains them in this order; an item only waits on items of
// earlier queues, so every wait ends):
//   x16     fp16 copy of x per 512-k block and token (for the shared gate/up MMAs)
//   router  16 rows x K range, fp64 MMAs; the warp that completes the last row group ranks the
//           experts (top-k per token) and builds the expert buckets
//   W_dn    16 rows x K range; a completed block of h is converted to fp16 hi/lo once
//   shared  gate/up, 64 rows x K range; a completed block of sh_a is converted once
//   expert  gate/up, 64 rows of one active expert x K range; a completed expert's a is converted
//   shared  down, 64 rows x K range
//   expert  down, 64 rows of one active expert; completing a token's 64 latent rows combines them
//   W_up    16 rows x K range (K-range major, so it starts on the first final block of ylat)
// Activations crossing CTAs live in global memory in MMA-ready form: fp16 hi/lo columns scaled by
// a power of two per (token, block) for the MXFP4 products, bf16 hi/lo columns for W_up.
#include <algorithm>

#include "moedec_items.cuh"

namespace moedec {

namespace {

constexpr int kStWarps = 12;
constexpr int kStStages = 3;
constexpr int kStMaxBatch = 2;
// slot layout: weights | scales | activation columns | exponents
constexpr int kSlotSc = 4096, kSlotAct = 4352, kSlotExp = 5632, kSlotBytes = 5648;
constexpr int kPitchF16 = 272;  // fp16 activation column (128 k, 16-unit swizzle) in a slot
constexpr int kPitchB16 = 320;  // bf16 activation column in a slot
constexpr int kStDynSmem = kStWarps * kStStages * kSlotBytes;
constexpr int kMaxActive = 64;  // active experts at <= 2 tokens x <= 32 slots

enum StQueue { SQ_X16 = 0, SQ_RT, SQ_DN, SQ_SGU, SQ_EGU, SQ_SD, SQ_EDOWN, SQ_UP, SQ_N };

// dependency ids of a stage's activation block (bit index in the CTA's ready bitmap)
constexpr int kDepNone = -1, kDepX16 = 0, kDepH16 = 64, kDepSh16 = 80, kDepYl = 96, kDepA16 = 128;
constexpr int kDepBits = 192;

struct SlotMeta {
    int q, item, c, n;  // queue, item, stage within the item, stages of the item
    int act;            // 1 once the activation part of the slot is copied
};

struct StSmem {
    SlotMeta meta[kStWarps][kStStages];
    unsigned dep_ready[kDepBits / 32];
    int route_state;  // 0 not loaded, 1 loading, 2 loaded
    int n_active;
    int act_e[kMaxActive], act_cnt[kMaxActive], act_off[kMaxActive], ent[kMaxActive];
    // top-k scratch of the warp that ranks the experts
    int tk_idx[kMaxActive], srt_e[kMaxActive], srt_i[kMaxActive], first_pos[kMaxActive + 1];
    int exit_last;
    CtaTake claim;
};

// ---------------------------------------------------------------------------------------------
// async copies

DEVI uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

DEVI void cp16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
DEVI void cp16_zfill(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
DEVI void cp4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
DEVI void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most n of this thread's copy groups are pending
DEVI void cp_wait(int n) {
    if (n <= 0)
        asm volatile("cp.async.wait_group 0;" ::: "memory");
    else if (n == 1)
        asm volatile("cp.async.wait_group 1;" ::: "memory");
    else
        asm volatile("cp.async.wait_group 2;" ::: "memory");
}

// unit u (16 bytes) of an fp16 activation column: within each 16-unit column, units of lane
// quads 2 and 3 are shifted by two, so that a phase's four lane quads hit distinct bank groups
DEVI int swz2(int u) { return u ^ (((u >> 3) & 1) << 1); }

// ---------------------------------------------------------------------------------------------
// the step's geometry

struct Geo {
    int H, L, E, K, I, Is, B, ns;  // ns: 1 with a shared expert
    int rt_groups, dn_tiles, sgu_tiles, egu_tiles, sd_tiles, ed_tiles, up_tiles;
};

DEVI Geo geo(const StepArgs &a) {
    Geo g;
    g.H = a.d.H; g.L = a.d.L; g.E = a.d.E; g.K = a.d.k; g.I = a.d.I; g.Is = a.d.Is; g.B = a.B;
    g.ns = a.d.n_shared ? 1 : 0;
    g.rt_groups = (g.E + 15) / 16;
    g.dn_tiles = g.L / 16;
    g.sgu_tiles = g.Is / 64;
    g.egu_tiles = g.I / 64;
    g.sd_tiles = g.H / 64;
    g.ed_tiles = g.L / 64;
    g.up_tiles = g.H / 16;
    return g;
}

DEVI int queue_len(const StepArgs &a, const Geo &g, int q, int n_active) {
    const StreamPlan &p = a.p.st;
    switch (q) {
        case SQ_X16: return g.ns ? g.B * p.s_sgu : 0;
        case SQ_RT: return g.rt_groups * p.s_rt;
        case SQ_DN: return g.dn_tiles * p.s_dn;
        case SQ_SGU: return g.ns ? g.sgu_tiles * p.s_sgu : 0;
        case SQ_EGU: return n_active * g.egu_tiles * p.s_egu;
        case SQ_SD: return g.ns ? g.sd_tiles * p.s_sd : 0;
        case SQ_EDOWN: return n_active * g.ed_tiles;
        case SQ_UP: return g.up_tiles * p.s_up;
    }
    return 0;
}

DEVI int item_stages(const StepArgs &a, const Geo &g, int q) {
    const StreamPlan &p = a.p.st;
    switch (q) {
        case SQ_RT: return p.kr_rt / 128;
        case SQ_DN: return p.kr_dn / 128;
        case SQ_SGU: return 2 * (p.kr_sgu / 128);
        case SQ_EGU: return 2 * (p.kr_egu / 128);
        case SQ_SD: return p.kr_sd / 128;
        case SQ_EDOWN: return g.I / 128;
        case SQ_UP: return p.kr_up / 128;
    }
    return 0;
}

// ---------------------------------------------------------------------------------------------
// stage issue: weights (always) and the activation columns (when their block is final)

// Activation part of a stage: column c of the slot is 128 k of global row src(c) starting at k0.
// ASYNC: cp.async into the stage's copy group; else synchronous L2 loads and shared stores.
template <bool ASYNC, class Src>
DEVI void copy_act_cols(unsigned char *slot, int ncols, int pitch, bool swizzle, Src src) {
    const int lane = threadIdx.x & 31;
    for (int p = lane; p < ncols * 16; p += 32) {
        const int c = p >> 4, u = p & 15;
        unsigned char *dst = slot + kSlotAct + c * pitch + 16 * (swizzle ? swz2(u) : u);
        const uint16_t *s = src(c) + 8 * u;
        if (ASYNC)
            cp16(smem_addr(dst), s);
        else
            *reinterpret_cast<uint4 *>(dst) = __ldcg(reinterpret_cast<const uint4 *>(s));
    }
}

template <bool ASYNC>
DEVI void copy_exp(unsigned char *slot, int idx, const int *src) {
    if (ASYNC)
        cp4(smem_addr(slot + kSlotExp + 4 * idx), src);
    else
        *reinterpret_cast<int *>(slot + kSlotExp + 4 * idx) = __ldcg(src);
}

struct Item {
    int a, b, ks;  // kind-specific: (group|tile|slot j, tile, k split)
};

DEVI Item decode_item(const StepArgs &a, const Geo &g, int q, int it) {
    const StreamPlan &p = a.p.st;
    Item r = {0, 0, 0};
    switch (q) {
        case SQ_X16: r.a = it / p.s_sgu; r.ks = it % p.s_sgu; break;                 // token, block
        case SQ_RT: r.a = it / p.s_rt; r.ks = it % p.s_rt; break;                    // group
        case SQ_DN: r.a = it / p.s_dn; r.ks = it % p.s_dn; break;                    // tile
        case SQ_SGU: r.a = it / p.s_sgu; r.ks = it % p.s_sgu; break;                 // tile
        case SQ_EGU: {
            const int jt = it / p.s_egu;
            r.ks = it % p.s_egu; r.a = jt / g.egu_tiles; r.b = jt % g.egu_tiles;     // slot j, tile
            break;
        }
        case SQ_SD: r.a = it / p.s_sd; r.ks = it % p.s_sd; break;                    // tile
        case SQ_EDOWN: r.a = it / g.ed_tiles; r.b = it % g.ed_tiles; break;          // slot j, tile
        case SQ_UP: r.ks = it / g.up_tiles; r.a = it % g.up_tiles; break;            // tile, K-range major
    }
    return r;
}

// dependency of the activation block of an item
DEVI int item_dep(int q, const Item &t) {
    switch (q) {
        case SQ_SGU: return kDepX16 + t.ks;
        case SQ_EGU: return kDepH16 + t.ks;
        case SQ_SD: return kDepSh16 + t.ks;
        case SQ_EDOWN: return kDepA16 + t.a;
        case SQ_UP: return kDepYl + t.ks;
    }
    return kDepNone;
}

DEVI bool dep_known(const StSmem &sm, int dep) {
    return dep < 0 || ((*(volatile const unsigned *)&sm.dep_ready[dep >> 5]) >> (dep & 31) & 1u);
}

// global flag and target that make a dependency final
DEVI void dep_flag(const StepArgs &a, const Geo &g, int dep, const unsigned **flag, unsigned *target) {
    const StreamPlan &p = a.p.st;
    const unsigned *ctl = a.ws.ctl;
    if (dep >= kDepA16) { *flag = ctl + p.c_a16 + (dep - kDepA16); *target = 1u; }
    else if (dep >= kDepYl) { *flag = ctl + p.c_yl + (dep - kDepYl); *target = (unsigned)(g.B * (p.kr_up / 64)); }
    else if (dep >= kDepSh16) { *flag = ctl + p.c_sh16 + (dep - kDepSh16); *target = 1u; }
    else if (dep >= kDepH16) { *flag = ctl + p.c_h16 + (dep - kDepH16); *target = 1u; }
    else { *flag = ctl + p.c_x16 + dep; *target = (unsigned)g.B; }
}

// activation columns (and exponents) of stage c of item t of queue q
template <bool ASYNC>
DEVI void copy_act(const StepArgs &a, const Geo &g, const StSmem &sm, unsigned char *slot, int q, const Item &t,
                   int c) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31;
    switch (q) {
        case SQ_RT: {
            const int k0 = t.ks * p.kr_rt + 128 * c;
            copy_act_cols<ASYNC>(slot, g.B, kPitchB16, false, [&](int col) { return a.x + (size_t)col * g.H + k0; });
            break;
        }
        case SQ_DN: {
            const int k0 = t.ks * p.kr_dn + 128 * c;
            copy_act_cols<ASYNC>(slot, g.B, kPitchB16, false, [&](int col) { return a.x + (size_t)col * g.H + k0; });
            break;
        }
        case SQ_UP: {
            const int k0 = t.ks * p.kr_up + 128 * c;
            copy_act_cols<ASYNC>(slot, 2 * g.B, kPitchB16, false,
                                 [&](int col) { return (const uint16_t *)a.ws.ylat16 + (size_t)col * g.L + k0; });
            break;
        }
        case SQ_SGU: {
            const int k0 = t.ks * p.kr_sgu + 128 * (c >> 1);
            copy_act_cols<ASYNC>(slot, g.B, kPitchF16, true,
                                 [&](int col) { return (const uint16_t *)a.ws.x16 + (size_t)col * g.H + k0; });
            if (lane < g.B) copy_exp<ASYNC>(slot, lane, a.ws.x16e + t.ks * 4 + lane);
            break;
        }
        case SQ_EGU: {
            const int k0 = t.ks * p.kr_egu + 128 * (c >> 1);
            const int cnt = sm.act_cnt[t.a], off = sm.act_off[t.a];
            copy_act_cols<ASYNC>(slot, 2 * cnt, kPitchF16, true, [&](int col) {
                const int tok = sm.ent[off + (col >> 1)] / g.K;
                return (const uint16_t *)a.ws.h16 + (size_t)(2 * tok + (col & 1)) * g.L + k0;
            });
            if (lane < cnt) copy_exp<ASYNC>(slot, lane, a.ws.h16e + t.ks * 4 + sm.ent[off + lane] / g.K);
            break;
        }
        case SQ_SD: {
            const int k0 = t.ks * p.kr_sd + 128 * c;
            copy_act_cols<ASYNC>(slot, 2 * g.B, kPitchF16, true,
                                 [&](int col) { return (const uint16_t *)a.ws.sh16 + (size_t)col * g.Is + k0; });
            if (lane < g.B) copy_exp<ASYNC>(slot, lane, a.ws.sh16e + t.ks * 4 + lane);
            break;
        }
        case SQ_EDOWN: {
            const int k0 = 128 * c;
            const int cnt = sm.act_cnt[t.a], off = sm.act_off[t.a];
            copy_act_cols<ASYNC>(slot, 2 * cnt, kPitchF16, true, [&](int col) {
                const int ent = sm.ent[off + (col >> 1)];
                return (const uint16_t *)a.ws.a16 + (size_t)(2 * ent + (col & 1)) * g.I + k0;
            });
            if (lane < cnt) copy_exp<ASYNC>(slot, lane, a.ws.a16e + t.a * 4 + lane);
            break;
        }
    }
}

// Per-lane copy plan of the item being issued, computed once per item: every stage's copies are
// then the plan's pointers plus a per-stage offset (a few instructions per 16-byte copy).
struct IssuePlan {
    const unsigned char *w;       // lane's weight piece 0, stage 0, matrix 0
    const unsigned char *s;       // MXFP4: lane's scale row, stage 0, matrix 0; bf16: a valid address
    long long dw, ds;             // MXFP4 pairs: byte offset of the up matrix from the gate matrix
    int wpi, spi;                 // bytes between the lane's weight pieces / its two scale rows
    unsigned valid;               // bf16: bit i set when piece i's row exists
    uint32_t dst;                 // lane's piece-0 offset in a slot
    const unsigned char *a0, *a1; // lane's activation pieces at stage 0 (null: none)
    uint32_t adst0, adst1;
    const int *ex;                // lane's exponent source (null: none)
    bool fp4, pair;
};

// activation column c of item t (its source row at the item's first k), for c < ncols
DEVI const uint16_t *act_col(const StepArgs &a, const Geo &g, const StSmem &sm, int q, const Item &t, int c) {
    const StreamPlan &p = a.p.st;
    switch (q) {
        case SQ_RT: return a.x + (size_t)c * g.H + t.ks * p.kr_rt;
        case SQ_DN: return a.x + (size_t)c * g.H + t.ks * p.kr_dn;
        case SQ_UP: return a.ws.ylat16 + (size_t)c * g.L + t.ks * p.kr_up;
        case SQ_SGU: return a.ws.x16 + (size_t)c * g.H + t.ks * p.kr_sgu;
        case SQ_EGU:
            return a.ws.h16 + (size_t)(2 * (sm.ent[sm.act_off[t.a] + (c >> 1)] / g.K) + (c & 1)) * g.L + t.ks * p.kr_egu;
        case SQ_SD: return a.ws.sh16 + (size_t)c * g.Is + t.ks * p.kr_sd;
        default: return a.ws.a16 + (size_t)(2 * sm.ent[sm.act_off[t.a] + (c >> 1)] + (c & 1)) * g.I;  // SQ_EDOWN
    }
}

DEVI IssuePlan make_plan(const StepArgs &a, const Geo &g, const StSmem &sm, int q, const Item &t) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31;
    IssuePlan P;
    P.dw = P.ds = 0;
    P.ex = nullptr;
    P.fp4 = !(q == SQ_RT || q == SQ_DN || q == SQ_UP);
    P.pair = (q == SQ_SGU || q == SQ_EGU);
    if (!P.fp4) {
        const uint16_t *W = q == SQ_RT ? a.w.router : q == SQ_DN ? a.w.w_dn : a.w.w_up;
        const int ld = q == SQ_UP ? g.L : g.H;
        const int nrows = q == SQ_RT ? g.E : q == SQ_DN ? g.L : g.H;
        const int k0 = t.ks * (q == SQ_RT ? p.kr_rt : q == SQ_DN ? p.kr_dn : p.kr_up);
        const int r0 = lane >> 4, u = lane & 15, row = 16 * t.a + r0;
        P.w = reinterpret_cast<const unsigned char *>(W + (size_t)(row < nrows ? row : 0) * ld + k0 + 8 * u);
        P.s = reinterpret_cast<const unsigned char *>(W);
        P.wpi = 2 * ld * 2;
        P.spi = 0;
        P.valid = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) P.valid |= (row + 2 * i < nrows ? 1u : 0u) << i;
        P.dst = r0 * 256 + 16 * (u ^ ((r0 & 1) << 2));
    } else {
        const uint8_t *Q, *S;
        size_t ldq, lds, row0;
        int k0;
        if (q == SQ_SGU) {
            Q = a.w.sh_gate_q; S = a.w.sh_gate_s; ldq = g.H / 2; lds = g.H / 32; row0 = (size_t)64 * t.a;
            k0 = t.ks * p.kr_sgu;
            P.dw = a.w.sh_up_q - a.w.sh_gate_q;
            P.ds = a.w.sh_up_s - a.w.sh_gate_s;
        } else if (q == SQ_EGU) {
            Q = a.w.gate_q; S = a.w.gate_s; ldq = g.L / 2; lds = g.L / 32;
            row0 = (size_t)sm.act_e[t.a] * g.I + 64 * t.b;
            k0 = t.ks * p.kr_egu;
            P.dw = a.w.up_q - a.w.gate_q;
            P.ds = a.w.up_s - a.w.gate_s;
        } else if (q == SQ_SD) {
            Q = a.w.sh_down_q; S = a.w.sh_down_s; ldq = g.Is / 2; lds = g.Is / 32; row0 = (size_t)64 * t.a;
            k0 = t.ks * p.kr_sd;
        } else {  // SQ_EDOWN
            Q = a.w.down_q; S = a.w.down_s; ldq = g.I / 2; lds = g.I / 32;
            row0 = (size_t)sm.act_e[t.a] * g.L + 64 * t.b;
            k0 = 0;
        }
        P.w = Q + (row0 + (lane >> 2)) * ldq + k0 / 2 + 16 * (lane & 3);
        P.s = S + (row0 + lane) * lds + k0 / 32;
        P.wpi = (int)(8 * ldq);
        P.spi = (int)(32 * lds);
        P.valid = 0xffu;
        P.dst = (lane >> 2) * 64 + 16 * (lane & 3);
    }
    // activation pieces of this lane (lane + 32j for j < 2) and its exponent
    int ncols, pitch = kPitchF16;
    bool swz = true;
    switch (q) {
        case SQ_RT: case SQ_DN: ncols = g.B; pitch = kPitchB16; swz = false; break;
        case SQ_UP: ncols = 2 * g.B; pitch = kPitchB16; swz = false; break;
        case SQ_SGU: ncols = g.B; break;
        case SQ_SD: ncols = 2 * g.B; break;
        default: ncols = 2 * sm.act_cnt[t.a]; break;  // SQ_EGU, SQ_EDOWN
    }
    if (q == SQ_SGU && lane < g.B) P.ex = a.ws.x16e + t.ks * 4 + lane;
    if (q == SQ_SD && lane < g.B) P.ex = a.ws.sh16e + t.ks * 4 + lane;
    if (q == SQ_EGU && lane < sm.act_cnt[t.a]) P.ex = a.ws.h16e + t.ks * 4 + sm.ent[sm.act_off[t.a] + lane] / g.K;
    if (q == SQ_EDOWN && lane < sm.act_cnt[t.a]) P.ex = a.ws.a16e + t.a * 4 + lane;
    P.a0 = P.a1 = nullptr;
    P.adst0 = P.adst1 = 0;
    {
        const int c = lane >> 4, u = lane & 15;
        if (c < ncols) {
            P.a0 = reinterpret_cast<const unsigned char *>(act_col(a, g, sm, q, t, c) + 8 * u);
            P.adst0 = kSlotAct + c * pitch + 16 * (swz ? swz2(u) : u);
        }
        if (c + 2 < ncols) {
            P.a1 = reinterpret_cast<const unsigned char *>(act_col(a, g, sm, q, t, c + 2) + 8 * u);
            P.adst1 = kSlotAct + (c + 2) * pitch + 16 * (swz ? swz2(u) : u);
        }
    }
    return P;
}

// stage c of the planned item: weights always, the activation part when `act`
DEVI void issue_planned(const IssuePlan &P, uint32_t slot, int c, bool act) {
    const int lane = threadIdx.x & 31;
    const int kk = P.pair ? (c >> 1) : c;
    const bool up = P.pair && (c & 1);
    if (P.fp4) {
        const unsigned char *b = P.w + (up ? P.dw : 0) + 64 * kk;
#pragma unroll
        for (int i = 0; i < 8; ++i) cp16(slot + P.dst + 512 * i, b + i * P.wpi);
        const unsigned char *sb = P.s + (up ? P.ds : 0) + 4 * kk;
        cp4(slot + kSlotSc + 4 * lane, sb);
        cp4(slot + kSlotSc + 4 * (lane + 32), sb + P.spi);
    } else {
        const unsigned char *b = P.w + 256 * kk;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const bool ok = (P.valid >> i) & 1u;
            cp16_zfill(slot + P.dst + 512 * i, ok ? b + i * P.wpi : P.s, ok);
        }
    }
    if (act) {
        const int ka = 256 * kk;
        if (P.a0) cp16(slot + P.adst0, P.a0 + ka);
        if (P.a1) cp16(slot + P.adst1, P.a1 + ka);
        if (P.ex) cp4(slot + kSlotExp + 4 * lane, P.ex);
    }
}

// ---------------------------------------------------------------------------------------------
// stage compute

// bf16: 16 rows x 128 k against up to 4 staged columns; two accumulator chains
DEVI void mma_stage_bf16(const unsigned char *slot, int ncols, float (&acc0)[4], float (&acc1)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, sw = (g & 1) << 2;
    const unsigned char *ra = slot + g * 256, *rb = slot + (g + 8) * 256;
    const unsigned char *xc = slot + kSlotAct + (g < ncols ? g : 0) * kPitchB16;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int u = 4 * r + q, uw = 16 * (u ^ sw);
        const uint4 A = *reinterpret_cast<const uint4 *>(ra + uw);
        const uint4 Bm = *reinterpret_cast<const uint4 *>(rb + uw);
        uint4 xb = *reinterpret_cast<const uint4 *>(xc + 16 * u);
        if (g >= ncols) xb = make_uint4(0u, 0u, 0u, 0u);
        mma_bf16(acc0, A.x, Bm.x, A.y, Bm.y, xb.x, xb.y);
        mma_bf16(acc1, A.z, Bm.z, A.w, Bm.w, xb.z, xb.w);
    }
}

// router: 16 rows (two 8-row groups) x 128 k in fp64 (slot q of step s of a 32-k chunk holds
// k = 8q + s); column g is token g
DEVI void mma_stage_router(const unsigned char *slot, int B, double (&c)[2][2], double (&d)[2][2]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const unsigned char *xc = slot + kSlotAct + (g < B ? g : 0) * kPitchB16;
#pragma unroll
    for (int G = 0; G < 2; ++G) {
        const int row = 8 * G + g, sw = (row & 1) << 2;
        const unsigned char *ra = slot + row * 256;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int u = 4 * r + q;
            const uint4 A = *reinterpret_cast<const uint4 *>(ra + 16 * (u ^ sw));
            uint4 xb = *reinterpret_cast<const uint4 *>(xc + 16 * u);
            if (g >= B) xb = make_uint4(0u, 0u, 0u, 0u);
            const double av[8] = {bf16_lo(A.x), bf16_hi(A.x), bf16_lo(A.y), bf16_hi(A.y),
                                  bf16_lo(A.z), bf16_hi(A.z), bf16_lo(A.w), bf16_hi(A.w)};
            const double xv[8] = {bf16_lo(xb.x), bf16_hi(xb.x), bf16_lo(xb.y), bf16_hi(xb.y),
                                  bf16_lo(xb.z), bf16_hi(xb.z), bf16_lo(xb.w), bf16_hi(xb.w)};
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                mma_f64(c[G][0], c[G][1], av[2 * s], xv[2 * s]);
                mma_f64(d[G][0], d[G][1], av[2 * s + 1], xv[2 * s + 1]);
            }
        }
    }
}

// MXFP4: 64 rows (four 16-row tiles) x 128 k; lane quad q owns 32-element block q of each row;
// word w of its 16 code bytes holds MMA steps 2w, 2w+1 against activation unit 4q + w
DEVI void mma_stage_fp4(const unsigned char *slot, int ncols, float (&acc)[4][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, sh = 8 * q;
    uint4 v[4];
    const unsigned char *xc = slot + kSlotAct + (g < ncols ? g : 0) * kPitchF16;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        v[w] = *reinterpret_cast<const uint4 *>(xc + 16 * swz2(4 * q + w));
        if (g >= ncols) v[w] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int r0 = 16 * t + g, r1 = r0 + 8;
        const uint4 c0 = *reinterpret_cast<const uint4 *>(slot + r0 * 64 + 16 * q);
        const uint4 c1 = *reinterpret_cast<const uint4 *>(slot + r1 * 64 + 16 * q);
        const uint32_t s0 = *reinterpret_cast<const uint32_t *>(slot + kSlotSc + 4 * r0);
        const uint32_t s1 = *reinterpret_cast<const uint32_t *>(slot + kSlotSc + 4 * r1);
        const uint32_t f0 = e8m0_to_f16x2((s0 >> sh) & 0xffu), f1 = e8m0_to_f16x2((s1 >> sh) & 0xffu);
        const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w}, w1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint32_t d0[4], d1[4];
            fp4_decode_word(w0[w], f0, d0);
            fp4_decode_word(w1[w], f1, d1);
            mma_f16(acc[t], d0[0], d1[0], d0[1], d1[1], v[w].x, v[w].y);
            mma_f16(acc[t], d0[2], d1[2], d0[3], d1[3], v[w].z, v[w].w);
        }
    }
}

// ---------------------------------------------------------------------------------------------
// tickets, flags, conversions

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

DEVI float warp_max(float m) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
}

// fp32 src[0..n) -> fp16 hi/lo rows dst_hi/dst_lo scaled by 2^-e, e from the block's max |v|;
// n <= 1024 and a multiple of 64 (every load is issued before the first use)
constexpr int kConvMax = 1024;
DEVI int warp_to_f16_hilo(const float *src, uint16_t *dst_hi, uint16_t *dst_lo, int n) {
    const int lane = threadIdx.x & 31;
    float2 v[kConvMax / 64];
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < kConvMax / 64; ++j) {
        const int i = 64 * j + 2 * lane;
        v[j] = i < n ? __ldcg(reinterpret_cast<const float2 *>(src + i)) : make_float2(0.0f, 0.0f);
    }
#pragma unroll
    for (int j = 0; j < kConvMax / 64; ++j) m = fmaxf(m, fmaxf(fabsf(v[j].x), fabsf(v[j].y)));
    const int e = prescale_shift(warp_max(m));
    const float sc = exp2i(-e);
#pragma unroll
    for (int j = 0; j < kConvMax / 64; ++j) {
        const int i = 64 * j + 2 * lane;
        if (i < n) {
            const float x0 = v[j].x * sc, x1 = v[j].y * sc;
            const uint32_t hi = pack_f16x2(x0, x1);
            const uint32_t lo = pack_f16x2(x0 - f16_lo(hi), x1 - f16_hi(hi));
            *reinterpret_cast<uint32_t *>(dst_hi + i) = hi;
            *reinterpret_cast<uint32_t *>(dst_lo + i) = lo;
        }
    }
    return e;
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

// the CTA's copy of the routing tables (first warp to need it loads it)
DEVI bool ensure_routing(const StepArgs &a, StSmem &sm) {
    const int lane = threadIdx.x & 31;
    volatile int *state = &sm.route_state;
    if (*state == 2) return true;
    int mine = 0;
    if (lane == 0) mine = atomicCAS(&sm.route_state, 0, 1) == 0 ? 1 : 0;
    mine = __shfl_sync(0xffffffffu, mine, 0);
    if (mine) {
        if (!warp_wait_geq(a, a.ws.ctl + CTL_ROUTE_READY, 1u)) {
            if (lane == 0) atomicExch(&sm.route_state, 3);  // aborted
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
        if (a.ws.trace && lane == 0)
            a.ws.trace[((size_t)blockIdx.x * kTraceRowsPerSm + (threadIdx.x >> 5)) * kTraceStamps + 12] = global_ns();
        __threadfence_block();
        __syncwarp();
        if (lane == 0) atomicExch(&sm.route_state, 2);
        return true;
    }
    // another warp of this CTA loads it
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
// epilogues (after the last stage of an item)

struct Acc {
    float f[2][4][4];     // [gate|up][row tile][4] for MXFP4; f[0][0..1] chains for bf16
    double c[2][2], d[2][2];
};

DEVI void acc_zero(Acc &r) {
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int j = 0; j < 4; ++j) r.f[m][t][j] = 0.0f;
#pragma unroll
    for (int G = 0; G < 2; ++G) r.c[G][0] = r.c[G][1] = r.d[G][0] = r.d[G][1] = 0.0;
}

// x16 block (token, 512 k): bf16 x -> fp16 x * 2^-e
DEVI void st_x16(const StepArgs &a, const Geo &g, int it) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, t = it / p.s_sgu, kb = it % p.s_sgu, k0 = kb * p.kr_sgu;
    const uint16_t *src = a.x + (size_t)t * g.H + k0;
    float m = 0.0f;
    for (int i = 2 * lane; i < p.kr_sgu; i += 64) {
        const uint32_t v = *reinterpret_cast<const uint32_t *>(src + i);
        m = fmaxf(m, fmaxf(fabsf(bf16_lo(v)), fabsf(bf16_hi(v))));
    }
    const int e = prescale_shift(warp_max(m));
    const float sc = exp2i(-e);
    uint16_t *dst = a.ws.x16 + (size_t)t * g.H + k0;
    for (int i = 2 * lane; i < p.kr_sgu; i += 64) {
        const uint32_t v = *reinterpret_cast<const uint32_t *>(src + i);
        *reinterpret_cast<uint32_t *>(dst + i) = pack_f16x2(bf16_lo(v) * sc, bf16_hi(v) * sc);
    }
    if (lane == 0) a.ws.x16e[kb * 4 + t] = e;
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(a.ws.ctl + p.c_x16 + kb, 1u);
}

DEVI void epi_router(const StepArgs &a, const Geo &g, StSmem &sm, const Item &t, Acc &r) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    double *part = a.ws.st_rt_part + (size_t)t.ks * 2 * g.E;
#pragma unroll
    for (int G = 0; G < 2; ++G) {
        const int row = 16 * t.a + 8 * G + gg;
        if (row < g.E) {
            if (2 * q < g.B) part[(size_t)(2 * q) * g.E + row] = r.c[G][0] + r.d[G][0];
            if (2 * q + 1 < g.B) part[(size_t)(2 * q + 1) * g.E + row] = r.c[G][1] + r.d[G][1];
        }
    }
    if (!warp_last_of(a.ws.ctl + p.c_rt_tk + t.a, (unsigned)p.s_rt)) return;
    for (int i = lane; i < 16 * g.B; i += 32) {
        const int b = i >> 4, row = 16 * t.a + (i & 15);
        if (row < g.E) {
            const float lg = (float)sum_splits<double, 16>(a.ws.st_rt_part + (size_t)b * g.E + row, (size_t)2 * g.E, p.s_rt);
            a.ws.logits[(size_t)b * g.E + row] = lg;
            // top-k key: fp32 sigmoid score (computed in double) bits + 1; 0 marks "no expert"
            const float sc = (float)(1.0 / (1.0 + exp(-(double)lg)));
            a.ws.st_key[(size_t)b * g.E + row] = (sc >= 0.0f ? __float_as_uint(sc) : 0u) + 1u;
        }
    }
    if (a.flags & kFlagTestStall) return;  // the routing never completes: its waits must time out
    if (!warp_count_reaches(a.ws.ctl + CTL_RT_DONE, (unsigned)g.rt_groups)) return;
    unsigned long long *tr =
        a.ws.trace ? a.ws.trace + ((size_t)blockIdx.x * kTraceRowsPerSm + (threadIdx.x >> 5)) * kTraceStamps : nullptr;
    if (tr && lane == 0) tr[14] = global_ns();
    const long long c0 = clock64();
    for (int b = 0; b < g.B; ++b) st_topk_token(a, g, sm, b);
    const long long c1 = clock64();
    if (tr && lane == 0) tr[15] = global_ns();
    st_buckets(a, g, sm);
    const long long c2 = clock64();
    if (tr && lane == 0) {
        tr[11] = global_ns();
        tr[8] = c1 - c0;
        tr[13] = c2 - c1;
    }
}

DEVI void epi_dn(const StepArgs &a, const Geo &g, const Item &t, Acc &r) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    float *part = a.ws.st_dn_part + (size_t)t.ks * 2 * g.L;
    const int row = 16 * t.a + gg;
#pragma unroll
    for (int j = 0; j < 2; ++j)
        if (2 * q + j < g.B) {
            part[(size_t)(2 * q + j) * g.L + row] = r.f[0][0][j] + r.f[0][1][j];
            part[(size_t)(2 * q + j) * g.L + row + 8] = r.f[0][0][2 + j] + r.f[0][1][2 + j];
        }
    if (!warp_last_of(a.ws.ctl + p.c_dn_tk + t.a, (unsigned)p.s_dn)) return;
    for (int i = lane; i < 16 * g.B; i += 32) {
        const int b = i >> 4, rr = 16 * t.a + (i & 15);
        a.ws.h[(size_t)b * g.L + rr] = sum_splits(a.ws.st_dn_part + (size_t)b * g.L + rr, (size_t)2 * g.L, p.s_dn);
    }
    const int kb = (16 * t.a) / p.kr_egu;
    if (!warp_count_reaches(a.ws.ctl + p.c_dnb + kb, (unsigned)(p.kr_egu / 16))) return;
    for (int b = 0; b < g.B; ++b) {
        const int e = warp_to_f16_hilo(a.ws.h + (size_t)b * g.L + kb * p.kr_egu,
                                       a.ws.h16 + (size_t)(2 * b) * g.L + kb * p.kr_egu,
                                       a.ws.h16 + (size_t)(2 * b + 1) * g.L + kb * p.kr_egu, p.kr_egu);
        if (lane == 0) a.ws.h16e[kb * 4 + b] = e;
    }
    warp_publish(a.ws.ctl + p.c_h16 + kb, 1u);
}

DEVI void epi_up(const StepArgs &a, const Geo &g, const Item &t, Acc &r) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    float *part = a.ws.st_up_part + (size_t)t.ks * 2 * g.H;
    const int row = 16 * t.a + gg;
    if (q < g.B) {  // columns 2q, 2q+1: token q's hi and lo parts
        part[(size_t)q * g.H + row] = (r.f[0][0][0] + r.f[0][1][0]) + (r.f[0][0][1] + r.f[0][1][1]);
        part[(size_t)q * g.H + row + 8] = (r.f[0][0][2] + r.f[0][1][2]) + (r.f[0][0][3] + r.f[0][1][3]);
    }
    if (!warp_last_of(a.ws.ctl + p.c_up_tk + t.a, (unsigned)p.s_up)) return;
    if (g.ns && !warp_wait_geq(a, a.ws.ctl + CTL_SD_DONE, (unsigned)g.sd_tiles)) return;
    for (int i = lane; i < 16 * g.B; i += 32) {
        const int b = i >> 4, rr = 16 * t.a + (i & 15);
        const float s = sum_splits(a.ws.st_up_part + (size_t)b * g.H + rr, (size_t)2 * g.H, p.s_up);
        if (a.ws.up_tap) a.ws.up_tap[(size_t)b * g.H + rr] = s;
        const float shv = g.ns ? __ldcg(a.ws.sh + (size_t)b * g.H + rr) : 0.0f;
        a.out[(size_t)b * g.H + rr] = f32_to_bf16_rne(s + shv);
    }
}

DEVI void epi_sgu(const StepArgs &a, const Geo &g, const Item &t, Acc &r, const unsigned char *slot) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    float *part = a.ws.st_sgu_part + (size_t)t.ks * 2 * 2 * g.Is;
    const int *ex = reinterpret_cast<const int *>(slot + kSlotExp);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int b = 2 * q + j;  // x16 columns are tokens
        if (b < g.B) {
            const float sc = exp2i(ex[b]);
            float *pg = part + (size_t)b * 2 * g.Is, *pu = pg + g.Is;
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
                const int row = 64 * t.a + 16 * tt + gg;
                pg[row] = r.f[0][tt][j] * sc;
                pg[row + 8] = r.f[0][tt][2 + j] * sc;
                pu[row] = r.f[1][tt][j] * sc;
                pu[row + 8] = r.f[1][tt][2 + j] * sc;
            }
        }
    }
    if (!warp_last_of(a.ws.ctl + p.c_sgu_tk + t.a, (unsigned)p.s_sgu)) return;
    const size_t st = (size_t)2 * 2 * g.Is;
    for (int i = lane; i < 64 * g.B; i += 32) {
        const int b = i >> 6, rr = 64 * t.a + (i & 63);
        const float *pb = a.ws.st_sgu_part + (size_t)b * 2 * g.Is;
        const float gs = sum_splits(pb + rr, st, p.s_sgu), us = sum_splits(pb + g.Is + rr, st, p.s_sgu);
        a.ws.sh_a[(size_t)b * g.Is + rr] = gs / (1.0f + expf(-gs)) * us;
    }
    const int kb = (64 * t.a) / p.kr_sd;
    if (!warp_count_reaches(a.ws.ctl + p.c_sgb + kb, (unsigned)(p.kr_sd / 64))) return;
    for (int b = 0; b < g.B; ++b) {
        const int e = warp_to_f16_hilo(a.ws.sh_a + (size_t)b * g.Is + kb * p.kr_sd,
                                       a.ws.sh16 + (size_t)(2 * b) * g.Is + kb * p.kr_sd,
                                       a.ws.sh16 + (size_t)(2 * b + 1) * g.Is + kb * p.kr_sd, p.kr_sd);
        if (lane == 0) a.ws.sh16e[kb * 4 + b] = e;
    }
    warp_publish(a.ws.ctl + p.c_sh16 + kb, 1u);
}

DEVI void epi_egu(const StepArgs &a, const Geo &g, const StSmem &sm, const Item &t, Acc &r,
                  const unsigned char *slot) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    const int cnt = sm.act_cnt[t.a], off = sm.act_off[t.a];
    const int nent = g.B * g.K;
    const int *ex = reinterpret_cast<const int *>(slot + kSlotExp);
    if (q < cnt) {  // columns 2q, 2q+1: the slot's entry q, hi and lo parts
        const int ent = sm.ent[off + q];
        const float sc = exp2i(ex[q]);
        float *pg = a.ws.st_egu_part + ((size_t)t.ks * nent + ent) * 2 * g.I, *pu = pg + g.I;
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
            const int row = 64 * t.b + 16 * tt + gg;
            pg[row] = (r.f[0][tt][0] + r.f[0][tt][1]) * sc;
            pg[row + 8] = (r.f[0][tt][2] + r.f[0][tt][3]) * sc;
            pu[row] = (r.f[1][tt][0] + r.f[1][tt][1]) * sc;
            pu[row + 8] = (r.f[1][tt][2] + r.f[1][tt][3]) * sc;
        }
    }
    if (!warp_last_of(a.ws.ctl + p.c_egu_tk + t.a * g.egu_tiles + t.b, (unsigned)p.s_egu)) return;
    const size_t st = (size_t)nent * 2 * g.I;
    for (int i = lane; i < 64 * cnt; i += 32) {
        const int m = i >> 6, rr = 64 * t.b + (i & 63);
        const int ent = sm.ent[off + m];
        const float *pb = a.ws.st_egu_part + (size_t)ent * 2 * g.I;
        const float gs = sum_splits(pb + rr, st, p.s_egu), us = sum_splits(pb + g.I + rr, st, p.s_egu);
        a.ws.a[(size_t)ent * g.I + rr] = gs / (1.0f + expf(-gs)) * us;
    }
    if (!warp_count_reaches(a.ws.ctl + p.c_gu + t.a, (unsigned)g.egu_tiles)) return;
    for (int m = 0; m < cnt; ++m) {
        const int ent = sm.ent[off + m];
        const int e = warp_to_f16_hilo(a.ws.a + (size_t)ent * g.I, a.ws.a16 + (size_t)(2 * ent) * g.I,
                                       a.ws.a16 + (size_t)(2 * ent + 1) * g.I, g.I);
        if (lane == 0) a.ws.a16e[t.a * 4 + m] = e;
    }
    warp_publish(a.ws.ctl + p.c_a16 + t.a, 1u);
}

DEVI void epi_sd(const StepArgs &a, const Geo &g, const Item &t, Acc &r, const unsigned char *slot) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    const int *ex = reinterpret_cast<const int *>(slot + kSlotExp);
    float *part = a.ws.st_sd_part + (size_t)t.ks * 2 * g.H;
    if (q < g.B) {
        const float sc = exp2i(ex[q]);
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
            const int row = 64 * t.a + 16 * tt + gg;
            part[(size_t)q * g.H + row] = (r.f[0][tt][0] + r.f[0][tt][1]) * sc;
            part[(size_t)q * g.H + row + 8] = (r.f[0][tt][2] + r.f[0][tt][3]) * sc;
        }
    }
    if (!warp_last_of(a.ws.ctl + p.c_sd_tk + t.a, (unsigned)p.s_sd)) return;
    for (int i = lane; i < 64 * g.B; i += 32) {
        const int b = i >> 6, rr = 64 * t.a + (i & 63);
        a.ws.sh[(size_t)b * g.H + rr] = sum_splits(a.ws.st_sd_part + (size_t)b * g.H + rr, (size_t)2 * g.H, p.s_sd);
    }
    warp_signal_add(a.ws.ctl + CTL_SD_DONE, 1u);
}

DEVI void epi_edown(const StepArgs &a, const Geo &g, const StSmem &sm, const Item &t, Acc &r,
                    const unsigned char *slot) {
    const StreamPlan &p = a.p.st;
    const int lane = threadIdx.x & 31, gg = lane >> 2, q = lane & 3;
    const int cnt = sm.act_cnt[t.a], off = sm.act_off[t.a];
    const int *ex = reinterpret_cast<const int *>(slot + kSlotExp);
    if (q < cnt) {
        const int ent = sm.ent[off + q];
        const float sc = exp2i(ex[q]);
        float *y = a.ws.y + (size_t)ent * g.L;
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
            const int row = 64 * t.b + 16 * tt + gg;
            y[row] = (r.f[0][tt][0] + r.f[0][tt][1]) * sc;
            y[row + 8] = (r.f[0][tt][2] + r.f[0][tt][3]) * sc;
        }
    }
    __threadfence();
    __syncwarp();
    // one count per entry on its (token, 64-row tile); the K-th combines the token's rows
    unsigned mine = 0;
    if (lane < cnt) {
        const int tok = sm.ent[off + lane] / g.K;
        mine = atomicAdd(a.ws.ctl + p.c_comb + tok * g.ed_tiles + t.b, 1u) == (unsigned)(g.K - 1) ? 1u : 0u;
    }
    unsigned todo = __ballot_sync(0xffffffffu, mine != 0);
    if (todo) __threadfence();
    while (todo) {
        const int m = __ffs(todo) - 1;
        todo &= todo - 1;
        const int tok = sm.ent[off + m] / g.K;
        // ylat rows 64*tile + 2*lane, +1: weighted slot sum in slot order
        const int l = 64 * t.b + 2 * lane;
        float s0 = 0.0f, s1 = 0.0f;
        for (int r0 = 0; r0 < g.K; r0 += 8) {
            float wv[8];
            float2 yv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int rr = r0 + j;
                wv[j] = rr < g.K ? __ldcg(a.ws.wts + (size_t)tok * g.K + rr) : 0.0f;
                yv[j] = rr < g.K ? __ldcg(reinterpret_cast<const float2 *>(a.ws.y + ((size_t)tok * g.K + rr) * g.L + l))
                                 : make_float2(0.0f, 0.0f);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (r0 + j < g.K) {
                    s0 += wv[j] * yv[j].x;
                    s1 += wv[j] * yv[j].y;
                }
        }
        a.ws.ylat[(size_t)tok * g.L + l] = s0;
        a.ws.ylat[(size_t)tok * g.L + l + 1] = s1;
        const uint32_t hi = pack_bf16x2(s0, s1);
        const uint32_t lo = pack_bf16x2(s0 - bf16_lo(hi), s1 - bf16_hi(hi));
        *reinterpret_cast<uint32_t *>(a.ws.ylat16 + (size_t)(2 * tok) * g.L + l) = hi;
        *reinterpret_cast<uint32_t *>(a.ws.ylat16 + (size_t)(2 * tok + 1) * g.L + l) = lo;
        warp_signal_add(a.ws.ctl + p.c_yl + (64 * t.b) / p.kr_up, 1u);
    }
}

}  // namespace

// ---------------------------------------------------------------------------------------------
// the kernel

// One launch runs queues [q_lo, q_hi); the step is four launches (see launch_stream), and the
// last one (q_hi == SQ_N) clears the control block for the next step.
__global__ void __launch_bounds__(kStWarps * 32, 1) k_stream(StepArgs a, int q_lo, int q_hi) {
    extern __shared__ __align__(128) unsigned char st_dyn[];
    __shared__ StSmem sm;
    const Geo g = geo(a);
    const StreamPlan &p = a.p.st;
    unsigned *ctl = a.ws.ctl;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *ring = st_dyn + (size_t)warp * kStStages * kSlotBytes;
    unsigned long long *trace =
        a.ws.trace ? a.ws.trace + ((size_t)blockIdx.x * kTraceRowsPerSm + warp) * kTraceStamps : nullptr;
    auto stamp = [&](int i) {
        if (trace && lane == 0) trace[i] = global_ns();
    };
    if (trace && lane < kTraceStamps) trace[lane] = 0ull;
    __syncwarp();
    stamp(0);
    // row 12 of the SM: start and end of this CTA in each of the step's launches
    unsigned long long *launch_row =
        a.ws.trace ? a.ws.trace + ((size_t)blockIdx.x * kTraceRowsPerSm + 12) * kTraceStamps : nullptr;
    const int launch_no = q_lo == SQ_X16 ? 0 : q_lo == SQ_EGU ? 1 : q_lo == SQ_EDOWN ? 2 : 3;
    if (launch_row && threadIdx.x == 0) launch_row[2 * launch_no] = global_ns();

    // after the first launch, every activation block a queue reads was finished by an earlier launch
    for (int i = threadIdx.x; i < kDepBits / 32; i += blockDim.x) sm.dep_ready[i] = q_lo > SQ_SGU ? ~0u : 0u;
    cta_take_init(sm.claim);
    if (threadIdx.x == 0) {
        sm.route_state = 0;
        sm.n_active = 0;
    }
    __syncthreads();

    // producer state (warp-uniform)
    int pq = q_lo, pit = -1, pc = 0, pn = 0, pdep = kDepNone;
    Item pitem = {0, 0, 0};
    IssuePlan pplan;
    int n_iss = 0, n_con = 0;
    bool alive = true;
    int n_active = -1;  // known once the CTA's routing copy is loaded

    // items come from this CTA's range of each queue (one lane per warp takes)
    auto claim_next = [&](int q, int n) {
        int v = -1;
        if (lane == 0) v = cta_take(sm.claim, q, n);
        return __shfl_sync(0xffffffffu, v, 0);
    };
    auto routing_known = [&]() {
        if (n_active >= 0) return true;
        if (*(volatile int *)&sm.route_state == 2) {
            n_active = sm.n_active;
            return true;
        }
        return false;
    };
    // next item for the producer; false when none can start now (routing unknown) or all done
    auto next_item = [&](bool may_block) -> bool {
        while (pq < q_hi) {
            if ((pq == SQ_EGU || pq == SQ_EDOWN) && !routing_known()) {
                if (!may_block) return false;
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
                pitem = decode_item(a, g, pq, it);
                pc = 0;
                pn = item_stages(a, g, pq);
                pplan = make_plan(a, g, sm, pq, pitem);
                pdep = item_dep(pq, pitem);
                return true;
            }
            ++pq;
        }
        return false;
    };
    // issue stages until the ring is full or nothing more can start without waiting
    auto top_up = [&](bool may_block) {
        while (alive && n_iss - n_con < kStStages) {
            if (pit < 0 || pc == pn) {
                pit = -1;
                if (!next_item(may_block && n_iss == n_con)) return;
            }
            const int s = n_iss % kStStages;
            unsigned char *slot = ring + (size_t)s * kSlotBytes;
            const bool act = dep_known(sm, pdep);
            issue_planned(pplan, smem_addr(slot), pc, act);
            cp_commit();
            if (lane == 0) {
                sm.meta[warp][s].q = pq;
                sm.meta[warp][s].item = pit;
                sm.meta[warp][s].c = pc;
                sm.meta[warp][s].n = pn;
                sm.meta[warp][s].act = act ? 1 : 0;
            }
            __syncwarp();
            ++pc;
            ++n_iss;
        }
    };

    // fp16 copies of x for the shared gate/up (few items; taken before the rings start)
    if (g.ns && q_lo <= SQ_X16) {
        const int n = queue_len(a, g, SQ_X16, 0);
        for (int it = claim_next(SQ_X16, n); it >= 0; it = claim_next(SQ_X16, n)) st_x16(a, g, it);
    }
    stamp(1);

    Acc acc;
    acc_zero(acc);
    Item cit = {0, 0, 0};  // the item being consumed
    long long cyc_issue = 0, cyc_data = 0, cyc_dep = 0, cyc_compute = 0, cyc_epi = 0;
    for (;;) {
        const long long ti0 = trace ? clock64() : 0;
        top_up(true);
        const long long ti1 = trace ? clock64() : 0;
        cyc_issue += ti1 - ti0;
        if (!alive || n_con == n_iss) break;  // aborted, or every queue is drained
        const int s = n_con % kStStages;
        unsigned char *slot = ring + (size_t)s * kSlotBytes;
        cp_wait(n_iss - n_con - 1);
        __syncwarp();
        const long long td0 = trace ? clock64() : 0;
        cyc_data += td0 - ti1;
        const SlotMeta m = sm.meta[warp][s];
        if (m.c == 0) cit = decode_item(a, g, m.q, m.item);
        const Item it = cit;
        if (!m.act) {
            // the activation block was not final when the weights were issued: wait for it, then
            // copy the activation part of every issued stage that waits on the same block (those
            // copies write the slots' activation areas only, never bytes still in flight)
            const int dep = item_dep(m.q, it);
            if (!dep_known(sm, dep)) {
                const unsigned *flag;
                unsigned target;
                dep_flag(a, g, dep, &flag, &target);
                if (!warp_wait_geq(a, flag, target)) {
                    alive = false;
                    break;
                }
                if (lane == 0) atomicOr(&sm.dep_ready[dep >> 5], 1u << (dep & 31));
            }
            for (int k = n_con; k < n_iss; ++k) {
                const int s2 = k % kStStages;
                const SlotMeta m2 = sm.meta[warp][s2];
                if (m2.act) continue;
                const Item it2 = decode_item(a, g, m2.q, m2.item);
                if (item_dep(m2.q, it2) != dep) continue;
                copy_act<false>(a, g, sm, ring + (size_t)s2 * kSlotBytes, m2.q, it2, m2.c);
                __syncwarp();
                if (lane == 0) sm.meta[warp][s2].act = 1;
            }
            __syncwarp();
        }
        if (trace) cyc_dep += clock64() - td0;
        if (m.c == 0) acc_zero(acc);
        const long long tc0 = trace ? clock64() : 0;
        const bool upm = m.c & 1;
        switch (m.q) {
            case SQ_RT: mma_stage_router(slot, g.B, acc.c, acc.d); break;
            case SQ_DN: mma_stage_bf16(slot, g.B, acc.f[0][0], acc.f[0][1]); break;
            case SQ_UP: mma_stage_bf16(slot, 2 * g.B, acc.f[0][0], acc.f[0][1]); break;
            case SQ_SGU:
                if (upm) mma_stage_fp4(slot, g.B, acc.f[1]);
                else mma_stage_fp4(slot, g.B, acc.f[0]);
                break;
            case SQ_EGU:
                if (upm) mma_stage_fp4(slot, 2 * sm.act_cnt[it.a], acc.f[1]);
                else mma_stage_fp4(slot, 2 * sm.act_cnt[it.a], acc.f[0]);
                break;
            case SQ_SD: mma_stage_fp4(slot, 2 * g.B, acc.f[0]); break;
            case SQ_EDOWN: mma_stage_fp4(slot, 2 * sm.act_cnt[it.a], acc.f[0]); break;
        }
        __syncwarp();
        const long long tc1 = trace ? clock64() : 0;
        cyc_compute += tc1 - tc0;
        if (m.c == m.n - 1) {
            switch (m.q) {
                case SQ_RT: epi_router(a, g, sm, it, acc); break;
                case SQ_DN: epi_dn(a, g, it, acc); break;
                case SQ_UP: epi_up(a, g, it, acc); break;
                case SQ_SGU: epi_sgu(a, g, it, acc, slot); break;
                case SQ_EGU: epi_egu(a, g, sm, it, acc, slot); break;
                case SQ_SD: epi_sd(a, g, it, acc, slot); break;
                case SQ_EDOWN: epi_edown(a, g, sm, it, acc, slot); break;
            }
            __syncwarp();
            if (trace) cyc_epi += clock64() - tc1;
        }
        ++n_con;
    }
    cp_wait(0);  // nothing of this warp's may still land in shared memory
    __syncwarp();
    stamp(9);
    if (trace && lane == 0) {
        trace[2] = cyc_issue;
        trace[3] = cyc_data;
        trace[4] = cyc_dep;
        trace[5] = cyc_compute;
        trace[6] = cyc_epi;
        trace[7] = n_con;
    }

    // leave; the last CTA out clears the control block for the next step
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        sm.exit_last = (atomicAdd(ctl + CTL_EXIT, 1u) == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    stamp(10);
    if (launch_row && threadIdx.x == 0) launch_row[2 * launch_no + 1] = global_ns();
    if (sm.exit_last) {
        __threadfence();
        if (q_hi == SQ_N) {
            for (int i = threadIdx.x; i < CTL_FIXED; i += blockDim.x) ctl[i] = 0u;
            for (int i = p.c_rt_tk + threadIdx.x; i < p.words; i += blockDim.x) ctl[i] = 0u;
        } else if (threadIdx.x == 0) {
            ctl[CTL_EXIT] = 0u;  // the next launch counts its own CTAs; everything else carries over
        }
    }
}

bool stream_supports(const Dims &d, int B) {
    if (B < 1 || B > kStMaxBatch || d.k > 32 || d.k > d.E || d.E > 1024 || B * d.k > kMaxActive) return false;
    if (d.H % 128 || d.L % 128 || d.I % 128 || d.I > kConvMax || (d.n_shared && d.Is % 128)) return false;
    StreamPlan sp;
    stream_plan(d, sp, 0);
    return sp.s_sgu <= 64 && sp.s_egu <= 16 && sp.kr_egu <= kConvMax && sp.s_sd <= 16 && sp.kr_sd <= kConvMax &&
           sp.s_up <= 32;
}

// largest multiple of 128 that is <= pref and divides K (K is a multiple of 128)
static int pick_range(int K, int pref) {
    for (int r = pref - pref % 128; r >= 128; r -= 128)
        if (K % r == 0) return r;
    return 128;
}

void stream_plan(const Dims &d, StreamPlan &sp, int ctl_base) {
    const int Is = d.n_shared ? d.Is : 128;
    sp.kr_rt = pick_range(d.H, 512);
    sp.kr_dn = pick_range(d.H, 896);
    sp.kr_sgu = pick_range(d.H, 512);
    sp.kr_egu = pick_range(d.L, 512);
    sp.kr_sd = pick_range(Is, 512);
    sp.kr_up = pick_range(d.L, 256);
    sp.s_rt = d.H / sp.kr_rt;
    sp.s_dn = d.H / sp.kr_dn;
    sp.s_sgu = d.H / sp.kr_sgu;
    sp.s_egu = d.L / sp.kr_egu;
    sp.s_sd = Is / sp.kr_sd;
    sp.s_up = d.L / sp.kr_up;
    int c = ctl_base;
    sp.c_rt_tk = c; c += (d.E + 15) / 16;
    sp.c_dn_tk = c; c += d.L / 16;
    sp.c_dnb = c; c += sp.s_egu;
    sp.c_h16 = c; c += sp.s_egu;
    sp.c_x16 = c; c += sp.s_sgu;
    sp.c_sgu_tk = c; c += Is / 64;
    sp.c_sgb = c; c += sp.s_sd;
    sp.c_sh16 = c; c += sp.s_sd;
    sp.c_egu_tk = c; c += d.E * (d.I / 64);
    sp.c_gu = c; c += d.E;
    sp.c_a16 = c; c += d.E;
    sp.c_sd_tk = c; c += d.H / 64;
    sp.c_comb = c; c += kStMaxBatch * (d.L / 64);
    sp.c_yl = c; c += sp.s_up;
    sp.c_up_tk = c; c += d.H / 16;
    sp.words = c;
}

// The step as four launches, each of which only runs work whose inputs the previous launches
// finished: (x16, router and top-k, W_dn, shared gate/up), (expert gate/up, shared down),
// (expert down and combine), (W_up).  Inside a launch no warp waits on another's results, so
// every warp streams; a stage's activation block is always final when it is issued.
cudaError_t launch_stream(const StepArgs &a, cudaStream_t s, int n_sm) {
    static const int bounds[5] = {SQ_X16, SQ_EGU, SQ_EDOWN, SQ_UP, SQ_N};
    cudaError_t e = cudaSuccess;
    for (int ph = 0; ph < kStreamLaunches && e == cudaSuccess; ++ph) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(n_sm);
        cfg.blockDim = dim3(kStWarps * 32);
        cfg.dynamicSmemBytes = kStDynSmem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k_stream, a, bounds[ph], bounds[ph + 1]);
    }
    return e;
}

cudaError_t init_stream_attributes() {
    return cudaFuncSetAttribute(k_stream, cudaFuncAttributeMaxDynamicSharedMemorySize, kStDynSmem);
}

}  // namespace moedec
