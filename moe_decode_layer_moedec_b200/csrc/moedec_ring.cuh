// moedec_ring.cuh -- routed-expert phases of the fused steps on per-warp TMA weight rings.
//
// The expert phases stream MXFP4 rows with almost no reuse (one or two tokens per active expert at
// 16 tokens), so they are bound by how many weight bytes each SM keeps in flight and by the
// instruction cost of decoding them.  Register-fed 128-bit loads hold a few KB per warp in flight
// (and stage their data in L1); here the weights bypass the registers on their way in:
//   * A unit is 8 rows of G_e and the same 8 rows of U_e (gate/up: 16 MMA rows, the lane that holds
//     gate row i also holds up row i) or 16 rows of D_e (down).  Units are listed (active slot,
//     token group of at most 8 tokens, unit); CTA c owns the contiguous range [n c / G, n (c+1) / G)
//     and its warp w takes units s0 + w, s0 + w + 8, ... of each token group [s0, s1) in it.
//   * Each warp streams the K/256 128-byte lines of its unit's rows through a private ring of 2 KB
//     stages, each filled by two 2D TMA boxes of 8 rows x 128 bytes (cp.async.bulk.tensor with the
//     128-byte swizzle, completion on the stage's mbarrier), and accumulates over all of K in
//     registers: no partial sums cross warps.  The E8M0 scales (8 bytes per row and line) come
//     with plain loads one stage ahead.
//   * The token group's activations are staged once per group in shared memory (fp16; hi/lo
//     column pairs for at most 4 tokens) behind two CTA barriers, and each lane reads them with one
//     16-byte load per 32-element block.
//   * Each lane reads one 32-bit word (8 codes) of every 32-element block, so the four lanes of an
//     MMA k-step hold the same block: the block's two m16n8k16 MMAs run on unscaled fp16 codes and
//     the E8M0 scale multiplies their fp32 sum once (an exact power of two).
// The kernel shape follows the small-matrix GEMV of the Kimi K3 decode work ("快是可以生成的，
// 可信只能证明（vLLM 重写 Kimi K3 解码路径…）", section 他们换掉了什么), with the Blackwell TMA in place of
// its register loads.
#pragma once

#include "moedec_experts.cuh"

namespace moedec {

constexpr int kRingBytes = 2048;  // one stage: two boxes of 8 rows x 128 bytes
constexpr int kRingMaxStages = 6;
constexpr int kRingTok = 8;       // tokens per group (one 8-column MMA tile)
constexpr int kRingMaxBlocks = 128;  // 16-row blocks of L (L <= 2048 on the ring path)

__host__ __device__ constexpr int ring_stages(int minb) { return minb > 1 ? 2 : 4; }
constexpr int kRingStagesSmall = 2;  // small-batch step: a few units per warp, keep the L1 share

// An issued stage: the row its box A starts at and the 128-byte line it covers.
struct RingUnit {
    int yA, line;
};

struct RingSync {
    unsigned long long full[8][kRingMaxStages];  // per warp and stage: codes landed
    RingUnit unit[8][kRingMaxStages];            // per warp and stage: the unit in it
    unsigned blk[kRingMaxBlocks];                // down: tokens added per 16-row block of L by this CTA
};

DEVI uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

DEVI void mbar_init(uint32_t bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

DEVI void mbar_expect_tx(uint32_t bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

DEVI bool mbar_test(uint32_t bar, unsigned parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Order this thread's earlier generic-proxy accesses of shared memory before its later TMA writes.
DEVI void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// One 2D box of a tensor map into shared memory, completing on `bar`; weights: evict-first in L2.
DEVI void tma_box(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(bar), "l"(l2_evict_first())
        : "memory");
}

DEVI uint64_t ldg_weights_u64(const void *p) {
    uint64_t r;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.u64 %0, [%1], %2;" : "=l"(r) : "l"(p), "l"(l2_evict_first()));
    return r;
}

DEVI uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// Bounded wait of a whole warp on a ring stage (every lane observes the completion; the outcome is
// the same in every lane).  A stage completes without any other CTA, so the limit only guards
// against a fault of the copy itself.
DEVI bool ring_wait(const StepArgs &a, uint32_t bar, unsigned parity) {
    if (__all_sync(0xffffffffu, mbar_test(bar, parity))) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        if (__all_sync(0xffffffffu, mbar_test(bar, parity))) return true;
        int late = (long long)(global_ns() - t0) > a.p.wait_limit_ns;
        late = __shfl_sync(0xffffffffu, late, 0);
        if (late) {
            if ((threadIdx.x & 31) == 0) {
                atomicOr(a.ws.err, kErrTimeout);
                atomicExch(a.ws.ctl + CTL_ABORT, 1u);
            }
            return false;
        }
    }
}

// Token groups of the active slots from the step's global tables (all threads; a barrier must
// follow): slot j has ceil(cnt_j / kRingTok) groups starting at gpref[j].
DEVI void ring_plan(const StepArgs &a, SegPlan &sp, int *s_warp, int n_active) {
    int c[4], tot = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = 4 * threadIdx.x + i;
        c[i] = j < n_active ? (__ldcg(a.ws.active_cnt + j) + kRingTok - 1) / kRingTok : 0;
        tot += c[i];
    }
    int n;
    int base = block_exclusive_scan(tot, s_warp, &n);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = 4 * threadIdx.x + i;
        if (j < n_active) sp.gpref[j] = base;
        base += c[i];
    }
    if (threadIdx.x == 0) sp.ngroups = n;
}

// all threads, once per kernel before the first barrier: every warp's stage barriers, and the
// three tensor maps fetched ahead into the TMA unit's descriptor cache
DEVI void ring_init(RingSync &rs, const ExpertMaps &maps) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane < kRingMaxStages) mbar_init(smem_u32(&rs.full[warp][lane]), 1u);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.gate) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.up) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.down) : "memory");
    }
}

// After a down phase (all threads): every ylat addition of this CTA is made visible, then the
// CTA's per-block token counts go into ctl_ylat.  The W_up items wait for B k counts per block; a
// block is final only once every active expert's rows of it are added, so counting per CTA at the
// end of its phase costs no overlap.
DEVI void ring_publish_down(const StepArgs &a, RingSync &rs) {
    __threadfence();
    __syncthreads();
    for (int i = threadIdx.x; i < a.d.L / 16; i += blockDim.x)
        if (rs.blk[i]) atomicAdd(a.ws.ctl + a.p.ctl_ylat + i, rs.blk[i]);
}

// ---------------------------------------------------------------------------------------------
// The ring phase: each warp owns whole units (see the top of the file).

constexpr int kRingXPad = 32;  // halfs after each staged column (pitch = K + 32: 64 bytes mod 128)

struct RingGroup {        // the token group being computed (written by the CTA at its start)
    int ent[kRingTok];    // entry of each token
    int shift[kRingTok];  // staging exponent of each token
    float w[kRingTok];    // routing weight of each entry (down)
    int ntok;
};

// Row-owner epilogues of unit t: lane (g, q) holds MMA rows g and g + 8 for columns 2q, 2q + 1
// (with at most 4 tokens: token q's hi and lo parts).  Gate/up: rows g (gate) and g + 8 (up) are
// the same row 8t + g of a.
DEVI void ring_rows_epi_gate_up(const StepArgs &a, const RingGroup &gr, int t, const float (&acc)[4], int ntok,
                                bool split) {
    const int I = a.d.I, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int row = 8 * t + g, t0 = split ? q : 2 * q;
    const bool ok0 = t0 < ntok, ok1 = !split && 2 * q + 1 < ntok;
    float m0 = 0.0f, m1 = 0.0f;
    if (ok0) {
        const float sc = exp2i(gr.shift[t0]);
        const float gv = (split ? acc[0] + acc[1] : acc[0]) * sc, uv = (split ? acc[2] + acc[3] : acc[2]) * sc;
        const float av = gv / (1.0f + expf(-gv)) * uv;
        a.ws.a[(size_t)gr.ent[t0] * I + row] = av;
        m0 = fabsf(av);
    }
    if (ok1) {
        const float sc = exp2i(gr.shift[2 * q + 1]);
        const float gv = acc[1] * sc, uv = acc[3] * sc;
        const float av = gv / (1.0f + expf(-gv)) * uv;
        a.ws.a[(size_t)gr.ent[2 * q + 1] * I + row] = av;
        m1 = fabsf(av);
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
    }
    if (g == 0) {
        if (ok0) atomicMax(a.ws.a_amax + gr.ent[t0], __float_as_uint(m0));
        if (ok1) atomicMax(a.ws.a_amax + gr.ent[2 * q + 1], __float_as_uint(m1));
    }
}

// Down: w * y of rows 16t + g and 16t + g + 8 added into ylat; the block's token count in shared
// memory (published after the phase).
DEVI void ring_rows_epi_down(const StepArgs &a, RingSync &rs, const RingGroup &gr, int t, const float (&acc)[4],
                             int ntok, bool split) {
    const int L = a.d.L, K = a.d.k, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int row = 16 * t + g, t0 = split ? q : 2 * q;
    const bool ok0 = t0 < ntok, ok1 = !split && 2 * q + 1 < ntok;
    if (ok0) {
        float *y = a.ws.ylat + (size_t)(gr.ent[t0] / K) * L + row;
        const float sc = exp2i(gr.shift[t0]), w = gr.w[t0];
        atomicAdd(y, (split ? acc[0] + acc[1] : acc[0]) * sc * w);
        atomicAdd(y + 8, (split ? acc[2] + acc[3] : acc[2]) * sc * w);
    }
    if (ok1) {
        float *y = a.ws.ylat + (size_t)(gr.ent[2 * q + 1] / K) * L + row;
        const float sc = exp2i(gr.shift[2 * q + 1]), w = gr.w[2 * q + 1];
        atomicAdd(y, acc[1] * sc * w);
        atomicAdd(y + 8, acc[3] * sc * w);
    }
    if (lane == 0) atomicAdd(&rs.blk[t], (unsigned)ntok);
}

// dynamic shared memory of the row-owner ring phases: alignment slack, rings, staged columns
__host__ __device__ inline size_t ring_rows_smem(int nsw, const Dims &d) {
    const int k = d.L > d.I ? d.L : d.I;
    return 1024 + (size_t)8 * nsw * kRingBytes + (size_t)kRingTok * (k + kRingXPad) * 2;
}

// The group's tokens as fp16 columns (pitch K + kRingXPad halfs): with at most 4 tokens column
// 2c = fp16(v) and 2c + 1 = fp16(v - fp16(v)), else column c = fp16(v); v = source row * 2^-shift.
// All threads; L1-bypassing loads (other CTAs wrote the sources).
template <bool GU>
DEVI void ring_stage(const StepArgs &a, const RingGroup &gr, uint16_t *xs) {
    const int K = GU ? a.d.L : a.d.I, pitch = K + kRingXPad, units = K / 8, ntok = gr.ntok;
    const bool split = ntok <= 4;
    for (int i = threadIdx.x; i < ntok * units; i += blockDim.x) {
        const int t = i / units, u = i % units, ent = gr.ent[t];
        const float *src = (GU ? a.ws.h + (size_t)(ent / a.d.k) * a.d.L : a.ws.a + (size_t)ent * a.d.I) + 8 * u;
        const float4 v0 = __ldcg(reinterpret_cast<const float4 *>(src));
        const float4 v1 = __ldcg(reinterpret_cast<const float4 *>(src) + 1);
        const float sc = exp2i(-gr.shift[t]);
        const float v[8] = {v0.x * sc, v0.y * sc, v0.z * sc, v0.w * sc, v1.x * sc, v1.y * sc, v1.z * sc, v1.w * sc};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            hi[h] = pack_f16x2(v[2 * h], v[2 * h + 1]);
            lo[h] = pack_f16x2(v[2 * h] - f16_lo(hi[h]), v[2 * h + 1] - f16_hi(hi[h]));
        }
        const int col = split ? 2 * t : t;
        *reinterpret_cast<uint4 *>(xs + (size_t)col * pitch + 8 * u) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        if (split) *reinterpret_cast<uint4 *>(xs + (size_t)(col + 1) * pitch + 8 * u) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// Units [lo, hi) of an expert phase.  Warp w takes units s0 + w, s0 + w + 8, ...
// of each token group [s0, s1) of the range.  `pos` is the warp's running ring position (stages
// consumed so far, the same in every lane; it carries over between the phases).  The caller zeroes
// rs.blk before a down phase and publishes it afterwards (ring_publish_down).  The CTA's threads
// all call it (it has barriers); returns this warp's outcome (false after an abort).
template <bool GU, int NSW>
DEVI bool ring_rows(const StepArgs &a, const ExpertMaps &maps, int na, const SegPlan &sp, RingSync &rs,
                    RingGroup &gr, uint8_t *ring, uint16_t *xs, int lo, int hi, unsigned &pos) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    const int K = GU ? a.d.L : a.d.I, lines = K / 256;
    const int nt = GU ? a.d.I / 8 : a.d.L / 16;  // units per token group
    const int rows_e = GU ? a.d.I : a.d.L;       // rows of one expert in the streamed matrices
    const size_t sld = (size_t)K / 32;
    const uint32_t wring = smem_u32(ring) + (uint32_t)(warp * NSW * kRingBytes);
    const uint32_t xsa = smem_u32(xs);
    const int pitch_b = 2 * (K + kRingXPad);
    uint32_t swo[8];  // this lane's offsets of word q of each 16-byte block chunk (128-byte swizzle)
#pragma unroll
    for (int b = 0; b < 8; ++b) swo[b] = (uint32_t)(g * 128 + ((b ^ g) << 4) + 4 * q);
    RingUnit *info = rs.unit[warp];

    // issue cursor (the same in every lane): group igi with its range end is1, unit iu, line il,
    // slot ij, expert ie; idone once this warp's units are all requested
    int igi = lo / nt, is1 = min(hi, (igi + 1) * nt), iu = lo + warp, il = 0, ij = 0, ie = 0;
    bool idone = lo >= hi;
    auto iseek = [&]() {  // the first group from igi on that has a unit for this warp
        while (!idone && iu >= is1) {
            if (is1 >= hi) {
                idone = true;
                break;
            }
            ++igi;
            iu = igi * nt + warp;
            is1 = min(hi, (igi + 1) * nt);
        }
        if (!idone) {
            ij = seg_slot(sp, na, igi);
            ie = __ldcg(a.ws.active_e + ij);
        }
    };
    iseek();
    unsigned pi = pos;
    auto issue = [&]() {
        if (idone) return;
        if (lane == 0) {
            const int yA = ie * rows_e + (GU ? 8 : 16) * (iu - igi * nt);
            const unsigned st = pi % NSW;
            info[st] = RingUnit{yA, il};
            const uint32_t dst = wring + st * kRingBytes, bar = smem_u32(&rs.full[warp][st]);
            mbar_expect_tx(bar, kRingBytes);
            tma_box(dst, GU ? &maps.gate : &maps.down, 128 * il, yA, bar);
            tma_box(dst + 1024, GU ? &maps.up : &maps.down, 128 * il, GU ? yA : yA + 8, bar);
        }
        ++pi;
        if (++il == lines) {
            il = 0;
            iu += 8;
            if (iu >= is1) iseek();
        }
    };
    if (lane == 0) fence_proxy_async_smem();  // the staging buffers of the previous phase alias the ring
    for (int k = 0; k < NSW; ++k) issue();
    __syncwarp();
    // E8M0 scales of the stage st: bytes [8 l, 8 l + 8) of its rows g and g + 8
    auto scales = [&](unsigned st, uint64_t &s0, uint64_t &s1) {
        const int yA = info[st].yA, l = info[st].line;
        s0 = ldg_weights_u64((GU ? a.w.gate_s : a.w.down_s) + (size_t)(yA + g) * sld + 8 * l);
        s1 = ldg_weights_u64((GU ? a.w.up_s : a.w.down_s) + (size_t)(GU ? yA + g : yA + 8 + g) * sld + 8 * l);
    };
    uint64_t c0 = 0, c1 = 0;
    if (pi != pos) scales(pos % NSW, c0, c1);

    bool ok = true;
    for (int gi = lo / nt; gi * nt < hi; ++gi) {
        const int s0 = gi * nt > lo ? gi * nt : lo, s1 = min(hi, (gi + 1) * nt);
        const int j = seg_slot(sp, na, gi);
        // the group's tokens, once every warp is done with the previous group's columns
        __syncthreads();
        if (threadIdx.x < kRingTok) {
            const int cnt = __ldcg(a.ws.active_cnt + j), gg = gi - sp.gpref[j];
            const int ntok = min(kRingTok, cnt - gg * kRingTok), t = threadIdx.x;
            if (t == 0) gr.ntok = ntok;
            if (t < ntok) {
                const int ent = __ldcg(a.ws.entries + __ldcg(a.ws.active_off + j) + gg * kRingTok + t);
                gr.ent[t] = ent;
                gr.w[t] = GU ? 0.0f : __ldcg(a.ws.wts + ent);
                if (GU) gr.shift[t] = prescale_shift(__uint_as_float(__ldcg(a.ws.ctl + a.p.ctl_hamax + ent / a.d.k)));
            }
        }
        if (!GU) {
            // every gate/up unit of slot j (all its token groups) must be written; then the
            // exponents of the entries' a rows
            const int cnt = __ldcg(a.ws.active_cnt + j);
            const unsigned want = (unsigned)(((cnt + kRingTok - 1) / kRingTok) * (a.d.I / 8));
            __syncthreads();
            if (threadIdx.x == 0) {
                const bool w_ok = wait_geq(a, a.ws.ctl + a.p.ctl_gu + j, want);
                __threadfence();
                gr.ntok = w_ok ? gr.ntok : -gr.ntok - 1;  // negative: aborted
            }
            __syncthreads();
            if (gr.ntok < 0) {
                ok = false;
                break;
            }
            if (threadIdx.x < gr.ntok)
                gr.shift[threadIdx.x] = prescale_shift(__uint_as_float(__ldcg(a.ws.a_amax + gr.ent[threadIdx.x])));
        }
        __syncthreads();
        ring_stage<GU>(a, gr, xs);
        __syncthreads();
        const int ntok = gr.ntok;
        const bool split = ntok <= 4;
        unsigned units_done = 0;
        for (int u = s0 + warp; u < s1 && ok; u += 8) {
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int l = 0; l < lines; ++l) {
                uint64_t m0 = 0, m1 = 0;
                if (pi - pos >= 2u) scales((pos + 1) % NSW, m0, m1);
                const unsigned st = pos % NSW;
                if (!ring_wait(a, smem_u32(&rs.full[warp][st]), (pos / NSW) & 1u)) {
                    ok = false;
                    break;
                }
                const uint32_t base = wring + st * kRingBytes;
                uint32_t w0[8], w1[8];
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    w0[b] = lds_u32(base + swo[b]);
                    w1[b] = lds_u32(base + 1024 + swo[b]);
                }
                ++pos;
                __syncwarp();
                if (lane == 0) fence_proxy_async_smem();  // this stage's reads come before its refill
                issue();
                __syncwarp();  // the refilled stage's unit record is visible to the warp
                const uint64_t sc0 = c0, sc1 = c1;
                c0 = m0;
                c1 = m1;
                const uint32_t xrow = xsa + g * pitch_b + 2 * (256 * l + 8 * q);
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    const float f0 = __int_as_float((int)((sc0 >> (8 * b)) & 0xffu) << 23);
                    const float f1 = __int_as_float((int)((sc1 >> (8 * b)) & 0xffu) << 23);
                    uint4 xv;
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(xv.x), "=r"(xv.y), "=r"(xv.z), "=r"(xv.w)
                                 : "r"(xrow + 64 * b));
                    uint32_t d0[4], d1[4];
                    e2m1x8_to_f16x2(w0[b], d0);
                    e2m1x8_to_f16x2(w1[b], d1);
                    float tmp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    mma_f16(tmp, d0[0], d1[0], d0[1], d1[1], xv.x, xv.y);
                    mma_f16(tmp, d0[2], d1[2], d0[3], d1[3], xv.z, xv.w);
                    acc[0] = fmaf(tmp[0], f0, acc[0]);
                    acc[1] = fmaf(tmp[1], f0, acc[1]);
                    acc[2] = fmaf(tmp[2], f1, acc[2]);
                    acc[3] = fmaf(tmp[3], f1, acc[3]);
                }
            }
            if (!ok) break;
            const int t = u - gi * nt;
            if (GU) ring_rows_epi_gate_up(a, gr, t, acc, ntok, split);
            else ring_rows_epi_down(a, rs, gr, t, acc, ntok, split);
            ++units_done;
        }
        if (GU && units_done && !(a.flags & kFlagTestStallExperts)) warp_signal_add(a.ws.ctl + a.p.ctl_gu + j, units_done);
    }
    if (!ok) {
        // copies still in flight must land before the ring's shared memory is used again
        for (; pos != pi; ++pos) ring_wait(a, smem_u32(&rs.full[warp][pos % NSW]), (pos / NSW) & 1u);
    }
    return ok;
}

}  // namespace moedec
