// moedec_ring.cuh -- routed-expert phases of the split-K step on per-warp TMA weight rings.
//
// The expert phases stream MXFP4 rows with almost no reuse (one or two tokens per active expert at
// 16 tokens), so they are bound by how many weight bytes each SM keeps in flight and by the
// instruction cost of decoding them.  Register-fed 128-bit loads hold a few KB per warp in flight;
// here the weights bypass the registers on their way in:
//   * Warp w of a CTA owns one 128-byte line (a 256-wide K slice) of every row its row group
//     streams: w % (K/256) is the line, w / (K/256) the row group (K/256 = 1, 2, 4 or 8).  Its
//     codes arrive through a private ring of 2 KB stages, each two 2D TMA boxes of 8 rows x 128
//     bytes (cp.async.bulk.tensor with the 128-byte swizzle, completion on the stage's mbarrier);
//     up to four (two CTAs per SM) or six stages of a warp are in flight.  Its E8M0 scales (8 bytes
//     per row) come with plain loads two units ahead; its activation fragment stays in registers
//     for the whole token group.
//   * Each lane reads one 32-bit word (8 codes) of every 32-element block, so the four lanes of an
//     MMA k-step hold the same block: the block's two m16n8k16 MMAs run on unscaled fp16 codes and
//     the E8M0 scale multiplies their fp32 sum once (an exact power of two).
//   * The K-split partials of a unit meet in shared memory; the last warp of the row group to add
//     its partial (a shared-memory counter) sums them in line order and runs the epilogue.
// Expert gate/up units are 8 rows of G_e and the same 8 rows of U_e (16 MMA rows; the lane that
// holds gate row i also holds up row i), expert down units 16 rows of D_e.  Units are listed
// (active slot, token group of at most 8 tokens, unit); CTA c owns the contiguous range
// [n c / G, n (c+1) / G), and its row groups take every (8 / lines)-th unit of it.
// The kernel shape follows the small-matrix GEMV of the Kimi K3 decode work ("快是可以生成的，
// 可信只能证明（vLLM 重写 Kimi K3 解码路径…）", section 他们换掉了什么), with the Blackwell TMA in place of
// its register loads.
#pragma once

#include "moedec_experts.cuh"

namespace moedec {

constexpr int kRingBytes = 2048;  // one stage: two boxes of 8 rows x 128 bytes
constexpr int kRingSlots = 2;     // partial-sum slots per row group
constexpr int kRingMaxStages = 6;
constexpr int kRingTok = 8;       // tokens per group (one 8-column MMA tile)
constexpr int kRingMaxBlocks = 128;  // 16-row blocks of L (L <= 2048 on the ring path)

__host__ __device__ constexpr int ring_stages(int minb) { return minb > 1 ? 3 : 6; }
constexpr int kRingStagesSmall = 2;  // small-batch step: a few units per warp, keep the L1 share

// dynamic shared memory of the ring phases (1 KB of alignment slack, the rings, the partials)
__host__ __device__ inline size_t ring_smem(int nsw) {
    return 1024 + (size_t)8 * nsw * kRingBytes + (size_t)kRingSlots * 8 * 32 * sizeof(float4);
}

// An issued unit: first row of its box A, active slot, token group (global index), unit in group.
struct RingUnit {
    int yA, j, gi, t;
};

struct RingSync {
    unsigned long long full[8][kRingMaxStages];  // per warp and stage: codes landed
    RingUnit unit[8][kRingMaxStages];            // per warp and stage: the unit in it
    unsigned cnt[8][kRingSlots];                 // per row group and slot: partials written
    unsigned gen[8][kRingSlots];                 // per row group and slot: units reduced
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

// Bounded wait of a whole warp for a shared-memory word to reach `want` (a partial-sum slot of its
// row group); gives up when the step was aborted.  Uniform outcome.
DEVI bool slot_wait(const StepArgs &a, const unsigned *wp, unsigned want) {
    const volatile unsigned *w = wp;
    if (__all_sync(0xffffffffu, *w == want)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        if (__all_sync(0xffffffffu, *w == want)) return true;
        int stop = 0;
        if ((threadIdx.x & 31) == 0) {
            if (ld_acquire(a.ws.ctl + CTL_ABORT)) stop = 1;
            else if ((long long)(global_ns() - t0) > a.p.wait_limit_ns) {
                atomicOr(a.ws.err, kErrTimeout);
                atomicExch(a.ws.ctl + CTL_ABORT, 1u);
                stop = 1;
            }
        }
        if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
}

// Unit cursor: unit u of an expert phase with nt units per token group, its active slot j and
// that slot's expert e.  The routing comes from the step's global tables (L2), read when j changes.
struct RingCur {
    int u, j, e;
};

DEVI void cur_seek(const StepArgs &a, RingCur &c, const SegPlan &sp, int n_active, int u, int nt) {
    c.u = u;
    c.j = n_active > 0 ? seg_slot(sp, n_active, u / nt) : 0;
    c.e = n_active > 0 ? __ldcg(a.ws.active_e + c.j) : 0;
}

DEVI void cur_step(const StepArgs &a, RingCur &c, const SegPlan &sp, int n_active, int step, int nt) {
    c.u += step;
    const int gi = c.u / nt, j0 = c.j;
    while (c.j + 1 < n_active && sp.gpref[c.j + 1] <= gi) ++c.j;
    if (c.j != j0) c.e = __ldcg(a.ws.active_e + c.j);
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

// ---------------------------------------------------------------------------------------------
// one expert phase

// Gate/up epilogue of one unit (8 gate rows and the same 8 up rows): a = silu(g) * u for the
// group's tokens and a_amax per entry (the caller counts the unit into ctl_gu later).  r: the unit's summed MMA tile
// (rows g and g + 8, columns 2q and 2q + 1); column c was staged by lane 4c.
DEVI void ring_epi_gate_up(const StepArgs &a, int t, float4 r, int ntok, bool split, int lent, int lsh) {
    const int I = a.d.I, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int ent0 = __shfl_sync(0xffffffffu, lent, 8 * q), ent1 = __shfl_sync(0xffffffffu, lent, 8 * q + 4);
    const int sh0 = __shfl_sync(0xffffffffu, lsh, 8 * q), sh1 = __shfl_sync(0xffffffffu, lsh, 8 * q + 4);
    const int row = 8 * t + g;
    const bool ok0 = split ? q < ntok : 2 * q < ntok, ok1 = !split && 2 * q + 1 < ntok;
    float m0 = 0.0f, m1 = 0.0f;
    if (ok0) {
        const float sc = exp2i(sh0);
        const float gv = (split ? r.x + r.y : r.x) * sc, uv = (split ? r.z + r.w : r.z) * sc;
        const float av = gv / (1.0f + expf(-gv)) * uv;
        a.ws.a[(size_t)ent0 * I + row] = av;
        m0 = fabsf(av);
    }
    if (ok1) {
        const float sc = exp2i(sh1);
        const float gv = r.y * sc, uv = r.w * sc;
        const float av = gv / (1.0f + expf(-gv)) * uv;
        a.ws.a[(size_t)ent1 * I + row] = av;
        m1 = fabsf(av);
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
    }
    if (g == 0) {
        if (ok0) atomicMax(a.ws.a_amax + ent0, __float_as_uint(m0));
        if (ok1) atomicMax(a.ws.a_amax + ent1, __float_as_uint(m1));
    }
}

// Down epilogue of one unit (16 rows of L): w * y added into ylat with fp32 reductions; the unit's
// 16-row block counts the group's tokens in shared memory (published by the caller after the phase).
DEVI void ring_epi_down(const StepArgs &a, RingSync &rs, int t, float4 r, int ntok, bool split, int lent, int lsh, float lw) {
    const int L = a.d.L, K = a.d.k, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int ent0 = __shfl_sync(0xffffffffu, lent, 8 * q), ent1 = __shfl_sync(0xffffffffu, lent, 8 * q + 4);
    const int sh0 = __shfl_sync(0xffffffffu, lsh, 8 * q), sh1 = __shfl_sync(0xffffffffu, lsh, 8 * q + 4);
    const float w0 = __shfl_sync(0xffffffffu, lw, 8 * q), w1 = __shfl_sync(0xffffffffu, lw, 8 * q + 4);
    const int row = 16 * t + g;
    const bool ok0 = split ? q < ntok : 2 * q < ntok, ok1 = !split && 2 * q + 1 < ntok;
    if (ok0) {
        float *y = a.ws.ylat + (size_t)(ent0 / K) * L + row;
        const float sc = exp2i(sh0);
        atomicAdd(y, (split ? r.x + r.y : r.x) * sc * w0);
        atomicAdd(y + 8, (split ? r.z + r.w : r.z) * sc * w0);
    }
    if (ok1) {
        float *y = a.ws.ylat + (size_t)(ent1 / K) * L + row;
        const float sc = exp2i(sh1);
        atomicAdd(y, r.y * sc * w1);
        atomicAdd(y + 8, r.w * sc * w1);
    }
    if (lane == 0) atomicAdd(&rs.blk[t], (unsigned)ntok);
}

// Units [lo, hi) of an expert phase (GU: gate/up, else down) for this CTA.  `pos` is the warp's
// running ring position (stages consumed so far, the same in every lane; it carries over between
// the phases).  The caller zeroes rs.cnt / rs.gen (and rs.blk for down) and passes a barrier
// first; after a down phase it publishes rs.blk into ctl_ylat (ring_publish_down).  Unit i of a
// row group is reduced by its warp i % lines when that warp starts its next unit, so the
// epilogues rotate over the warps.  Returns false after an abort; every copy this warp issued has
// landed (or its bounded wait gave up) by then.
template <bool GU, int NSW>
DEVI bool ring_phase(const StepArgs &a, const ExpertMaps &maps, int na, const SegPlan &sp, RingSync &rs,
                     uint8_t *ring, float4 *part, int lo, int hi, unsigned &pos) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, q = lane & 3;
    const int lines = (GU ? a.d.L : a.d.I) / 256, rowg = 8 / lines;
    const int line = warp % lines, rg = warp / lines;
    const int nt = GU ? a.d.I / 8 : a.d.L / 16;  // units per token group
    const int first = lo + rg;
    const int n = first < hi ? (hi - first + rowg - 1) / rowg : 0;
    const uint32_t wring = smem_u32(ring) + (uint32_t)(warp * NSW * kRingBytes);
    RingUnit *info = rs.unit[warp];

    // issue cursor (the same in every lane): unit ti of token group gi, active slot cj, expert ce
    int gi = first / nt, ti = first % nt, cj = 0, ce = 0;
    if (n > 0) {
        cj = seg_slot(sp, na, gi);
        ce = __ldcg(a.ws.active_e + cj);
    }
    unsigned pi = pos;
    int n_issued = 0;
    auto issue = [&]() {
        if (lane == 0) {
            const int yA = ce * (GU ? a.d.I : a.d.L) + (GU ? 8 : 16) * ti;
            const unsigned st = pi % NSW;
            info[st] = RingUnit{yA, cj, gi, ti};
            const uint32_t dst = wring + st * kRingBytes, bar = smem_u32(&rs.full[warp][st]);
            mbar_expect_tx(bar, kRingBytes);
            tma_box(dst, GU ? &maps.gate : &maps.down, 128 * line, yA, bar);
            tma_box(dst + 1024, GU ? &maps.up : &maps.down, 128 * line, GU ? yA : yA + 8, bar);
        }
        ++pi;
        ++n_issued;
        ti += rowg;
        while (ti >= nt) {
            ti -= nt;
            ++gi;
        }
        const int j0 = cj;
        while (cj + 1 < na && sp.gpref[cj + 1] <= gi) ++cj;
        if (cj != j0) ce = __ldcg(a.ws.active_e + cj);
    };
    if (lane == 0) fence_proxy_async_smem();  // the staging buffers of the previous phase alias the ring
    while (n_issued < n && n_issued < NSW) issue();
    __syncwarp();
    // E8M0 scales of the unit in stage st: bytes [8 line, 8 line + 8) of its rows g and g + 8
    auto scales = [&](unsigned st, uint64_t &s0, uint64_t &s1) {
        const int yA = info[st].yA;
        const size_t sld = (size_t)(GU ? a.d.L : a.d.I) / 32;
        s0 = ldg_weights_u64((GU ? a.w.gate_s : a.w.down_s) + (size_t)(yA + g) * sld + 8 * line);
        s1 = ldg_weights_u64((GU ? a.w.up_s : a.w.down_s) + (size_t)(GU ? yA + g : yA + 8 + g) * sld + 8 * line);
    };
    uint64_t c0 = 0, c1 = 0;
    if (n > 0) scales(pos % NSW, c0, c1);

    uint32_t xb[8][4];
    int xgi = -1, ntok = 0, lent = 0, lsh = 0, gu_j = -1, pj = 0, pt = 0;
    unsigned gu_n = 0;
    float lw = 0.0f;
    bool split = false, ok = true;
    // unit k's partials (all written) -> its epilogue, with the current token group's context
    auto reduce = [&](int k) -> bool {
        const int p = k % kRingSlots;
        if (!slot_wait(a, &rs.cnt[rg][p], (unsigned)lines)) return false;
        __threadfence_block();
        float4 r = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        for (int l = 0; l < lines; ++l) {
            const float4 v = part[(p * 8 + rg * lines + l) * 32 + lane];
            r.x += v.x;
            r.y += v.y;
            r.z += v.z;
            r.w += v.w;
        }
        __syncwarp();
        if (lane == 0) {
            rs.cnt[rg][p] = 0u;
            __threadfence_block();
            *reinterpret_cast<volatile unsigned *>(&rs.gen[rg][p]) = (unsigned)(k / kRingSlots) + 1u;
        }
        if (GU) {
            // count the units per slot, one fence and atomic per slot and warp
            if (pj != gu_j) {
                if (gu_n) warp_signal_add(a.ws.ctl + a.p.ctl_gu + gu_j, gu_n);
                gu_j = pj;
                gu_n = 0;
            }
            ring_epi_gate_up(a, pt, r, ntok, split, lent, lsh);
            ++gu_n;
        } else {
            ring_epi_down(a, rs, pt, r, ntok, split, lent, lsh, lw);
        }
        return true;
    };
    for (int i = 0; i < n; ++i) {
        const RingUnit u = info[pos % NSW];
        if (i > 0 && (i - 1) % lines == line && !reduce(i - 1)) {
            ok = false;
            break;
        }
        if (u.gi != xgi) {
            // a new token group: its activations into this warp's fragment (K slice of the line)
            xgi = u.gi;
            const int gg = u.gi - sp.gpref[u.j];
            const int cnt = __ldcg(a.ws.active_cnt + u.j);
            ntok = min(kRingTok, cnt - gg * kRingTok);
            split = ntok <= 4;  // hi/lo column pairs
            const int c = split ? (g >> 1) : g;
            const bool valid = c < ntok;
            lent = valid ? __ldcg(a.ws.entries + __ldcg(a.ws.active_off + u.j) + gg * kRingTok + c) : 0;
            if (!GU) {
                // every gate/up unit of slot j (all its token groups) must be written
                const unsigned want = (unsigned)(((cnt + kRingTok - 1) / kRingTok) * (a.d.I / 8));
                if (!warp_wait_geq(a, a.ws.ctl + a.p.ctl_gu + u.j, want)) {
                    ok = false;
                    break;
                }
            }
            const float amax = valid ? __uint_as_float(__ldcg(GU ? a.ws.ctl + a.p.ctl_hamax + lent / a.d.k
                                                                : a.ws.a_amax + lent))
                                     : 0.0f;
            lsh = prescale_shift(amax);
            lw = (!GU && valid) ? __ldcg(a.ws.wts + lent) : 0.0f;
            const float sc = exp2i(-lsh);
            const float *src = (GU ? a.ws.h + (size_t)(lent / a.d.k) * a.d.L : a.ws.a + (size_t)lent * a.d.I) +
                               256 * line + 8 * q;
            const bool lo_part = split && (g & 1);
            float4 v0[8], v1[8];
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                v0[b] = v1[b] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (valid) {
                    v0[b] = __ldcg(reinterpret_cast<const float4 *>(src + 32 * b));
                    v1[b] = __ldcg(reinterpret_cast<const float4 *>(src + 32 * b) + 1);
                }
            }
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                const float v[8] = {v0[b].x * sc, v0[b].y * sc, v0[b].z * sc, v0[b].w * sc,
                                    v1[b].x * sc, v1[b].y * sc, v1[b].z * sc, v1[b].w * sc};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    uint32_t hv = pack_f16x2(v[2 * h], v[2 * h + 1]);
                    if (lo_part) hv = pack_f16x2(v[2 * h] - f16_lo(hv), v[2 * h + 1] - f16_hi(hv));
                    xb[b][h] = hv;
                }
            }
        }
        uint64_t m0 = 0, m1 = 0;
        if (i + 1 < n) scales((pos + 1) % NSW, m0, m1);
        // the unit's codes: word q of each 32-element block of rows g and g + 8 (128-byte swizzle:
        // 16-byte chunk b of row r sits at chunk b ^ r)
        const unsigned st = pos % NSW;
        if (!ring_wait(a, smem_u32(&rs.full[warp][st]), (pos / NSW) & 1u)) {
            ok = false;
            break;
        }
        const uint32_t base = wring + st * kRingBytes;
        uint32_t w0[8], w1[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            w0[b] = lds_u32(base + g * 128 + ((b ^ g) << 4) + 4 * q);
            w1[b] = lds_u32(base + 1024 + g * 128 + ((b ^ g) << 4) + 4 * q);
        }
        ++pos;
        __syncwarp();
        if (n_issued < n) {
            if (lane == 0) fence_proxy_async_smem();  // this stage's reads come before its refill
            issue();
        }
        const uint64_t s0 = c0, s1 = c1;
        c0 = m0;
        c1 = m1;
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const float f0 = __int_as_float((int)((s0 >> (8 * b)) & 0xffu) << 23);
            const float f1 = __int_as_float((int)((s1 >> (8 * b)) & 0xffu) << 23);
            uint32_t d0[4], d1[4];
            e2m1x8_to_f16x2(w0[b], d0);
            e2m1x8_to_f16x2(w1[b], d1);
            float tmp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            mma_f16(tmp, d0[0], d1[0], d0[1], d1[1], xb[b][0], xb[b][1]);
            mma_f16(tmp, d0[2], d1[2], d0[3], d1[3], xb[b][2], xb[b][3]);
            acc[0] = fmaf(tmp[0], f0, acc[0]);
            acc[1] = fmaf(tmp[1], f0, acc[1]);
            acc[2] = fmaf(tmp[2], f1, acc[2]);
            acc[3] = fmaf(tmp[3], f1, acc[3]);
        }
        // this warp's K-split partial of unit i into slot i % kRingSlots (free once unit
        // i - kRingSlots is reduced)
        const int p = i % kRingSlots;
        if (!slot_wait(a, &rs.gen[rg][p], (unsigned)(i / kRingSlots))) {
            ok = false;
            break;
        }
        __threadfence_block();
        part[(p * 8 + warp) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            atomicAdd(&rs.cnt[rg][p], 1u);
        }
        pj = u.j;
        pt = u.t;
    }
    if (ok && n > 0 && (n - 1) % lines == line) ok = reduce(n - 1);
    if (GU && gu_n) warp_signal_add(a.ws.ctl + a.p.ctl_gu + gu_j, gu_n);
    if (!ok) {
        // copies still in flight must land before the ring's shared memory is used again
        for (; pos != pi; ++pos) ring_wait(a, smem_u32(&rs.full[warp][pos % NSW]), (pos / NSW) & 1u);
    }
    return ok;
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

}  // namespace moedec
