// moedec_fused.cu -- the whole decode layer step as one persistent kernel.
//
// One or two CTAs per SM (cooperative launch, so every CTA is resident).  The step's work items
// sit in queues that every CTA drains in the same order (the routed experts in static per-CTA
// segments, the top-k one token per CTA):
//
//   0 router row blocks        (fp64 logits)                       CTA items
//   1 top-k, one per token     waits: all router blocks            token t on CTA t; last builds buckets
//   2 W_dn row blocks          (h)                                 CTA items
//   3 shared gate/up blocks    (sh_a)                              CTA items
//   4 expert gate/up           waits: buckets, all of h            static per-CTA segments
//   5 shared down blocks       waits: all of sh_a                  CTA items
//   6 expert down              waits: that expert's gate/up tiles  static per-CTA segments; w * y added into ylat
//   7 W_up row blocks          waits: their ylat rows, all of sh   CTA items; writes out
//
// An item only ever waits on items of earlier queues (all of which were claimed by resident CTAs
// before any CTA moved on), so the waits always end; each one is still bounded (a.p.wait_limit_ns).  On a timeout the CTA records MOEDEC_ERR_TIMEOUT, sets the
// abort word and leaves; the others see the abort word in their next wait and leave too.  The
// last CTA to leave clears the control block, so the next step starts clean either way.
//
// Routing is known only after queue 1, but nothing waits for a kernel boundary: while one CTA
// ranks the experts the others already stream W_dn and the shared expert, and an expert's down
// rows start as soon as its own gate/up rows are done.
#include "moedec_ring.cuh"

namespace moedec {

enum Queue { Q_ROUTER = 0, Q_TOPK, Q_DN, Q_SGU, Q_EGU, Q_SD, Q_EDOWN, Q_UP, Q_COUNT };

// Batch tiers: token-column tiles of the x consumers (NTX), the shared down (NTS, hi/lo split at
// B <= 4) and the up-projection (NTU, always hi/lo); larger batches run the dense parts in token
// groups of that width.  Up to 64 tokens the kernel runs two CTAs per SM (128 registers per
// thread: 16 warps per SM hide the latency of the MXFP4 decode and MMA chains that 8 warps at
// 255 registers cannot), with 8-token expert groups and routing tables for 64 x 32 selections;
// above 64 tokens one CTA per SM, 16-token expert groups and tables for 8192 selections.  (Two CTAs
// per SM above 64 tokens with the rings, which need no tables, ran B = 256 in 2,468 against
// 1,970 us: the dense parts' 32-token groups cost more than the 16 ring warps per SM gained.)
template <int TIER>
struct Tier;
template <> struct Tier<0> {
    static constexpr int NTX = 1, NTS = 1, NTU = 1, MINB = 2;
    static constexpr int MAXB = 64;
    static constexpr bool SPLITS = true;
    using RT = RouteTables<kMaxExperts, 64 * kMaxTopK>;
};
template <> struct Tier<1> {
    static constexpr int NTX = 1, NTS = 1, NTU = 2, MINB = 2;
    static constexpr int MAXB = 64;
    static constexpr bool SPLITS = false;
    using RT = RouteTables<kMaxExperts, 64 * kMaxTopK>;
};
template <> struct Tier<2> {
    static constexpr int NTX = 2, NTS = 2, NTU = 4, MINB = 2;
    static constexpr int MAXB = 64;
    static constexpr bool SPLITS = false;
    using RT = RouteTables<kMaxExperts, 64 * kMaxTopK>;
};
template <> struct Tier<3> {
    static constexpr int NTX = 4, NTS = 4, NTU = 8, MINB = 2;
    static constexpr int MAXB = 64;
    static constexpr bool SPLITS = false;
    using RT = RouteTables<kMaxExperts, 64 * kMaxTopK>;
};
template <> struct Tier<4> {
    static constexpr int NTX = 8, NTS = 8, NTU = 16, MINB = 1;
    static constexpr int MAXB = kMaxBatch;
    static constexpr bool SPLITS = false;
    using RT = SplitKRoute;
};

__host__ __device__ inline int tier_for_batch(int B) { return B <= 4 ? 0 : B <= 8 ? 1 : B <= 16 ? 2 : B <= 64 ? 3 : 4; }

// Dynamic shared memory: the phases' staging buffers from offset 0 (fused_stage_smem bytes), then
// the routing tables of the step (they must survive the shared-down staging between the two
// expert phases).
template <int TIER>
__host__ __device__ inline size_t fused_stage_smem(const StepArgs &a) {
    using T = Tier<TIER>;
    size_t m = router_smem(a.p.rt.krange);
    auto mx = [&](size_t v) { m = v > m ? v : m; };
    mx((size_t)8 * T::NTX * bf16_pitch(a.p.dn.krange) * 2);
    mx((size_t)8 * T::NTX * f16_pitch(a.p.sgu.krange) * 2);
    mx((size_t)8 * T::NTS * f16_pitch(a.p.sd.krange) * 2);
    mx((size_t)8 * T::NTU * bf16_pitch(up_chunk(T::NTU, a.p.up.krange)) * 2);
    mx(seg_smem(a.d, seg_tok(T::MINB)));
    mx(topk_lists_smem(a.d.E, a.B));  // the top-k's candidates, token masks and offsets
    return (m + 15) & ~(size_t)15;
}

// Dynamic shared memory of a launch: with the TMA rings the expert phases read the routing from
// global memory and the route tables are not kept (ring and staging buffers share offset 0).
template <int TIER>
__host__ __device__ inline size_t fused_smem(const StepArgs &a, bool ring) {
    const size_t st = fused_stage_smem<TIER>(a), r = ring_rows_smem(ring_stages(Tier<TIER>::MINB), a.d);
    return ring ? (st > r ? st : r) : st + sizeof(typename Tier<TIER>::RT);
}

template <int TIER>
__global__ void __launch_bounds__(256, Tier<TIER>::MINB) k_fused(StepArgs a, const __grid_constant__ ExpertMaps maps) {
    using T = Tier<TIER>;
    using RT = typename T::RT;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ TopkSmem topk;
    __shared__ unsigned s_flag;
    __shared__ int s_ok;
    RT &route = *reinterpret_cast<RT *>(smem + fused_stage_smem<TIER>(a));
    __shared__ SegPlan segp;
    __shared__ SegSmem segs;
    __shared__ int s_scan[32];
    __shared__ int s_next;
    __shared__ RingSync rs;
    unsigned *ctl = a.ws.ctl;
    bool alive = true;
    const int n_rt = a.p.rt.blocks * a.p.rt.splits, n_dn = a.p.dn.blocks * a.p.dn.splits;
    const int n_sgu = a.d.n_shared ? a.p.sgu.blocks * a.p.sgu.splits : 0;
    const int n_sd = a.d.n_shared ? a.p.sd.blocks * a.p.sd.splits : 0;
    const int n_up = a.p.up.blocks * a.p.up.splits;
    unsigned long long *trace = a.ws.trace ? a.ws.trace + (size_t)blockIdx.x * kTraceStamps : nullptr;
    auto stamp = [&](int i) {
        if (trace && threadIdx.x == 0) trace[i] = global_ns();
    };
    stamp(0);
    constexpr int NSW = ring_stages(T::MINB);
    const bool use_ring = maps.ok != 0;
    uint8_t *ring = smem + ((1024u - (smem_u32(smem) & 1023u)) & 1023u);  // 1 KB aligned (128-byte swizzle)
    uint16_t *ring_xs = reinterpret_cast<uint16_t *>(ring + 8 * NSW * kRingBytes);
    __shared__ RingGroup ring_gr;
    unsigned ring_pos = 0;
    if (use_ring) ring_init(rs, maps);

    // Items are taken dynamically, one atomic per item on the queue head, each when the CTA is
    // ready for it.  (Claiming one item ahead, to prefetch its weights into L2, let the first CTAs
    // into a queue hold two items each while later ones got none: the dense queues have fewer
    // items than two per CTA.)
    auto cta_queue = [&](int q, int n, auto body) {
        while (alive) {
            __syncthreads();
            if (threadIdx.x == 0) s_next = (int)atomicAdd(ctl + CTL_QHEAD + q, 1u);
            __syncthreads();
            const int it = s_next;
            if (it >= n) break;
            alive = body(it);
        }
    };
    // 0: router
    cta_queue(Q_ROUTER, n_rt, [&](int it) { item_router<true>(a, it, smem, &s_flag); return true; });
    stamp(1);
    // 1: top-k, token t on CTA t (and t + G, ...).  While fewer tokens than CTAs, the top-k CTAs
    // take no W_dn or shared gate/up items: a CTA that ranked a token would claim them late and
    // enter its static range of the expert phase after the others
    for (int t = blockIdx.x; alive && t < a.B; t += gridDim.x)
        alive = item_topk<true>(a, t, topk, smem, (unsigned)a.p.rt.blocks, nullptr, a.ws.ylat, nullptr);
    stamp(2);
    if ((int)blockIdx.x >= a.B || a.B >= (int)gridDim.x) {
        // 2: W_dn
        cta_queue(Q_DN, n_dn, [&](int it) { item_dn<true, T::NTX, T::MAXB>(a, it, smem, &s_flag); return true; });
        stamp(3);
        // 3: shared gate/up
        cta_queue(Q_SGU, n_sgu, [&](int it) {
            if constexpr (TIER == 3) {  // record the CTA (see the expert gate/up ranges below)
                if (threadIdx.x == 0 && gridDim.x <= 32 * kSguBitWords) {
                    atomicOr(ctl + CTL_SGU_BITS + blockIdx.x / 32, 1u << (blockIdx.x % 32));
                    __threadfence();
                    atomicAdd(ctl + CTL_SGU_REC, 1u);
                }
            }
            item_sgu<true, T::NTX, T::MAXB>(a, it, smem, &s_flag);
            return true;
        });
    }
    stamp(4);
    // 4: expert gate/up: routing and all of h must be final; the CTA's static range of the
    // (slot, token group, 128-row block) items, one activation staging per segment
    if (alive) alive = cta_wait_geq(a, ctl + CTL_ROUTE_READY, 1u, &s_ok);
    if (alive) alive = cta_wait_geq(a, ctl + CTL_DN_DONE, (unsigned)a.p.dn.blocks, &s_ok);
    stamp(5);
    auto range = [&](int n, int &lo, int &hi) {
        lo = (int)((long long)n * blockIdx.x / gridDim.x);
        hi = (int)((long long)n * (blockIdx.x + 1) / gridDim.x);
    };
    uint16_t *xs_e = reinterpret_cast<uint16_t *>(smem);
    int n_act = 0;
    if (alive && use_ring) {
        n_act = __ldcg(a.ws.n_active);
        ring_plan(a, segp, s_scan, n_act);
        __syncthreads();
        int lo, hi;
        range((a.d.I / 8) * segp.ngroups, lo, hi);
        if constexpr (TIER == 3) {
            // At 17-64 tokens the CTAs that took a shared gate/up item enter this phase late (those
            // items run into the expert streams), so they get 6/8 of an equal share of its units.
            // Every CTA reads the same final bitmap: the ranges still partition [0, n).
            if (n_sgu && gridDim.x <= 32 * kSguBitWords) {
                alive = cta_wait_geq(a, ctl + CTL_SGU_REC, (unsigned)n_sgu, &s_ok);
                const int c = blockIdx.x, G = gridDim.x;
                int before = 0, total = 0;
                for (int w = 0; w < (G + 31) / 32; ++w) {
                    const unsigned bits = __ldcg(ctl + CTL_SGU_BITS + w);
                    total += __popc(bits);
                    if (w < c / 32) before += __popc(bits);
                    else if (w == c / 32) before += __popc(bits & ((1u << (c % 32)) - 1u));
                }
                const bool mine = (__ldcg(ctl + CTL_SGU_BITS + c / 32) >> (c % 32)) & 1u;
                constexpr long long WN = 8, WS = 6;
                const long long wpre = WN * c - (WN - WS) * before, wtot = WN * G - (WN - WS) * total;
                const long long n = (long long)(a.d.I / 8) * segp.ngroups;
                lo = (int)(n * wpre / wtot);
                hi = (int)(n * (wpre + (mine ? WS : WN)) / wtot);
            }
        }
        const bool ok = alive && ring_rows<true, NSW>(a, maps, n_act, segp, rs, ring_gr, ring, ring_xs, lo, hi, ring_pos);
        alive = __syncthreads_and(ok ? 1 : 0) != 0;
    } else if (alive) {
        cta_load_routing(a, route);
        __syncthreads();
        seg_plan<seg_tok(T::MINB)>(segp, route, s_scan);
        __syncthreads();
        const int nb = a.d.I / 128;
        int lo, hi;
        range(nb * segp.ngroups, lo, hi);
        for_each_segment(segp, route, nb, lo, hi, [&](int j, int g, int b0, int b1) {
            seg_gate_up_any<T::MINB>(a, route, segs, xs_e, j, g, b0, b1);
            return true;
        });
    }
    stamp(6);
    // 5: shared down (above 64 tokens after the expert down phase, see 7)
    if constexpr (TIER != 4)
        cta_queue(Q_SD, n_sd, [&](int it) { return item_sd<true, T::NTS, T::SPLITS, T::MAXB>(a, it, smem, &s_flag, &s_ok); });
    stamp(7);
    // 6: expert down: the same plan over L / 128 blocks per expert; each segment waits for its
    // expert's gate/up tiles
    if (alive) {
        __syncthreads();
        bool ok;
        if (use_ring) {
            for (int i = threadIdx.x; i < kRingMaxBlocks; i += blockDim.x) rs.blk[i] = 0u;
            __syncthreads();
            int lo, hi;
            range((a.d.L / 16) * segp.ngroups, lo, hi);
            ok = ring_rows<false, NSW>(a, maps, n_act, segp, rs, ring_gr, ring, ring_xs, lo, hi, ring_pos);
            ring_publish_down(a, rs);
        } else {
            const int nb = a.d.L / 128;
            int lo, hi;
            range(nb * segp.ngroups, lo, hi);
            ok = for_each_segment(segp, route, nb, lo, hi, [&](int j, int g, int b0, int b1) {
                return seg_down_any<T::MINB>(a, route, segs, xs_e, j, g, b0, b1);
            });
        }
        alive = __syncthreads_and(ok ? 1 : 0) != 0;
    }
    // 7: above 64 tokens the shared down comes after the expert down phase, where the CTAs that
    // finish early take its items while the others complete their ranges (W_up needs all of ylat
    // first, sh only in its last splits): B = 256 1,960 -> 1,907 us; at 16 and 64 tokens it
    // measured neutral and 1 % slower
    if constexpr (TIER == 4)
        cta_queue(Q_SD, n_sd, [&](int it) { return item_sd<true, T::NTS, T::SPLITS, T::MAXB>(a, it, smem, &s_flag, &s_ok); });
    stamp(8);
    if (alive) prefetch_next_router(a, blockIdx.x, gridDim.x);
    // 8: W_up and the output
    cta_queue(Q_UP, n_up, [&](int it) { return item_up<true, T::NTU>(a, it, smem, &s_flag, &s_ok); });
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
        const int nblk = a.d.L / 16;
        for (int i = threadIdx.x; i < CTL_FIXED; i += blockDim.x) ctl[i] = 0u;
        for (int i = threadIdx.x; i < a.d.E; i += blockDim.x) ctl[a.p.ctl_gu + i] = 0u;
        for (int i = threadIdx.x; i < a.B * nblk; i += blockDim.x) ctl[a.p.ctl_comb + i] = 0u;
        for (int i = threadIdx.x; i < nblk; i += blockDim.x) ctl[a.p.ctl_ylat + i] = 0u;
        for (int i = threadIdx.x; i < a.B; i += blockDim.x) ctl[a.p.ctl_hamax + i] = 0u;
    }
}

template <int TIER>
static cudaError_t launch_fused_tier(const StepArgs &a, const ExpertMaps &maps, cudaStream_t s, int n_sm) {
    const size_t sm = fused_smem<TIER>(a, maps.ok != 0);
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_fused<TIER>, 256, sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (per_sm > Tier<TIER>::MINB) per_sm = Tier<TIER>::MINB;
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
    return cudaLaunchKernelEx(&cfg, k_fused<TIER>, a, maps);
}

cudaError_t launch_fused(const StepArgs &a, const ExpertMaps &maps, cudaStream_t s, int n_sm) {
    switch (tier_for_batch(a.B)) {
        case 0: return launch_fused_tier<0>(a, maps, s, n_sm);
        case 1: return launch_fused_tier<1>(a, maps, s, n_sm);
        case 2: return launch_fused_tier<2>(a, maps, s, n_sm);
        case 3: return launch_fused_tier<3>(a, maps, s, n_sm);
        default: return launch_fused_tier<4>(a, maps, s, n_sm);
    }
}

cudaError_t init_fused_attributes() {
    const void *fns[] = {(const void *)k_fused<0>, (const void *)k_fused<1>, (const void *)k_fused<2>,
                         (const void *)k_fused<3>, (const void *)k_fused<4>};
    int dev = 0, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    for (const void *f : fns) {
        // all the dynamic shared memory the device allows next to the kernel's static part (the
        // full-size layer needs at most 132 KB at 64 tokens)
        cudaFuncAttributes fa;
        if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, f);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace moedec
