// moedec_internal.h -- parameter blocks shared by the host orchestration and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moedec {

constexpr int kMaxBatch = 512;     // tokens per step (speculative decoding: batch x (drafts + 1))
constexpr int kMaxTopK = 32;
constexpr int kMaxEntries = 8192;  // tokens x top_k per step (routing tables of a fused step in shared memory)
constexpr int kMaxExperts = 1024;  // one top-k thread per expert
constexpr int kDenseWarps = 8;     // dense split-K kernels: 8 warps x 16 rows = 128 rows per CTA
constexpr int kDenseRows = 128;
constexpr int kRouterRows = 64;    // router CTA: 8 warps x 8 rows (fp64 m8n8k4)
constexpr int kExpertWarps = 4;    // expert kernels: 4 warps x 16 rows per item
constexpr int kExpertRows = 64;
constexpr int kKChunk = 512;       // activation staging chunk along K
constexpr int kExpertTokGroup = 16;  // tokens of one expert per pass (two 8-column n-tiles)
constexpr int kMaxCtasPerSm = 2;  // persistent kernels: CTAs per SM at most
constexpr int kTraceRowsPerSm = 16;  // trace rows per SM (one per CTA, or one per warp)
// 64ths of the small-batch grid that run the shared expert (the rest run the routed chain)
constexpr int kSmallSharedPer64 = 8;
// Largest K splits of the small-batch step's warp items (router, W_dn, shared gate/up, expert
// gate/up, shared down, W_up); the plan takes the largest count <= these that divides K evenly.
constexpr int kSmallSplitRt = 16, kSmallSplitDn = 16, kSmallSplitSgu = 8, kSmallSplitEgu = 2, kSmallSplitSd = 1,
              kSmallSplitUp = 4;
constexpr int kSmallMaxBatch = 4;  // tokens of the small-batch step
constexpr int kSguBitWords = 16;   // CTL_SGU_BITS words: grids up to 512 CTAs
constexpr int kTraceStamps = 16;     // MOEDEC_TRACE_STAMPS

// e0, ne: the experts whose weights this handle holds, [e0, e0 + ne) of the E the router scores
// (all of them, e0 = 0 and ne = E, unless the handle is one shard of an expert-parallel layer);
// the expert weight arrays are indexed by e - e0.
struct Dims {
    int H, L, E, k, I, Is, n_shared, max_batch, e0, ne;
};

struct Weights {
    const uint16_t *router, *w_dn, *w_up;
    const uint8_t *gate_q, *gate_s, *up_q, *up_s, *down_q, *down_s;
    const uint8_t *sh_gate_q, *sh_gate_s, *sh_up_q, *sh_up_s, *sh_down_q, *sh_down_s;
};

// Split-K plan of one dense matrix-vector product: `blocks` row blocks x `splits` K ranges.
struct SplitPlan {
    int blocks, splits, krange;
};

// Streaming small-batch step (moedec_stream.cu): K range of one work item per matrix (a multiple
// of the stage width dividing K; the splits are K / range), and its control words (offsets into
// ctl[]).
struct StreamPlan {
    int kr_rt, kr_dn, kr_sgu, kr_egu, kr_sd, kr_up;
    int s_rt, s_dn, s_sgu, s_egu, s_sd, s_up;
    int c_rt_tk;   // [E/16]         router 16-row groups: K splits done
    int c_dn_tk;   // [L/16]         W_dn tiles: K splits done
    int c_sgu_tk;  // [I_s/16]       shared gate/up tiles: K splits done
    int c_egu_tk;  // [E*(I/16)]     expert gate/up tiles (per active slot): K splits done
    int c_sd_tk;   // [H/16]         shared down tiles: K splits done
    int c_comb;    // [2*(L/16)]     expert down tiles done per (token, 16-row latent tile)
    int c_up_tk;   // [H/16]         W_up tiles: K splits done
    int words;     // end of the region
};

struct Plan {
    SplitPlan rt, dn, up, sgu, sd;
    StreamPlan st;
    int ticket_rt, ticket_dn, ticket_up, ticket_sgu, ticket_sd, ticket_topk;  // offsets into tickets[]
    int n_tickets;
    // control words of the fused step (zero at rest), offsets into ctl[]
    int ctl_gu;     // [E]           gate/up warp items finished per active-expert slot
    int ctl_comb;   // [maxB][L/16]  expert outputs finished per (token, 16-row latent block)
    int ctl_ylat;   // [L/16]        tokens whose ylat rows of a 16-row block are final
    int ctl_hamax;  // [maxB]        max |h| per token (float bits)
    int ctl_shamax; // [maxB]        max |sh_a| per token (float bits), small-batch schedule
    int ctl_tk;     // [E/8 + L/16 + I_s/16 + 2*H/16 + E*I/16] per-tile tickets of the small-batch schedule
    int ctl_tk_words;
    int s_rt, s_dn, s_sgu, s_egu, s_sd, s_up;  // K splits of the small-batch schedule
    int ctl_words;
    long long wait_limit_ns;  // bound of every device-side wait of the fused step
};

// fixed control words of the fused step
enum CtlWord {
    CTL_QHEAD = 0,      // [8] next item of each work queue
    CTL_RT_DONE = 8,    // router row blocks whose logits are final
    CTL_DN_DONE,        // W_dn row blocks whose h rows are final
    CTL_SGU_DONE,       // shared gate/up row blocks whose sh_a rows are final
    CTL_SD_DONE,        // shared down row blocks whose sh rows are final
    CTL_ROUTE_READY,    // 1 once idx / weights / expert buckets are final
    CTL_TOPK_TICKET,    // tokens whose top-k is written
    CTL_EXIT,           // CTAs that left the fused kernel
    CTL_ABORT,          // set when a bounded wait gave up; every CTA then leaves
    CTL_SGU_REC = 16,   // shared gate/up items whose CTA is recorded in CTL_SGU_BITS (split-K, 17-64 tokens)
    CTL_SGU_BITS = 17,  // [kSguBitWords] one bit per CTA that took a shared gate/up item
    CTL_FIXED = 33
};

// Device workspace of one handle (all sized for max_batch).
struct Work {
    double *rt_part;    // [rt.splits][maxB][E]   router partial sums (fp64)
    double *rt_acc;     // [min(maxB, 4)][E] small-batch router sums (fp64 reductions; zero at rest)
    float *logits;      // [maxB][E]
    float *dn_part;     // [dn.splits][maxB][L]
    float *h;           // [maxB][L]
    int *h_shift;       // [maxB] fp16 staging exponent of h per token
    int *idx;           // [maxB][k]
    float *wts;         // [maxB][k]
    int *n_active;      // [1]  experts with at least one token
    int *active_e;      // [E]  their ids, ascending
    int *active_cnt;    // [E]  tokens per active expert
    int *active_off;    // [E]  offset of the expert's entries
    int *entries;       // [maxB*k] entry = b*k + r, grouped by expert, token-ascending inside a group
    float *egu_part;    // [s_egu][min(maxB,4)*k][2][I] expert gate then up partials (small-batch step)
    float *a;           // [maxB*k][I]  silu(gate) * up per entry
    unsigned *a_amax;   // [maxB*k]     max |a| per entry (float bits)
    float *y;           // [maxB*k][L]  expert output per entry
    float *ylat;        // [maxB][L]
    float *sgu_part;    // [sgu.splits][maxB][2*Is] shared gate then up partials
    float *sh_a;        // [maxB][Is]
    float *sd_part;     // [sd.splits][maxB][H]
    float *sh;          // [maxB][H]
    float *up_part;     // [up.splits][maxB][H]
    float *up_tap;      // [maxB][H] or nullptr
    // streaming small-batch step (at most 2 tokens): split-K partials and top-k keys
    double *st_rt_part;   // [s_rt][2][E]
    unsigned *st_key;     // [2][E]       top-k key per (token, expert): fp32 score bits + 1
    float *st_dn_part;    // [s_dn][2][L]
    float *st_sgu_part;   // [s_sgu][2][2][I_s]
    float *st_egu_part;   // [s_egu][2k][2][I]
    float *st_sd_part;    // [s_sd][2][H]
    float *st_up_part;    // [s_up][2][H]
    unsigned *tickets;  // [n_tickets]
    unsigned *ctl;      // [ctl_words] fused-step control block (zero at rest)
    unsigned long long *trace;  // [n_sm * 16][kTraceStamps] phase timestamps or nullptr
    unsigned *err;      // [1] sticky device error word
};

struct StepArgs {
    Dims d;
    Weights w;
    const uint16_t *next_router;  // [E][H] router of the layer that steps next (L2 prefetch hint), or nullptr
    Work ws;
    Plan p;
    const uint16_t *x;  // [B][H]
    uint16_t *out;      // [B][H]
    float *out_f32;     // [B][H] fp32 W_up ylat + sh before rounding (partial step of a shard), or nullptr
    int B;
    unsigned flags;     // MOEDEC_FLAG_* of the handle
};

// TMA tensor maps of the routed experts' MXFP4 codes (2D uint8 [rows][K/2 bytes]: gate and up
// E*I rows of L/2 bytes, down E*L rows of I/2 bytes), boxes of 8 rows x 128 bytes with the
// 128-byte swizzle.  Made at create when L/256 and I/256 are 1, 2, 4 or 8; `ok` is 0 otherwise
// (the split-K step then stages the experts' activations per segment instead).
struct alignas(64) ExpertMaps {
    CUtensorMap gate, up, down;
    int ok;
};

// K dimensions the ring phases cover: L/256 and I/256 in {1, 2, 4, 8} (one 128-byte line of a row per warp)
__host__ __device__ inline bool ring_dims_ok(const Dims &d) {
    auto ok = [](int k) { return k % 256 == 0 && (k / 256 == 1 || k / 256 == 2 || k / 256 == 4 || k / 256 == 8); };
    return ok(d.L) && ok(d.I);
}

// error word bits
constexpr unsigned kErrBucket = 1u;    // routing bucket overflow (internal invariant)
constexpr unsigned kErrTimeout = 2u;   // a bounded device wait gave up

// host launchers (moedec_kernels.cu)
cudaError_t launch_router_dn(const StepArgs &a, cudaStream_t s);
cudaError_t launch_topk(const StepArgs &a, cudaStream_t s);
cudaError_t launch_expert_gate_up(const StepArgs &a, cudaStream_t s, int n_sm);
cudaError_t launch_expert_down(const StepArgs &a, cudaStream_t s, int n_sm);
cudaError_t launch_combine(const StepArgs &a, cudaStream_t s);
cudaError_t launch_up(const StepArgs &a, cudaStream_t s);
cudaError_t launch_shared_gate_up(const StepArgs &a, cudaStream_t s);
cudaError_t launch_shared_down(const StepArgs &a, cudaStream_t s);
cudaError_t launch_scale_check(const uint8_t *s, size_t n, unsigned *bad, cudaStream_t st);
cudaError_t launch_scores(const float *logits, float *scores, size_t n, cudaStream_t st);
cudaError_t launch_fused(const StepArgs &a, const ExpertMaps &maps, cudaStream_t s, int n_sm);
cudaError_t init_fused_attributes();
constexpr int kStreamLaunches = 4;  // launches of the streaming small-batch step
bool stream_supports(const Dims &d, int B);
void stream_plan(const Dims &d, StreamPlan &sp, int ctl_base);
cudaError_t launch_stream(const StepArgs &a, cudaStream_t s, int n_sm);
cudaError_t init_stream_attributes();
bool fused_small_supports(const Dims &d, int B);
cudaError_t launch_fused_small(const StepArgs &a, const ExpertMaps &maps, cudaStream_t s, int n_sm);
cudaError_t init_fused_small_attributes();
int kernels_per_step(const Dims &d);
// exchange step of an expert-parallel layer (moedec_ep.cu)
constexpr int kEpMaxWorld = 16;
struct EpSlots {
    unsigned *p[kEpMaxWorld];  // this rank's flag word in each rank's flag array (peer pointers)
};
struct EpParts {
    const float *p[kEpMaxWorld];  // each rank's fp32 partial output [B][H] (peer pointers)
};
cudaError_t launch_ep_publish(const EpSlots &slots, int world, unsigned epoch, cudaStream_t s);
cudaError_t launch_ep_combine(const EpParts &parts, const unsigned *flags, int world, unsigned epoch, size_t n,
                              uint16_t *out, unsigned *err, long long wait_ns, int n_sm, cudaStream_t s);
cudaError_t init_kernel_attributes();

}  // namespace moedec
