/*
 * moedec.h -- C ABI of the B200 (sm_100a) sparse latent-MoE decode layer step.
 *
 * The operation.  One decode step of one MoE layer of a Kimi-K3-shaped model: E routed
 * experts with top-k active per token, MXFP4 expert weights, a latent space of width L
 * below the hidden width H, and one always-on shared expert.  Kimi K3 has 896 experts with
 * 16 active per token and stores its weights as MXFP4 ("快是可以生成的，可信只能证明（vLLM
 * 重写 Kimi K3 解码路径，以及怎么放心合并 Agent 写的内核）", section 为什么一条请求会慢).
 * The step's parts -- router scoring, the latent projection, the routed experts, the shared
 * expert on its own stream -- are the ones that page lists (section 他们换掉了什么), and
 * decode at small batch is bounded by streaming the weights from HBM (same page, section
 * 为什么一条请求会慢; "NVIDIA uses a 12,000-line Megakernel to optimize Kimi K3 inference…",
 * section 为什么解码优化比训练优化更难).  For tokens x[b] (bf16, width H):
 *
 *   logit[b,e] = fp32( sum_j R[e,j] x[b,j] )    exact products, fp64 accumulation
 *   s[b,e]     = fp32( 1 / (1 + exp(-logit)) )  (evaluated in fp64)
 *   idx[b,:]   = the top_k experts by s, the lower index first among equal s
 *   w[b,r]     = s_r / (fp32 sum of the k selected s, in rank order)
 *   h          = W_dn x[b]                       (H -> L)
 *   ylat       = sum_r w[b,r] * D_e( silu(G_e h) * (U_e h) ),  e = idx[b,r]
 *   out[b]     = bf16( W_up ylat + SD( silu(SG x[b]) * (SU x[b]) ) )   (L -> H, one rounding)
 *
 * Number formats.  bf16 values are passed as their 16-bit patterns (uint16_t).  An MXFP4
 * matrix [N, K] (OCP Microscaling Formats v1.0) is two arrays: codes uint8 [N][K/2], element
 * 2j in the low nibble of byte j and 2j+1 in the high nibble, and E8M0 scale bytes uint8
 * [N][K/32], one per 32-element block along K; element = E2M1(code) * 2^(scale - 127).
 *
 * Conventions for every call:
 *   - Every pointer is a CUDA device pointer unless the argument says "host".
 *   - Arrays are dense and row-major; every weight pointer is 16-byte aligned.
 *   - A stream argument is a cudaStream_t passed as void*; NULL is the legacy default stream.
 *   - Calls return MOEDEC_OK (0) or a negative moedec_status; they never abort the process.
 *   - A handle is not thread-safe: one host thread at a time, one step in flight per handle
 *     (steps of one handle issued on one stream are ordered by that stream).
 */
#ifndef MOEDEC_H
#define MOEDEC_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define MOEDEC_API __declspec(dllexport)
#else
#define MOEDEC_API __attribute__((visibility("default")))
#endif

#define MOEDEC_ABI_VERSION 1

typedef enum moedec_status {
    MOEDEC_OK = 0,
    MOEDEC_ERR_INVALID_ARG = -1,  /* NULL handle/pointer, misaligned pointer, batch < 0, bad abi_version */
    MOEDEC_ERR_UNSUPPORTED = -2,  /* dimensions or batch outside what this library handles (see moedec_create) */
    MOEDEC_ERR_CUDA = -3,         /* a CUDA runtime call failed; the CUDA error is kept in the handle */
    MOEDEC_ERR_OOM = -4,          /* workspace allocation failed */
    MOEDEC_ERR_TIMEOUT = -5,      /* a bounded device-side wait gave up (reported by the next call) */
    MOEDEC_ERR_DEVICE = -6        /* a kernel recorded an internal error word (reported by the next call) */
} moedec_status;

/* Config flags. */
#define MOEDEC_FLAG_TAPS 1u            /* also materialise the fp32 `up` tap (W_up ylat) for tests */
#define MOEDEC_FLAG_SKIP_SCALE_CHECK 2u /* skip moedec_create's scan of the E8M0 scale bytes */
#define MOEDEC_FLAG_TEST_STALL 4u      /* tests only: the fused step's router never publishes its
                                          logits, so the first wait on them runs out after 20 ms and
                                          the step reports MOEDEC_ERR_TIMEOUT (no GPU fault, no hang) */
#define MOEDEC_FLAG_MULTI_KERNEL 8u    /* run each step as eight stream-ordered kernels (shared expert
                                          on the side stream) instead of one fused persistent kernel */
#define MOEDEC_FLAG_TRACE 16u          /* fused step: every CTA stamps %globaltimer at its phase
                                          boundaries (read with moedec_get_trace) */
#define MOEDEC_FLAG_STREAM 32u         /* batches of 1-2 tokens: run the step as four launches of the
                                          streaming kernel (each warp streams its work items through
                                          a shared-memory ring of cp.async stages) instead of the
                                          small-batch persistent kernel */
#define MOEDEC_FLAG_NO_TMA_RING 64u    /* batches above 4 tokens: stage each expert segment's activations
                                          in shared memory and stream its weights through registers,
                                          instead of the per-warp TMA weight rings (the default when
                                          latent/256 and expert_inter/256 are 1, 2, 4 or 8) */
#define MOEDEC_FLAG_TEST_STALL_EXPERTS 128u /* tests only: the TMA-ring expert gate/up phase never
                                          counts its units, so the expert down phase's wait for them
                                          runs out after 20 ms and the step reports
                                          MOEDEC_ERR_TIMEOUT (no GPU fault, no hang) */
#define MOEDEC_TRACE_STAMPS 16         /* stamps per CTA */

typedef struct moedec_config {
    int32_t abi_version;  /* MOEDEC_ABI_VERSION */
    int32_t hidden;       /* H: multiple of 128 */
    int32_t latent;       /* L: multiple of 128 */
    int32_t n_experts;    /* E: 1..1024 */
    int32_t top_k;        /* k: 1..min(E, 32) */
    int32_t expert_inter; /* I: multiple of 128 */
    int32_t shared_inter; /* I_s: multiple of 128 (ignored when n_shared == 0) */
    int32_t n_shared;     /* 0 or 1 shared expert */
    int32_t max_batch;    /* largest B a step will be called with: 1..512, and max_batch * top_k <= 8192 */
    uint32_t flags;       /* MOEDEC_FLAG_* */
} moedec_config;

/*
 * Weights of one layer.  All device pointers, borrowed: the caller keeps them alive and
 * unchanged for the handle's lifetime (they are read with non-coherent loads).  Shapes:
 *   router     bf16 [E][H]          w_down_lat bf16 [L][H]        w_up_lat bf16 [H][L]
 *   gate_q/up_q    [E][I][L/2]      gate_s/up_s    [E][I][L/32]
 *   down_q         [E][L][I/2]      down_s         [E][L][I/32]
 *   sh_gate_q/sh_up_q [I_s][H/2]    sh_gate_s/sh_up_s [I_s][H/32]
 *   sh_down_q      [H][I_s/2]       sh_down_s      [H][I_s/32]
 * The sh_* pointers may be NULL when n_shared == 0.
 */
typedef struct moedec_weights {
    const uint16_t *router, *w_down_lat, *w_up_lat;
    const uint8_t *gate_q, *gate_s, *up_q, *up_s, *down_q, *down_s;
    const uint8_t *sh_gate_q, *sh_gate_s, *sh_up_q, *sh_up_s, *sh_down_q, *sh_down_s;
} moedec_weights;

typedef struct moedec_handle moedec_handle;

/*
 * Create a handle for one layer on the current CUDA device.
 *   cfg, w      host pointers to the config and the weight-pointer table (copied).
 *   out         host pointer that receives the new handle (set to NULL on failure).
 * Allocates the step workspace for cfg->max_batch tokens, a side stream and two events.
 * Unless MOEDEC_FLAG_SKIP_SCALE_CHECK is set it scans every E8M0 scale byte once (one device
 * kernel and one synchronisation): the tensor-core expert kernels fold the block scale into
 * fp16 weights, which is exact for scale bytes 104..140 (2^-23 .. 2^13); any byte outside that
 * range gives MOEDEC_ERR_UNSUPPORTED.
 * Errors: INVALID_ARG (NULL, misaligned, abi_version), UNSUPPORTED (dimensions), OOM, CUDA.
 */
MOEDEC_API int moedec_create(const moedec_config *cfg, const moedec_weights *w, moedec_handle **out);

/*
 * One layer step: out[b] for b < batch from x[b].  By default the whole step is one persistent
 * kernel (one CTA per SM, cooperative launch) whose CTAs take the step's work items in dependency
 * order; every device-side wait in it is bounded (1 s) and a timeout is reported as
 * MOEDEC_ERR_TIMEOUT by the next synchronising call.  MOEDEC_FLAG_MULTI_KERNEL selects the
 * stream-ordered schedule instead (same work items, same results up to fp32 rounding order).
 *   x       bf16 [batch][H], device, 16-byte aligned; read only.
 *   batch   0..max_batch (0 is a no-op that still reports pending device errors).
 *   out     bf16 [batch][H], device, 16-byte aligned; must not overlap x.
 *   stream  the caller's stream; all work is ordered after prior work on it and the call
 *           returns without synchronising.  Work also runs on the handle's side stream,
 *           forked from and joined back into `stream` with events, so the step can be
 *           captured into a CUDA graph on `stream`.
 * Errors: INVALID_ARG, UNSUPPORTED (batch > max_batch), CUDA (launch failure).  Errors that
 * kernels record on the device (TIMEOUT/DEVICE) are reported by the next synchronising call,
 * moedec_get_routing or moedec_get_taps, which also clear them.
 */
MOEDEC_API int moedec_step(moedec_handle *h, const uint16_t *x, int batch, uint16_t *out, void *stream);

/*
 * Expert parallelism.  A layer can be split over G ranks (one GPU each): rank r creates a shard
 * handle that holds the routed experts [expert_begin, expert_begin + expert_count) of the
 * n_experts the router scores, and a slice of the shared expert's inner width.  Router, top-k and
 * the H -> L projection run on every rank (identical routing everywhere); each rank runs only its
 * own experts and its shared slice, and the layer's output is the bf16 rounding of the sum over
 * ranks of their fp32 partial outputs
 *   partial_r[b] = W_up ylat_r[b] + SD_r( silu(SG_r x[b]) * (SU_r x[b]) ),
 * ylat_r summing the routed terms of rank r's experts only.  This follows from the step's
 * definition above: both terms are linear in the experts and in the shared expert's inner index.
 * The pages run this MoE tensor-parallel over the GPUs of one NVLink domain, with partial results
 * in buffers that every GPU can reach and one fused reduction ("快是可以生成的，可信只能证明（vLLM
 * 重写 Kimi K3 解码路径…）", section 他们换掉了什么); moedec_ep_publish / moedec_ep_combine are
 * that exchange over peer memory.
 *
 * moedec_create_shard: like moedec_create, with cfg->n_experts the layer's total E and
 *   expert_begin >= 0, expert_count >= 1, expert_begin + expert_count <= E.  The gate/up/down
 *   code and scale arrays hold expert_count experts (the first is expert expert_begin), in the
 *   layouts above with E replaced by expert_count.  cfg->shared_inter and the sh_* arrays describe
 *   this rank's slice of the shared expert: rows [s0, s0 + I_s') of SG and SU, and columns
 *   [s0, s0 + I_s') of SD stored as their own dense [H][I_s'/2] and [H][I_s'/32] arrays (I_s' a
 *   multiple of 128, or n_shared = 0 on a rank without a slice).  MOEDEC_FLAG_STREAM is not
 *   supported for shards (UNSUPPORTED).  Errors as moedec_create, plus INVALID_ARG for the range.
 * moedec_step_partial: one step of a shard (or of a whole layer) that writes
 *   partial fp32 [batch][H], device, 16-byte aligned, must not overlap x,
 *   with W_up ylat + sh before any rounding, instead of the bf16 output.  Errors as moedec_step.
 */
MOEDEC_API int moedec_create_shard(const moedec_config *cfg, const moedec_weights *w, int32_t expert_begin,
                                   int32_t expert_count, moedec_handle **out);
MOEDEC_API int moedec_step_partial(moedec_handle *h, const uint16_t *x, int batch, float *partial, void *stream);

#define MOEDEC_EP_MAX_WORLD 16
#define MOEDEC_IPC_HANDLE_BYTES 64

/*
 * The exchange of an expert-parallel step, on rank r of `world` (1..MOEDEC_EP_MAX_WORLD).  Every
 * rank owns a flag array uint32 [world] (zeroed once, never reset) and two partial buffers fp32
 * [max_batch][H] used alternately by step parity; the ranks exchange their addresses once (peer
 * pointers: moedec_ipc_export / moedec_ipc_open).  Step e (e = 1, 2, ...) on rank r is, on one
 * stream:
 *   moedec_step_partial(h, x, B, part_r[e % 2], s);
 *   moedec_ep_publish(h, slots, world, e, s);   slots[q] = &flags_q[r] (host array of device pointers)
 *   moedec_ep_combine(h, parts, flags_r, world, e, B, out, s);   parts[g] = part_g[e % 2]
 * moedec_ep_publish launches one thread that makes all prior work of the stream visible at system
 *   scope and release-stores e into each slot.
 * moedec_ep_combine launches a kernel whose blocks wait until flags[g] >= e for every g (acquire,
 *   system scope; bounded like the step's waits, a timeout is reported as MOEDEC_ERR_TIMEOUT by the
 *   next synchronising call of h and leaves out unwritten), then write
 *   out[b][j] = bf16(((parts[0][b][j] + parts[1][b][j]) + ...) + parts[world-1][b][j]) (fp32 sums in
 *   rank order, one round-to-nearest-even), so every rank gets the same bits.  flags may be NULL:
 *   no wait (the caller orders the partials itself, e.g. world = 1 after a library all-reduce).
 *   parts: host array of `world` device pointers, 16-byte aligned; out: bf16 [batch][H], device,
 *   16-byte aligned.
 * The two-buffer rotation is what makes reuse safe: rank r overwrites part_r[p] in step e + 2 only
 * after its combine of step e + 1, which waited for every rank's publish of e + 1, issued after
 * that rank's combine of step e had read part_r[p].
 * Errors: INVALID_ARG (NULL, misaligned, world out of range, batch < 0), UNSUPPORTED (batch >
 * max_batch), CUDA (launch).
 */
MOEDEC_API int moedec_ep_publish(moedec_handle *h, uint32_t *const *slots, int world, uint32_t epoch, void *stream);
MOEDEC_API int moedec_ep_combine(moedec_handle *h, const float *const *parts, const uint32_t *flags, int world,
                                 uint32_t epoch, int batch, uint16_t *out, void *stream);

/*
 * CUDA IPC of device memory, for handing a rank's flag array and partial buffers to the other
 * processes of its node.  moedec_ipc_export writes MOEDEC_IPC_HANDLE_BYTES bytes into the host
 * buffer `handle` for the whole device allocation that contains `ptr`, and the byte offset of ptr
 * inside it into the host word *offset; moedec_ipc_open maps such a handle exported by another
 * process into this one (peer access enabled lazily) and returns the allocation's base, to which
 * the importer adds the offset; moedec_ipc_close unmaps that base.  A process cannot open its own
 * handles.  Errors: INVALID_ARG (NULL), CUDA.
 */
MOEDEC_API int moedec_ipc_export(const void *ptr, void *handle, uint64_t *offset);
MOEDEC_API int moedec_ipc_open(const void *handle, void **ptr);
MOEDEC_API int moedec_ipc_close(void *ptr);

/* Release the workspace, side stream and events (synchronises the side stream). NULL is a no-op. */
MOEDEC_API int moedec_destroy(moedec_handle *h);

/*
 * Cross-layer prefetch hint.  Decode runs the layers one after another, and the next layer's
 * router matrix (E x H bf16) is the first thing its step reads, at the head of its dependency
 * chain.  With next set, every later fused step of h (the default schedules; the streaming and
 * multi-kernel schedules ignore the hint) has CTAs that have run out of work issue L2
 * prefetches of next's router rows (cp.async.bulk.prefetch.L2, no data returned to the SM), so
 * that the next layer's step starts on L2 hits ("快是可以生成的，可信只能证明（vLLM 重写 Kimi K3
 * 解码路径…）", section 他们换掉了什么: the next weights are prefetched into cache while the
 * current step waits).  Results never depend on the hint.
 *   next  a handle on the same device with the same hidden and n_experts, or NULL to clear the
 *         hint; only its router pointer is recorded, so it must stay valid while h keeps it.
 * Errors: INVALID_ARG (NULL h, mismatched next).
 */
MOEDEC_API int moedec_set_next(moedec_handle *h, const moedec_handle *next);

/*
 * Whether this handle can stream the routed experts of the fused steps through per-warp TMA
 * weight rings: 1 when create made tensor maps over gate_q, up_q and down_q, 0 with
 * MOEDEC_FLAG_NO_TMA_RING or when latent/256 or expert_inter/256 is not in {1, 2, 4, 8}.  With 1,
 * steps of 2 or more tokens use the rings; a step of 1 token keeps the register-fed expert path,
 * which is faster there.  Both paths agree within the float tolerance (the order of fp32 sums
 * differs).  Returns MOEDEC_ERR_INVALID_ARG for NULL h.
 */
MOEDEC_API int moedec_tma_ring(const moedec_handle *h);

/*
 * Routing of the last step, copied on `stream` into caller device buffers:
 *   idx  int32 [batch][top_k] expert indices in rank order (score descending, lower index first)
 *   w    fp32  [batch][top_k] routing weights in the same order
 * Either pointer may be NULL.  batch must equal the last step's batch.  Synchronises `stream`
 * and reports (then clears) any device-side error word of earlier steps: TIMEOUT or DEVICE.
 */
MOEDEC_API int moedec_get_routing(moedec_handle *h, int32_t *idx, float *w, int batch, void *stream);

/*
 * Intermediate values of the last step (test taps), copied on `stream` into caller device buffers:
 *   logits fp32 [batch][E]   h    fp32 [batch][L]   ylat fp32 [batch][L]
 *   sh     fp32 [batch][H]   up   fp32 [batch][H] (W_up ylat; only with MOEDEC_FLAG_TAPS)
 * Any pointer may be NULL.  `up` non-NULL without MOEDEC_FLAG_TAPS gives INVALID_ARG.
 * Synchronises `stream` and reports device-side errors like moedec_get_routing.
 */
MOEDEC_API int moedec_get_taps(moedec_handle *h, float *logits, float *hlat, float *ylat, float *sh, float *up,
                               int batch, void *stream);

/*
 * Router scores of the last step (test tap): scores[b][e] = fp32(1 / (1 + exp(-logit[b][e])))
 * evaluated in fp64 by the same device function the top-k ranks experts with, written on `stream`
 * into the caller's device buffer fp32 [batch][E].  batch must equal the last step's batch.
 * Synchronises `stream` and reports device-side errors like moedec_get_routing.
 */
MOEDEC_API int moedec_get_scores(moedec_handle *h, float *scores, int batch, void *stream);

/*
 * Launch counters (host values): launches[i] counts the kernels of variant i issued by this
 * handle since creation; i = 0 the small-batch schedules (batch <= 4), 1 the split-K schedule
 * (batch >= 5).  n_variants in/out.
 */
MOEDEC_API int moedec_get_launch_counts(moedec_handle *h, uint64_t *launches, int *n_variants);

/* Kernels issued per step of `batch` tokens by this handle (so a timed loop can count its launches):
 * 4 for the streaming schedule (MOEDEC_FLAG_STREAM, batch <= 2), 1 for the other fused schedules, 8 with
 * MOEDEC_FLAG_MULTI_KERNEL (7 without a shared expert). */
MOEDEC_API int moedec_kernels_per_step(moedec_handle *h, int batch);

/* Last CUDA error string recorded by the handle ("" if none); static storage of the handle. */
MOEDEC_API const char *moedec_last_cuda_error(moedec_handle *h);

/*
 * Per-kernel timing.  While enabled, every kernel a step launches is bracketed by a pair of CUDA
 * events recorded on the stream that kernel runs on (the caller's stream or the side stream).
 * moedec_profile_read synchronises both streams and returns, per kernel kind i < *n:
 *   total_ms[i]  summed event-measured duration of its launches since enabling (host array)
 *   launches[i]  number of its launches (host array)
 *   names[i]     static name of the kind (host array of const char*), may be NULL
 * *n is in/out (array capacity in, number of kinds out).  enable=1 resets the sums and starts
 * recording; enable=0 stops recording and keeps what was recorded for moedec_profile_read.  Event
 * pairs recorded while a stream is being captured become part of the graph and hold the times
 * of the graph's latest replay.
 */
MOEDEC_API int moedec_profile_enable(moedec_handle *h, int enable);
MOEDEC_API int moedec_profile_read(moedec_handle *h, double *total_ms, uint64_t *launches, const char **names, int *n);

/*
 * Router logits without any device allocation.  The pages have no counterpart of this call; it
 * exists for callers that cannot call cudaMalloc: code that runs while its stream is being
 * captured into a CUDA graph under a no-allocation policy, processes whose device memory is
 * entirely handed to another allocator, and runtimes with a fixed, pre-planned memory budget.
 *   router   bf16 [n_experts][hidden], device, 16-byte aligned      x  bf16 [batch][hidden], device, 16-byte aligned
 *   logits   fp32 [batch][n_experts], device (output)               stream  cudaStream_t as void*
 * Computes logits[b][e] = fp32(sum_j router[e][j] x[b][j]) (exact products, fp64 sums, one
 * rounding) with the step's router kernel body and its K-split order, so the values are bitwise
 * equal to moedec_get_taps' logits of a step that runs that body (batches above 4, or
 * MOEDEC_FLAG_MULTI_KERNEL).  The small-batch step (batch <= 4) adds its K splits with fp64
 * reductions in arrival order instead, so against its logits the values agree to within one fp32
 * ulp (they differ only where the exact sum lies within fp64 rounding of an fp32 rounding
 * boundary).  Its split-K scratch is one static 2 MiB device array in the library that every GPU
 * loading the library keeps until the process exits; the call only clears the ticket words it
 * needs (an async memset on `stream`).
 * Limit: (hidden / 512) * batch * n_experts * 8 bytes + 4 KiB <= 2 MiB (hidden a multiple of 512;
 * 256 or 128 when it is not, with proportionally more splits); beyond it the call returns
 * MOEDEC_ERR_UNSUPPORTED.  With hidden 7168 and 896 experts that allows batch <= 20.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call before any stream capture.  All calls
 * share the one array, so calls that may overlap on the GPU (different streams, or different
 * host threads) race; serialise them.
 * Errors: INVALID_ARG (NULL or misaligned pointer, batch < 0, non-positive sizes), UNSUPPORTED
 * (hidden not a multiple of 128, n_experts > 1024, scratch limit), CUDA.
 */
MOEDEC_API int moedec_router_logits_noalloc(const uint16_t *router, const uint16_t *x, int n_experts, int hidden,
                                            int batch, float *logits, void *stream);

/*
 * Phase timeline of the last fused step (MOEDEC_FLAG_TRACE): host array out[rows][MOEDEC_TRACE_STAMPS]
 * of %globaltimer nanoseconds, 0 where nothing was stamped; rows = 16 per SM.  *n_cta in/out:
 * capacity in rows in, rows written out.  Synchronises `stream`.  INVALID_ARG without
 * MOEDEC_FLAG_TRACE.
 *   split-K and small-batch kernels, row = CTA: 0 start, 1 router, 2 top-k, 3 W_dn, 4 shared
 *     gate/up, 5 routing wait, 6 expert gate/up, 7 shared down, 8 expert down, 9 W_up, 10 exit
 *     (small-batch: 11 routing seen; the shared-expert CTAs stamp 0, 4, 7, 9, 10 only);
 *     small-batch top-k CTAs also fill row (grid size + CTA): 0 logits complete, 1 scores,
 *     2 warp candidates, 3 ranked, 4 routing written, 5 expert masks (batch > 1), 6 buckets
 *     written, 7 buckets published.
 *   streaming kernel (batch <= 2), row = 16 * CTA + warp: 0 start, 1 fp16 copy of x done,
 *     2..6 SM clock cycles spent issuing copies and claiming work, waiting for a stage's data,
 *     waiting for activation blocks, in MMAs, in item epilogues; 7 stages consumed; 9 last stage
 *     done, 10 exit, 11 expert buckets published (the ranking warp), 12 routing tables loaded
 *     (the loading warp), 14 last router group done and 15 top-k done (the ranking warp);
 *     row 16 * CTA + 12: start and end of the CTA in each of the step's 4 launches (stamps 0..7);
 *     row 16 * CTA + 13: per launch, cycles summed over the CTA's warps in issue, data waits,
 *     MMAs and epilogues (stamps 4 * launch + 0..3); row 16 * CTA + 14: per launch, ns from the
 *     launch's start to its activations staged, and the latest and earliest warp finish after that
 *     (stamps 4 * launch + 0..2).
 */
MOEDEC_API int moedec_get_trace(moedec_handle *h, uint64_t *out, int *n_cta, void *stream);

/* Human-readable name of a status code (static storage). */
MOEDEC_API const char *moedec_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MOEDEC_H */
