/*
 * moe_b200.h -- C ABI of the fused MoE FFN layer forward for NVIDIA B200 (sm_100a).
 *
 * The layer (Mixture-of-Kittens blog, section "Overlapping compute and communication in
 * MoE", layer equation):
 *
 *     x' = W_shared(x) + sum_{e in top-k(x)} w_e * W_down^e * SwiGLU(W_up^e x, W_gate^e x),
 *     SwiGLU(u, g) = SiLU(u) (.) g.
 *
 * It runs as six stream-ordered kernels with no host synchronisation and no allocation:
 *   1. router projection  logits = x W_router^T (+ bias)     tcgen05 GEMM, fp32 out
 *   2. gating             warp-level top-k + renormalised softmax, per-chunk expert
 *                         histogram, and (last CTA) the expert/block/tile scans
 *   3. align scatter      grid-wide writes of sorted_ids / expert_ids and each slot's row
 *   4. row gather         x rows copied into expert-tile order
 *   5. expert GEMMs       one persistent kernel; its CTAs claim (expert, m-tile, n-tile)
 *                         tasks from an atomic counter (Weave blog, sections 2.1-2.2):
 *                         up/gate GEMM with SwiGLU in the epilogue, then down GEMM whose
 *                         epilogue applies the router weight to each slot's row
 *   6. combine            per token, the shared row plus its k weighted slot rows, summed
 *                         in slot order (deterministic)
 *
 * Conventions for every entry point below
 *  - Tensors are dense, row-major and contiguous. "bf16" buffers hold IEEE bfloat16 values
 *    as raw 16-bit patterns. Device pointers are CUDA global-memory addresses on the
 *    handle's device; they must be 16-byte aligned (the kernels read them with TMA).
 *  - The caller owns every pointer it passes; the library keeps none of them past the call
 *    (tensor-map descriptors built from weight pointers are cached by address, so a weight
 *    buffer may be reused but not freed and re-allocated at the same address with a
 *    different shape while a handle is alive).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Launches are
 *    asynchronous; a non-zero return means nothing was launched unless stated otherwise.
 *  - Errors: every function returns MOE_OK (0) or a negative MOE_ERR_* code. Device-side
 *    failures (a bounded wait that ran out) are reported by moe_get_status().
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------------------- */
#define MOE_OK                  0
#define MOE_ERR_INVALID_ARG    -1  /* null pointer, bad size, top_k > E, T > max_tokens ... */
#define MOE_ERR_UNSUPPORTED    -2  /* a shape this build cannot run (see moe_init) */
#define MOE_ERR_CUDA           -3  /* a CUDA runtime/driver call failed */
#define MOE_ERR_OUT_OF_MEMORY  -4  /* workspace allocation failed in moe_init */
#define MOE_ERR_MISALIGNED     -5  /* a device pointer is not 16-byte aligned */
#define MOE_ERR_DEVICE_TIMEOUT -6  /* a device-side wait exceeded moe_config.timeout_ns */
#define MOE_ERR_NOT_READY      -7  /* the requested data does not exist yet */

/* ---- moe_config.flags --------------------------------------------------------------- */
#define MOE_FLAG_STAGE_TIMING  1u  /* record CUDA events around each kernel (moe_stage_times) */
#define MOE_FLAG_HOST_STAGING  2u  /* allocate device staging buffers for moe_forward_host */
#define MOE_FLAG_TRACE         4u  /* record per-task claim/finish times (moe_trace_read) */
/* Shape of the expert GEMMs of batches of more than 16 tokens: 128-row m-tiles on single SMs
 * (the default), or with MOE_FLAG_PAIR_TILES 256-row m-tiles on pairs of SMs (2-CTA clusters,
 * tcgen05 cta_group::2; used only when the device fits such clusters). MOE_FLAG_SINGLE_TILES
 * forces single SMs and wins over MOE_FLAG_PAIR_TILES. Both shapes compute the same result. */
#define MOE_FLAG_PAIR_TILES    8u
#define MOE_FLAG_SINGLE_TILES 16u
/* moe_forward / moe_forward_host write `out` as bf16 [T][H] (the fp32 sum rounded to nearest
 * even once) instead of fp32 [T][H]. */
#define MOE_FLAG_OUT_BF16     32u
/* The one-SM expert GEMMs can merge m-tiles of one expert into one task set, computed from the
 * same weight stages: a tile's tail of at most 32 rows inside the tasks of the expert's previous
 * tile (the "tail" shape, MOE_FLAG_TAIL_TILES), or every group of two tiles (the "two-tile"
 * shape, MOE_FLAG_TWO_TILES, below). By default the two-tile shape runs when the mean load per
 * expert is above 96 slots and the capacity allows more than 128, else neither;
 * MOE_FLAG_NO_TAIL_TILES turns the default off (the flags that ask for a shape win over it). All
 * compute the same result. */
#define MOE_FLAG_TAIL_TILES   64u
#define MOE_FLAG_NO_TAIL_TILES 128u
/* Ablation baseline, not for production (the static per-expert SM quota of a fused MoE kernel
 * that the Weave blog, section 1.2, measures against): instead of claiming tasks from the shared
 * counter, each persistent CTA is given a fixed share of the experts at launch — with G CTAs and
 * X = E (+1 for the shared expert), floor(G/X) CTAs per expert and the rest idle, or with
 * X > G the experts c, c+G, ... for CTA c — and works through only its experts' tasks.
 * Single-SM expert GEMMs only (ignored for SM pairs). Same result, slower under skew. */
#define MOE_FLAG_STATIC_QUOTA 256u
/* Allocate the MXFP8 workspace at moe_init (x and h quantised to MXFP8, with their scales), for
 * moe_forward_mxfp8. Needs H, D and D_shared multiples of 128 (else MOE_ERR_UNSUPPORTED). */
#define MOE_FLAG_MXFP8        512u
/* Batches of at most 16 tokens normally run as ONE launch (on devices that allow a cooperative
 * launch of one CTA per SM, and with E <= 256): every CTA computes the router logits of a slice
 * of the experts; once every slice is in, every CTA computes the gating, the align and the task
 * schedule for itself, gathers its share of the x rows, then all claim the expert-GEMM tasks, and
 * the down task that brings in a token's last row of a 256-column block combines that token's
 * block (moe_query 11 reports 1 kernel). The align outputs (moe_debug_outputs) are written as
 * for the separate kernels. MOE_FLAG_UNFUSED_SMALL runs such batches as the six separate kernels
 * instead (for moe_forward and moe_forward_mxfp8). The fused router (fp32 on the CUDA cores) sums
 * each logit in another order than the separate router kernel (fp32 on the tensor cores): logits
 * and gating weights differ in the last bits, and an exact near-tie may go the other way; both
 * are deterministic. */
#define MOE_FLAG_UNFUSED_SMALL 1024u
/* The one-SM expert GEMMs of batches of more than 16 tokens run every group of two m-tiles of one
 * expert as one task set: each task computes both tiles from the same weight stages into the two
 * TMEM accumulators (a 3-stage ring of 64 KB stages; the "two-tile" shape, moe_query 8 reports 5).
 * Wins over MOE_FLAG_TAIL_TILES; the same result. */
#define MOE_FLAG_TWO_TILES    2048u

typedef struct moe_config {
    int32_t hidden;           /* H: model dimension; multiple of 8 */
    int32_t inter;            /* D: routed-expert intermediate dimension; multiple of 8 */
    int32_t inter_shared;     /* D_shared: shared-expert intermediate dimension, 0 = none */
    int32_t num_experts;      /* E: routed experts, 1..1024 */
    int32_t top_k;            /* largest top_k moe_forward will be called with, 1..min(E,32) */
    int32_t block_m;          /* align block size (segment padding), 1..1024 */
    float capacity_factor;    /* 0 = dropless; else C = ceil(cf * T * top_k / E) slots/expert */
    int32_t max_tokens;       /* largest T moe_forward will be called with, >= 1 */
    uint32_t flags;           /* MOE_FLAG_* */
    int32_t device;           /* CUDA device ordinal; -1 = the calling thread's current device */
    int64_t timeout_ns;       /* limit of every device-side wait; <= 0 = 2e9 (2 s) */
    int32_t claim_batch;      /* expert-GEMM tasks a CTA takes per claim on the shared counter,
                               * 0..64 (0 = 1). A CTA runs its batch's consecutive ids in order;
                               * larger batches mean fewer atomics on the counter but coarser load
                               * balance at the end of the queue (the two-level queue of the Weave
                               * blog, section 5.2). Same result for every value. */
} moe_config;

typedef struct moe_handle moe_handle;

/* Shared-expert weights (device, bf16): up [D_shared][H], gate [D_shared][H],
 * down [H][D_shared]. */
typedef struct moe_shared_w {
    const void *up;
    const void *gate;
    const void *down;
} moe_shared_w;

/* Create a handle: validates `cfg`, selects the device, allocates and owns the whole
 * workspace (router logits, top-k ids/weights, histograms, sorted_ids, expert_ids, tile and
 * task tables, the bf16 intermediate SwiGLU activations h, counters and status word; plus the
 * staging buffers when MOE_FLAG_HOST_STAGING is set), and queries the SM count.
 * Intermediate-cache pre-allocation follows the vLLM execution analysis ("Memory allocation
 * per step": allocate once, reuse across calls); moe_forward never allocates.
 * On success *out receives the handle. Returns MOE_ERR_INVALID_ARG for a bad cfg,
 * MOE_ERR_OUT_OF_MEMORY / MOE_ERR_CUDA for allocation or device failures. */
MOE_API int moe_init(const moe_config *cfg, moe_handle **out);

/* Release the workspace and the handle (synchronises the handle's device first). NULL is
 * allowed. */
MOE_API void moe_destroy(moe_handle *h);

/* One layer forward (Mixture-of-Kittens layer equation; top-k softmax gating renormalised
 * over the selected experts; moe_align_block_size-style sort padded to cfg.block_m;
 * dropless unless cfg.capacity_factor > 0, in which case a slot whose rank inside its
 * expert, in ascending slot order s = t*top_k + j, is >= C is dropped and contributes 0).
 *   x           device bf16 [T][H] (may be NULL when T == 0)
 *   T           0..cfg.max_tokens
 *   w_router    device bf16 [E][H]
 *   router_bias device fp32 [E], added to the logits before selection and softmax; nullable
 *   w_up,w_gate device bf16 [E][D][H]
 *   w_down      device bf16 [E][H][D]
 *   w_shared    nullable; required (all three non-null) iff cfg.inter_shared > 0
 *   top_k       1..cfg.top_k
 *   out         device fp32 [T][H], or bf16 [T][H] with MOE_FLAG_OUT_BF16; fully overwritten
 *               with x' (may be NULL when T == 0)
 * Asynchronous on `stream`; no host synchronisation, so it may be captured in a CUDA graph
 * once the handle's tensor-map cache holds the weight pointers. */
MOE_API int moe_forward(moe_handle *h, const void *x, int32_t T, const void *w_router,
                const float *router_bias, const void *w_up, const void *w_gate,
                const void *w_down, const moe_shared_w *w_shared, int32_t top_k, void *out,
                void *stream);

/* moe_forward with HOST activations: copies x_host (bf16 [T][H], pinned host memory for
 * full speed) to a device staging buffer, runs the forward, copies the result to out_host
 * (fp32 [T][H], or bf16 with MOE_FLAG_OUT_BF16) and synchronises `stream`. Weights stay device pointers. Needs
 * MOE_FLAG_HOST_STAGING at moe_init (else MOE_ERR_NOT_READY). */
MOE_API int moe_forward_host(moe_handle *h, const void *x_host, int32_t T, const void *w_router,
                     const float *router_bias, const void *w_up, const void *w_gate,
                     const void *w_down, const moe_shared_w *w_shared, int32_t top_k,
                     void *out_host, void *stream);

/* moe_forward_host without the synchronisation, for a caller that feeds batches back to back:
 * consecutive calls pipeline, so that the copy of call i+1's x to the device and the copy of
 * call i-1's result to the host overlap call i's forward (two device staging slots, two copy
 * streams of the handle, ordered by events; the forwards themselves run in order on `stream`).
 * Returns once the work is queued. x_host and out_host (pinned for the copies to overlap) must
 * stay valid and x_host unchanged until moe_forward_host_join has returned; a call's result is
 * in out_host from then on. Needs MOE_FLAG_HOST_STAGING (else MOE_ERR_NOT_READY). */
MOE_API int moe_forward_host_async(moe_handle *h, const void *x_host, int32_t T, const void *w_router,
                                   const float *router_bias, const void *w_up, const void *w_gate,
                                   const void *w_down, const moe_shared_w *w_shared, int32_t top_k,
                                   void *out_host, void *stream);

/* ---- MXFP8 experts ------------------------------------------------------------------------
 * The pages name MXFP8 expert weights (Mixture-of-Kittens blog, introduction; FlashMoE review,
 * "future directions": FP8 and lower precisions) without defining the format. It is read as the
 * OCP Microscaling format MXFP8: E4M3 elements (exponent bias 7, largest value 448, no
 * infinity) in blocks of 32 consecutive elements along the contraction dimension, each block
 * with one E8M0 scale 2^(floor(log2 amax) - 8) (scale code = exponent + 127, 0 for a block of
 * zeros); an element is v / scale rounded to nearest even and clamped to +-448.
 * A quantised matrix [R][K] (R and K multiples of 128) is a pair of device buffers, both
 * 16-byte aligned and owned by the caller:
 *   q       E4M3 codes, uint8 [R][K], row-major
 *   scales  E8M0 codes in 512-byte atoms, moe_mxfp8_scale_bytes(R, K) bytes in all: atom
 *           (r / 128) * (K / 128) + b / 4 holds the scale of row r, block b (columns 32b ..
 *           32b + 31) at byte (r % 32) * 16 + ((r / 32) % 4) * 4 + b % 4.
 */
typedef struct moe_mxfp8_mat {
    const void *q;
    const void *scales;
} moe_mxfp8_mat;

/* The experts of moe_forward_mxfp8, each a quantised matrix: up and gate [E*D][H] (the bf16
 * [E][D][H] tensors viewed as [E*D][H]), down [E*H][D]; the shared expert's [D_shared][H],
 * [D_shared][H] and [H][D_shared] (ignored when D_shared == 0). */
typedef struct moe_mxfp8_experts {
    moe_mxfp8_mat up, gate, down;
    moe_mxfp8_mat shared_up, shared_gate, shared_down;
} moe_mxfp8_experts;

/* Bytes of the scale array of an [rows][cols] quantised matrix: rows * cols / 32; -1 unless
 * both are positive multiples of 128. */
MOE_API int64_t moe_mxfp8_scale_bytes(int64_t rows, int64_t cols);

/* Quantise the device bf16 matrix src [rows][cols] to MXFP8, writing q [rows][cols] and its
 * scales (layout above), asynchronously on `stream`. rows and cols positive multiples of 128
 * (else MOE_ERR_UNSUPPORTED); pointers 16-byte aligned (else MOE_ERR_MISALIGNED). Any handle
 * works (MOE_FLAG_MXFP8 is not needed); nothing is kept. */
MOE_API int moe_quantize_mxfp8(moe_handle *h, const void *src, int64_t rows, int64_t cols, void *q,
                               void *scales, void *stream);

/* moe_forward with MXFP8 experts. The router projection and gating run on the bf16 x and
 * W_router exactly as in moe_forward; then each token's x row is quantised to MXFP8 (blocks
 * along H), the expert GEMMs read the quantised weights `w`, h = SwiGLU(W_up x, W_gate x) is
 * computed in fp32 and quantised to MXFP8 (blocks along D) before the down projection, and the
 * router-weighted rows are combined as in moe_forward (fp32 sums; `out` fp32 [T][H], or bf16
 * with MOE_FLAG_OUT_BF16). x, w_router, router_bias, top_k, out and stream as in moe_forward.
 * The expert GEMMs run on single SMs with 128-row tiles and the atomic task counter
 * (MOE_FLAG_PAIR_TILES, MOE_FLAG_TAIL_TILES, MOE_FLAG_TWO_TILES and MOE_FLAG_STATIC_QUOTA do not
 * apply; moe_query 8 reports 4). A batch of at most 16 tokens runs as one fused launch as in
 * moe_forward (MOE_FLAG_UNFUSED_SMALL: the separate kernels), its row gather quantising the x
 * rows. Needs MOE_FLAG_MXFP8 at moe_init (else MOE_ERR_NOT_READY). Asynchronous, no host
 * synchronisation, no allocation. */
MOE_API int moe_forward_mxfp8(moe_handle *h, const void *x, int32_t T, const void *w_router,
                              const float *router_bias, const moe_mxfp8_experts *w, int32_t top_k,
                              void *out, void *stream);

/* Makes `stream` wait for every copy back queued by moe_forward_host_async on this handle; with
 * `block` non-zero the host also waits for them. */
MOE_API int moe_forward_host_join(moe_handle *h, void *stream, int32_t block);

/* Synchronise the handle's last stream and report the device status word:
 * *device_status = 0 when every kernel since the last call finished normally, else a
 * device error code (bit 30 set, low bits naming the wait that ran out). The word is
 * cleared by this call. Returns MOE_ERR_DEVICE_TIMEOUT if a wait ran out, MOE_ERR_CUDA if
 * the stream reported a CUDA error, else MOE_OK. */
MOE_API int moe_get_status(moe_handle *h, int32_t *device_status);

/* Stage entry points (each is one step of moe_forward, callable on its own).
 *
 * moe_router_logits: logits (device fp32 [T][E]) = x W_router^T (+ bias). */
MOE_API int moe_router_logits(moe_handle *h, const void *x, int32_t T, const void *w_router,
                      const float *router_bias, float *logits, void *stream);

/* moe_gate_topk: per token, the top_k largest logits (ties to the lower expert index) in
 * descending order, and weights softmax(logits)[id] renormalised over the selected set.
 * logits device fp32 [T][E]; topk_ids device int32 [T][top_k]; topk_w device fp32
 * [T][top_k]. (Weave blog section 1.1; vLLM execution analysis, topk_softmax.) */
MOE_API int moe_gate_topk(moe_handle *h, const float *logits, int32_t T, int32_t top_k,
                  int32_t *topk_ids, float *topk_w, void *stream);

/* moe_align_block_size: from topk_ids (device int32 [T][top_k]) write
 *   sorted_ids      device int32 [moe_sorted_len(h, T, top_k)]: slot ids s = t*top_k + j
 *                   grouped by expert, ascending s inside an expert, each expert segment
 *                   padded with the sentinel T*top_k to a multiple of cfg.block_m; entries
 *                   from num_post_padded on are the sentinel
 *   expert_ids      device int32 [moe_blocks_len(h, T, top_k)]: expert of each block,
 *                   -1 past the last block
 *   num_post_padded device int32 [1]: total padded length P
 * with cfg.capacity_factor applied as in moe_forward. Expert ids outside [0, E) are
 * invalid input. (vLLM PR #53280 summary, implementation breakdown; all-blocks variant.) */
MOE_API int moe_align_block_size(moe_handle *h, const int32_t *topk_ids, int32_t T, int32_t top_k,
                         int32_t *sorted_ids, int32_t *expert_ids, int32_t *num_post_padded,
                         void *stream);

/* Buffer lengths of moe_align_block_size: T*top_k + E*(block_m-1) and
 * ceil(that / block_m). Return -1 for a NULL handle or negative sizes. */
MOE_API int64_t moe_sorted_len(const moe_handle *h, int32_t T, int32_t top_k);
MOE_API int64_t moe_blocks_len(const moe_handle *h, int32_t T, int32_t top_k);

/* Copy the intermediates of the most recent moe_forward on `stream` into caller device
 * buffers (each nullable): logits fp32 [T][E], topk_ids int32 [T][k], topk_w fp32 [T][k],
 * sorted_ids int32 [moe_sorted_len], expert_ids int32 [moe_blocks_len], num_post_padded
 * int32 [1]. Returns MOE_ERR_NOT_READY before the first forward. */
MOE_API int moe_debug_outputs(moe_handle *h, float *logits, int32_t *topk_ids, float *topk_w,
                      int32_t *sorted_ids, int32_t *expert_ids, int32_t *num_post_padded,
                      void *stream);

/* Copy the expert GEMMs' per-row results of the most recent forward on `stream` into caller
 * device buffers (each nullable), for checking the layer stage by stage:
 *   h_rows            bf16 [moe_query 9][moe_query 10]: SwiGLU(W_up^e x_t, W_gate^e x_t) of
 *                     every GEMM row (the up/gate GEMM's output; bf16 experts only: after
 *                     moe_forward_mxfp8, h_rows must be NULL, else MOE_ERR_NOT_READY)
 *   y_rows            bf16 [moe_query 9][H]: w_s * W_down^e h of every row (the down GEMM's
 *                     output, router weight applied; weight 1 for shared-expert rows)
 *   row_of_slot       int32 [T][k]: the GEMM row of slot s = t*k + j, or -1 if it was dropped
 *   num_routed_tiles  int32 [1]: M_r, the routed experts' m-tiles; the shared expert's tile i
 *                     (tokens i*tile_m ...) follows at rows (M_r + i) * tile_m (moe_query 6)
 * Rows are grouped in m-tiles of moe_query 6 rows; rows past a tile's valid rows hold no
 * result. (Layer equation of the Mixture-of-Kittens blog, its two GEMMs taken one by one.)
 * Returns MOE_ERR_NOT_READY before the first forward. */
MOE_API int moe_debug_expert_rows(moe_handle *h, void *h_rows, void *y_rows, int32_t *row_of_slot,
                                  int32_t *num_routed_tiles, void *stream);

/* Mean durations in milliseconds of the kernels of the forwards recorded since the previous
 * call (the first 256 of them; needs MOE_FLAG_STAGE_TIMING; synchronises, then starts a new
 * recording window): ms[0] router, ms[1] gating, ms[2] align scatter, ms[3] row gather,
 * ms[4] expert GEMMs, ms[5] combine. n = entries of ms (up to 6). Each duration is measured
 * with CUDA events recorded on the forward's stream around the kernel; a fused small batch
 * (one launch) is timed whole in ms[4], with 0 in the others. MOE_ERR_NOT_READY when nothing
 * was recorded. */
MOE_API int moe_stage_times(moe_handle *h, float *ms, int32_t n);

/* Handle facts: which = 0 SM count, 1 workers of the last forward's expert GEMMs (CTAs on
 * single SMs, or SM pairs; the SM count before any forward), 2 workspace bytes,
 * 3 tasks of the last forward (synchronises), 4 m-tiles of the last forward (synchronises),
 * 5 dependency lag (units) of the last forward, 6 rows per m-tile of the last forward
 * (128 or 256), 7 SM pairs the device can run at once for the pair shape (0 = none),
 * 8 expert-GEMM shape of the last forward (0 general, 1 small-tile, 2 tail, 3 SM pairs,
 * 4 MXFP8, 5 two-tile), 9 rows of the per-row buffers of moe_debug_expert_rows, 10 their h row stride
 * (elements, max(D, D_shared)), 11 kernels the last forward launched (1 for a fused small
 * batch, else 6), 12 whether batches of at most 16 tokens run fused on this handle (1) or not
 * (for moe_forward_mxfp8 on a handle made with MOE_FLAG_MXFP8, else for moe_forward). */
MOE_API int moe_query(const moe_handle *h, int32_t which, int64_t *value);

/* Per-task trace of the last forward (needs MOE_FLAG_TRACE; synchronises). Fills up to
 * `cap` records of 4 int64 each: {cta, task, t_claim_ns, t_done_ns} (device globaltimer),
 * sets *n to the records written. */
MOE_API int moe_trace_read(moe_handle *h, int64_t *records, int64_t cap, int64_t *n);

/* Wait accounting of the last forward's expert-GEMM kernel, bf16 or MXFP8 (needs MOE_FLAG_TRACE;
 * synchronises): per CTA (row) int64 %globaltimer ns summed over its tasks --
 *   0 producer waiting for a free operand stage     1 producer waiting for a down task's up
 *   2 producer waiting for a free task-ring entry      tasks (fused: for a tile's gathered rows)
 *   3 producer claiming and decoding tasks           4 MMA lane waiting for a filled stage
 *   5 MMA lane waiting for a free accumulator        6 MMA lane waiting for the next task
 *   7 epilogue waiting for the next task             8 epilogue waiting for a finished accumulator
 *   9 / 10 / 11 the producer / MMA / epilogue loop durations;
 * and for a fused small batch: 12 the CTA's router slice, 13 the arrival and the CTA's own
 * schedule, 14 its share of the row gather, 15 1 for CTA 0 (which also writes the align
 * outputs), 16 from the start of the front to the end of the epilogue loop, the schedule's
 * steps: 17 waiting for every CTA's router slice, 18 loading the logits, 19 gating, 20 the
 * count / offset / tile / unit tables, 21 the CTA's schedule in shared memory, 22 (CTA 0) the
 * align and tile outputs for the host; 23 the barrier,
 * per-token counters and combines after each fused down task, 24 the same for the tasks that
 * combined at least one token.
 * (25 per row.) Writes up to `rows` rows (at most one per SM) into the host buffer
 * `waits` and their number to *n_rows. The SM-pair and MXFP8 kernels leave zeros. */
MOE_API int moe_trace_waits(moe_handle *h, int64_t *waits, int32_t rows, int32_t *n_rows);

/* Testing hook: when `extra` > 0, the down-projection tasks of the next moe_forward wait
 * for `extra` more up-projection completions than can ever arrive, so their bounded wait
 * runs out after cfg.timeout_ns and the forward reports MOE_ERR_DEVICE_TIMEOUT through
 * moe_get_status. The hook clears itself after one forward. */
MOE_API int moe_debug_inject_stall(moe_handle *h, int32_t extra);

/* Allocation-free variant of moe_align_block_size. The pages have no counterpart: this entry
 * exists for callers that cannot let this library allocate device memory, such as a serving
 * runtime that owns all of HBM through its own allocator, or a latency-critical path that
 * cannot afford a cudaMalloc (which may synchronise the device). It needs no handle and never
 * allocates: the kernels' scratch memory is a fixed array of about 68 KB compiled into the
 * library, which every GPU that loads the library keeps until the process exits.
 *   topk_ids        device int32 [T][top_k], expert ids in [0, num_experts)
 *   num_experts     1..256;  T * top_k <= 131072  (larger: MOE_ERR_UNSUPPORTED)
 *   block_m, capacity_factor   as moe_config.block_m / capacity_factor
 *   sorted_ids      device int32 [T*top_k + num_experts*(block_m-1)]
 *   expert_ids      device int32 [ceil(that / block_m)]
 *   num_post_padded device int32 [1]
 * Outputs are those of moe_align_block_size for the same arguments. The first call on each
 * device looks up the array's device address and the SM count on the calling thread's current
 * device; make that first call before any stream capture. The look-up is repeated, on the next
 * call, when the device's context has changed since (after a cudaDeviceReset). Every call uses
 * the same array: each call clears what it needs, but calls whose work overlaps on the GPU
 * (different streams, or different host threads without ordering) race on it and must be
 * serialised by the caller. T = 0 is allowed (topk_ids may then be NULL): every sorted_ids
 * entry is the sentinel 0, every expert_ids entry -1, and num_post_padded 0. */
MOE_API int moe_align_block_size_noalloc(const int32_t *topk_ids, int32_t T, int32_t top_k,
                                         int32_t num_experts, int32_t block_m,
                                         float capacity_factor, int32_t *sorted_ids,
                                         int32_t *expert_ids, int32_t *num_post_padded,
                                         void *stream);

/* Human-readable name of a MOE_* status code. */
MOE_API const char *moe_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
