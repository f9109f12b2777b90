/*
 * moe.h -- C ABI of libmoe.so, a fused Mixture-of-Experts forward for NVIDIA
 * B200 (sm_100a).
 *
 * The function computed is the one defined on the pages this library
 * restates:
 *   - "tpu_inference/kernels/fused_moe/v1/kernel.py" (tpu-inference), ref_moe:
 *     softmax over router logits, top-k expert choice (optionally
 *     renormalised, 0.13.2 version of that page), a SwiGLU expert FFN per
 *     (token, chosen expert), and the top-k-weighted sum;
 *   - atrex-bench operator #009 "fused_moe", reference.py Model.forward and
 *     input.py: the weight layout used here (w1 [E, 2I, H], rows 0..I-1
 *     gate and I..2I-1 up; w2 [E, H, I]), fp32 top-k weights, int32 ids and
 *     an fp32 [T, H] output.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device,
 *     owned by the caller, dense and row-major.  bf16 tensors are passed as
 *     uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  No call
 *     synchronises the stream unless its comment says so; results are ready
 *     when the stream's work completes.
 *   - Return value: MOE_OK (0) or a negative MOE_ERR_* code.  Nothing is
 *     launched when an argument check fails.  No call throws.
 *   - The library owns a grow-only device workspace per device (routing
 *     permutation, the bf16 SwiGLU intermediate, per-(token, slot) expert
 *     outputs).  It grows on the first call that needs more; that call
 *     allocates (and synchronises the device if it frees a smaller one).
 *     Calls on two different streams of one device must not overlap in time
 *     (they share that workspace).
 *   - Two kernels expect all of their CTAs on the GPU at once: the
 *     small-batch kernel (a cooperative launch, which the runtime only
 *     starts when every CTA fits) and, for top-k <= 2 with at most about
 *     twelve waves of tiles, the grouped GEMM that runs both projections in
 *     one launch (its second-projection tiles wait for first-projection
 *     tiles of other CTAs).  Work that another stream keeps on the SMs while
 *     that GEMM runs -- a persistent kernel such as a running collective --
 *     can hold some of its CTAs back; its waits then give up after the wait
 *     limit (moe_set_wait_limit_ns, 2 s by default), out is invalid and
 *     MOE_STATUS_TIMEOUT is raised.  Order such work before or after the
 *     call on the stream.
 */
#ifndef MOE_H
#define MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG -1 /* null pointer, negative size, k outside [1, E] */
#define MOE_ERR_UNSUPPORTED -2 /* shape this build does not handle (see each call) */
#define MOE_ERR_CUDA -3        /* a CUDA runtime/driver call or a launch failed */
#define MOE_ERR_TIMEOUT -4     /* a bounded device-side wait expired */
#define MOE_ERR_NO_DEVICE -5   /* no usable sm_100 device is current */
#define MOE_ERR_OOM -6         /* workspace allocation failed */
#define MOE_ERR_SCRATCH_LIMIT -7 /* request larger than the fixed scratch of moe_forward_small_noalloc */

/* Bits of the device status word (moe_get_device_status). */
#define MOE_STATUS_TIMEOUT 0x1u  /* a pipeline wait gave up; that launch's output is invalid */
#define MOE_STATUS_BAD_ID 0x2u   /* moe_forward met an expert id outside [0, E) and skipped it */

/*
 * moe_route -- router softmax, top-k choice and optional renormalisation.
 * Pages: ref_moe (softmax over the experts, lax.top_k), its 0.13.2 version
 * (renormalize_topk_logits divides the k weights by their sum), and the
 * in-kernel top-k of the same file (an argmax that returns the lowest index
 * among equal values).
 *
 *   logits        [T, E] fp32, read only.
 *   topk_ids      [T, k] int32, written: the k experts with the largest
 *                 logits, largest first; equal logits go to the lower index.
 *   topk_weights  [T, k] fp32, written: p_id = exp(l_id - max) / sum exp(l - max)
 *                 and, when renorm != 0, divided by the sum of the k values.
 * Errors: INVALID_ARG for null pointers, T < 0, E < 1, k < 1 or k > E;
 *         UNSUPPORTED for E > 1024.  T == 0 launches nothing.
 * Logits may be -inf (probability 0; such experts fill leftover slots lowest
 * index first).  Rows that are all -inf or contain NaN are undefined.
 */
int moe_route(const float *logits, int64_t T, int E, int k, int renorm,
              int32_t *topk_ids, float *topk_weights, void *stream);

/*
 * moe_forward -- the expert FFNs and the weighted combine.
 * Pages: ref_moe (per token: x.[W_gate | W_up] -> silu(gate) * up -> .W2,
 * then sum_j w_j y_j); atrex-bench #009 Model.forward (same result written
 * as a loop over experts; a token routed twice to one expert gets the summed
 * weight; ids outside [0, E) never match an expert).
 *
 *   hidden        [T, H] bf16
 *   w1            [E, 2I, H] bf16; rows 0..I-1 of w1[e] are the gate
 *                 projection, rows I..2I-1 the up projection (x . w1[e]^T)
 *   w2            [E, H, I] bf16 (act . w2[e]^T)
 *   topk_weights  [T, k] fp32
 *   topk_ids      [T, k] int32; ids outside [0, E) are skipped and flagged
 *                 with MOE_STATUS_BAD_ID in the device status word
 *   out           [T, H] fp32, every element overwritten:
 *                 out[t] = sum over j = 0..k-1 of
 *                          topk_weights[t, j] * FFN_{topk_ids[t, j]}(hidden[t]),
 *                 accumulated in fp32 (grouped-GEMM path, k <= 2: out is
 *                 zeroed and each rounded product w_j * y_j is added at L2,
 *                 which gives the same bits in either order; k > 2 and the
 *                 small-T path: ascending j, one fused multiply-add per
 *                 term, acc = fma(w_j, y_j, acc) from acc = 0); a row with
 *                 no valid id is 0.
 * Numerics: bf16 inputs, fp32 accumulation; the SwiGLU intermediate is
 * rounded to bf16 before the second projection on both paths (grouped
 * GEMMs, and the small-T path: T <= the small-T limit, H <= 4096 and
 * I <= 12288).  The combine is deterministic: repeated calls give
 * identical bits.
 * hidden, w1, w2 and out must start on a 16-byte boundary.
 * Errors: INVALID_ARG for null pointers, hidden/w1/w2/out not 16-byte
 *         aligned, T < 0, H/I/E < 1, k < 1 or k > E;
 *         UNSUPPORTED unless H % 128 == 0 and I % 128 == 0 (the alignment
 *         the TPU page also demands), E <= 1024 and k <= 16;
 *         OOM if the workspace cannot grow.  T == 0 launches nothing.
 */
int moe_forward(const uint16_t *hidden, const uint16_t *w1, const uint16_t *w2,
                const float *topk_weights, const int32_t *topk_ids, float *out,
                int64_t T, int H, int I, int E, int k, void *stream);

/*
 * moe_forward_ex -- moe_forward with the expert-FFN variants of the 0.13.2
 * version of the TPU page: its activation_fn choice and the optional
 * per-expert biases that ref_moe adds to both projections.
 *
 *   b1    [E, 2I] fp32 or NULL; b1[e, 0..I-1] is added to the gate
 *         projection and b1[e, I..2I-1] to the up projection, before the
 *         activation
 *   b2    [E, H] fp32 or NULL; added to the expert's output, so it is
 *         scaled by the top-k weight like the rest of that output
 *   act   MOE_ACT_SILU:      silu(gate) * up (what moe_forward computes)
 *         MOE_ACT_GELU_TANH: gelu(gate) * up, gelu in its tanh form
 *                            0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3)))
 *         MOE_ACT_SWIGLUOAI: (clip(up, -7, 7) + 1) * g * sigmoid(1.702 g)
 *                            with g = min(gate, 7)
 * Everything else (arguments, layouts, numerics, paths, determinism) is as
 * in moe_forward, which equals moe_forward_ex(..., NULL, NULL,
 * MOE_ACT_SILU, ...).  b1 and b2 must start on a 16-byte boundary.
 * Errors: those of moe_forward, plus INVALID_ARG for an unknown act or an
 *         unaligned b1/b2.
 */
#define MOE_ACT_SILU 0
#define MOE_ACT_GELU_TANH 1
#define MOE_ACT_SWIGLUOAI 2
int moe_forward_ex(const uint16_t *hidden, const uint16_t *w1, const uint16_t *w2,
                   const float *b1, const float *b2, int act,
                   const float *topk_weights, const int32_t *topk_ids, float *out,
                   int64_t T, int H, int I, int E, int k, void *stream);

/*
 * moe_forward_fp8 -- moe_forward on sub-channel-quantised expert weights.
 * Page: the 0.13.2 version of the TPU page (ref_moe with w1_scale,
 * w2_scale and subc_quant_wsz): every weight is its code times the fp32
 * scale of its block of `block` consecutive contraction elements.
 *
 *   w1        [E, 2I, H] FP8 E4M3 codes (OCP "e4m3fn", one byte each), rows
 *             as in moe_forward (gate rows, then up rows)
 *   w1_scale  [E, 2I, H / block] fp32: scale of row r, columns
 *             b*block .. b*block + block - 1 (the page's w1_scale
 *             [E, 2, H / block, 1, I] transposed to this row layout)
 *   w2        [E, H, I] FP8 E4M3 codes
 *   w2_scale  [E, H, I / block] fp32
 *   block     a multiple of 128 that divides H and I (the page demands a
 *             multiple of 256)
 * Activation silu, no biases; other arguments, the output and the error
 * codes are those of moe_forward, plus UNSUPPORTED for a block that is not
 * a multiple of 128 or does not divide H and I, and INVALID_ARG for null
 * scales or block < 1.
 * Numerics: the small-T path (T <= the small-T limit) streams the codes and
 * multiplies each 16-weight partial dot product (fp32) by its scale; the
 * grouped-GEMM path first expands the chosen experts' weights to bf16
 * (bf16_rn(code * scale), one rounding) into a second library-owned
 * grow-only buffer of E * 3 * H * I * 2 bytes, then runs as moe_forward.
 */
int moe_forward_fp8(const uint16_t *hidden, const uint8_t *w1, const float *w1_scale,
                    const uint8_t *w2, const float *w2_scale, int block,
                    const float *topk_weights, const int32_t *topk_ids, float *out,
                    int64_t T, int H, int I, int E, int k, void *stream);

/*
 * moe_forward_small_noalloc -- the small-batch path of moe_forward (the two
 * GEMV kernels) in a form that never allocates device memory.  The pages
 * have no counterpart: it exists for callers that cannot allocate once they
 * are running, such as a serving runtime that reserves all of its device
 * memory at start-up, or a decode loop that must not pay the device-wide
 * synchronisation of cudaFree when a workspace grows.
 *
 * Arguments, layouts, numerics and the result are those of moe_forward on
 * its small-T path (bf16 SwiGLU intermediate, fixed-order fp32 combine).
 * Its only scratch is a fixed __device__ array of this library:
 * 256 bytes + MOE_NOALLOC_MAX_ACT fp32-sized values (1 MiB; the bf16
 * intermediate uses half of it), which every GPU that loads the library
 * holds until the process exits.
 *   - Limits: T <= MOE_NOALLOC_MAX_T and T*k*I <= MOE_NOALLOC_MAX_ACT, else
 *     MOE_ERR_SCRATCH_LIMIT and nothing is launched.  Other checks and
 *     codes as in moe_forward, plus UNSUPPORTED when H > 4096 or I > 12288
 *     (the largest rows the small-T kernels stage) or when the shape's
 *     token vectors and per-CTA buffers do not fit the kernel's shared
 *     memory on this device.
 *   - The first call on each device, with that device current, looks up
 *     the array's device address (cudaGetSymbolAddress, a host-side runtime
 *     query) and caches it for later calls.  cudaDeviceReset between calls
 *     is not supported (the cached address would be stale).
 *   - All calls share the one array, which keeps the last call's contents.
 *     Nothing in it has to be cleared between calls: every act value is
 *     written before it is read in the same call, and the grid-barrier
 *     counter in the array only ever advances by whole grids.  Calls whose
 *     kernels overlap on the GPU (e.g. on two streams without ordering)
 *     race on it: they mix each other's act values, and their CTAs count
 *     towards each other's grid barrier, which can open a barrier early
 *     (wrong output) or hold one until its 2 s limit (output unwritten).
 *   - Failures on the device are not reported: expert ids outside [0, E)
 *     are skipped as in moe_forward but flag nothing, and a grid-barrier or
 *     copy wait that gives up after its 2 s limit leaves out unwritten
 *     while the call has already returned MOE_OK.  moe_get_device_status
 *     does not see this path's status word.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define MOE_NOALLOC_MAX_T 16
#define MOE_NOALLOC_MAX_ACT 262144
int moe_forward_small_noalloc(const uint16_t *hidden, const uint16_t *w1, const uint16_t *w2,
                              const float *topk_weights, const int32_t *topk_ids, float *out,
                              int64_t T, int H, int I, int E, int k, void *stream);

/*
 * moe_permute -- the expert grouping that moe_forward uses internally,
 * exported so that it can be checked bit for bit: it runs the same grouping
 * kernel that moe_forward runs for this many entries (one kernel up to 8192
 * entries, a histogram / scan / scatter sequence above).  Pages: the TPU
 * kernel hands each expert its rows in (token, k) order
 * (start_a2a_scatter); Model.forward visits each expert's tokens in
 * ascending order.
 *
 *   topk_ids        [T, k] int32 (flat index i = t*k + j)
 *   sorted_rows     [T*k] int32, written for positions < expert_offsets[E]:
 *                   the flat indices grouped by expert, ascending within an
 *                   expert (a stable counting sort); later positions are
 *                   left untouched
 *   expert_offsets  [E+1] int32, written: exclusive prefix sum of the
 *                   per-expert counts; expert_offsets[E] = number of ids in
 *                   [0, E)
 * Ids outside [0, E) are left out; unlike moe_forward, neither call raises
 * MOE_STATUS_BAD_ID.
 * Errors: INVALID_ARG for null pointers, T < 0, k < 1, E < 1;
 *         UNSUPPORTED for E > 1024.
 */
int moe_permute(const int32_t *topk_ids, int64_t T, int k, int E,
                int32_t *sorted_rows, int32_t *expert_offsets, void *stream);

/*
 * moe_permute_ex -- moe_permute with everything the grouping stage of
 * moe_forward produces, and a choice of grouping kernel (debug and test
 * export).
 *
 *   inv     [T*k] int32 or NULL; written: inv[i] = the position of flat
 *           index i in sorted_rows, or -1 when topk_ids[i] is outside [0, E)
 *   hidden  [T, H] bf16 and xs [T*k, H] bf16, both NULL or both given
 *           (16-byte aligned, H % 128 == 0): xs[r] = hidden[sorted_rows[r] / k]
 *           for r < expert_offsets[E], the expert-sorted copy of the hidden
 *           rows that moe_forward makes for top-k <= 2; later rows untouched
 *   kernel  MOE_PERMUTE_AUTO: the kernel moe_forward uses for T*k entries;
 *           MOE_PERMUTE_SINGLE: the one-kernel grouping (T*k <= 8192, else
 *           UNSUPPORTED); MOE_PERMUTE_MULTI: histogram / scan / scatter
 * Both kernels give identical results.  Errors: those of moe_permute, plus
 * INVALID_ARG for an unknown kernel, only one of hidden / xs, or an
 * unaligned hidden / xs.
 */
#define MOE_PERMUTE_AUTO 0
#define MOE_PERMUTE_SINGLE 1
#define MOE_PERMUTE_MULTI 2
int moe_permute_ex(const int32_t *topk_ids, int64_t T, int k, int E,
                   int32_t *sorted_rows, int32_t *expert_offsets, int32_t *inv,
                   const uint16_t *hidden, int H, uint16_t *xs, int kernel, void *stream);

/*
 * Expert parallelism (EP) over `world` ranks, one per GPU: rank r owns the
 * experts [r * E / world, (r + 1) * E / world) (w1 / w2 hold only those
 * E / world experts on each rank) and routes its own tokens.  A forward is
 *   1. moe_ep_dispatch_plan: the send order (the (token, slot) rows grouped
 *      by owner rank) and its per-rank counts;
 *   2. an exchange of the counts (every rank learns where its rows land in
 *      every receiver's buffer);
 *   3. moe_ep_pack: the hidden rows and local expert ids, stored straight
 *      into the receivers' buffers;
 *   4. moe_forward on the received rows with top-k 1 and weight 1 (each row
 *      its own expert's FFN output);
 *   5. moe_ep_return: each output row stored straight into its sender's
 *      buffer;
 *   6. moe_ep_combine: out[t] = sum over j in ascending order of
 *      w[t, j] * y[t, j], fp32.
 * Pages: the TPU kernel's expert-parallel structure (all_reduce_metadata of
 * the per-device expert counts, start_a2a_scatter, the expert FFNs,
 * start_a2a_gather back to the token owner, the fixed-order bt_acc sum) and
 * the 0.13.2 version's fused_ep_moe wrapper (a shard_map over the expert
 * axis).  Steps 2 and the synchronisation between ranks are the caller's
 * (the Python package's ep module does them with torch.distributed).  The
 * destination buffers may be another GPU's memory mapped into this one: the
 * copies only store to them.
 */

/*
 * moe_ep_dispatch_plan -- the send order of this rank's (token, slot) rows.
 *   topk_ids      [T, k] int32 (global expert ids)
 *   send_rows     [T*k] int32, written for positions < send_offsets[world]:
 *                 flat indices t*k + j grouped by owner rank, ascending
 *                 within a rank
 *   send_offsets  [world+1] int32, written: exclusive prefix sum of the rows
 *                 sent to each rank
 *   inv           [T*k] int32, written: the position of flat index i in
 *                 send_rows, -1 for an id outside [0, E) (flagged with
 *                 MOE_STATUS_BAD_ID)
 * Errors: INVALID_ARG for null pointers, T < 0, k outside [1, E], world < 1;
 *         UNSUPPORTED for E > 1024, world > 64 or E % world != 0.
 */
int moe_ep_dispatch_plan(const int32_t *topk_ids, int64_t T, int k, int E, int world,
                         int32_t *send_rows, int32_t *send_offsets, int32_t *inv,
                         void *stream);

/*
 * moe_ep_pack -- row r of the send order (destination d: the segment of
 * send_offsets it falls in) is stored as row dst_row0[d] + r -
 * send_offsets[d] of d's buffers: dst_x[d] [rows, H] bf16 gets the hidden
 * row of its token, dst_eid[d] [rows] int32 its expert id minus d * E / world.
 *   send_offsets, dst_row0  HOST arrays of world + 1 and world int64 values
 *   dst_x, dst_eid          HOST arrays of world DEVICE pointers (16-byte
 *                           aligned; unused, and may be NULL, for a rank
 *                           that receives no rows)
 * Errors: INVALID_ARG for null pointers, offsets that are not a prefix sum
 *         starting at 0 or exceed T*k, negative rows, unaligned buffers;
 *         UNSUPPORTED for H % 128 != 0, world > 64 or E % world != 0.
 */
int moe_ep_pack(const uint16_t *hidden, int H, const int32_t *topk_ids, int64_t T, int k, int E,
                int world, const int32_t *send_rows, const int64_t *send_offsets,
                uint16_t *const *dst_x, int32_t *const *dst_eid, const int64_t *dst_row0,
                void *stream);

/*
 * moe_ep_return -- received row q (source s: the segment of recv_offsets it
 * falls in) of y [recv_offsets[world], H] fp32 is stored as row
 * dst_row0[s] + q - recv_offsets[s] of dst_y[s] (the source's buffer of its
 * send order).  Arrays and errors as in moe_ep_pack.
 */
int moe_ep_return(const float *y, int H, int world, const int64_t *recv_offsets,
                  float *const *dst_y, const int64_t *dst_row0, void *stream);

/*
 * moe_ep_combine -- out[t] = sum over j = 0..k-1 in ascending order of
 * topk_weights[t, j] * y_back[inv[t*k + j]] (one fp32 fused multiply-add per
 * term; slots with inv = -1 skipped and flagged), every row of out
 * [T, H] fp32 written.  y_back [T*k, H] fp32 in the send order.
 * Errors: INVALID_ARG for null pointers or unaligned y_back / out, T < 0,
 *         k < 1; UNSUPPORTED for H % 128 != 0 or k > 16.
 */
int moe_ep_combine(const float *y_back, const int32_t *inv, const float *topk_weights, float *out,
                   int64_t T, int H, int k, void *stream);

/* Static, NUL-terminated description of an MOE_* return code. */
const char *moe_error_string(int code);

/*
 * moe_get_device_status -- SYNCHRONISES `stream`, then returns in *status
 * the OR of the MOE_STATUS_* bits raised by this library's kernels on the
 * current device since the last call, and clears them.  Debug aid.
 */
int moe_get_device_status(void *stream, uint32_t *status);

/*
 * Tuning and debug switches (host-side, process-wide):
 *   moe_set_small_t_max(n)  -- moe_forward uses the GEMV path when T <= n
 *                              (default 8, at most 16, also read from
 *                              MOE_SMALL_T_MAX);
 *                              n = 0 forces the grouped-GEMM path.
 *   moe_set_sync_each_stage(on) -- synchronise and check for errors after
 *                              every launch (also MOE_SYNC_EACH_STAGE=1);
 *                              a failure returns MOE_ERR_CUDA and
 *                              moe_last_failed_stage() names the kernel.
 *   moe_set_wait_limit_ns(ns) -- bound of every device-side pipeline wait
 *                              (default 2e9 ns); ns <= 0 restores it.
 * Each returns the previous value.
 */
int moe_set_small_t_max(int n);
int moe_set_sync_each_stage(int on);
int64_t moe_set_wait_limit_ns(int64_t ns);
const char *moe_last_failed_stage(void);

/*
 * moe_debug_wait_timeout -- launches one CTA that waits on a shared-memory
 * barrier nothing will ever signal, bounded by `limit_ns`, and SYNCHRONISES
 * the stream.  Returns MOE_ERR_TIMEOUT when the bounded wait gave up as
 * designed (and leaves MOE_STATUS_TIMEOUT set), MOE_OK if it somehow
 * completed.  Exercises the failure path of the pipeline waits without
 * faulting or hanging the GPU.  limit_ns must be in (0, 1e10].
 */
int moe_debug_wait_timeout(int64_t limit_ns, void *stream);

/*
 * moe_timeline -- debug timeline of the kernels' inner schedule.  While buf
 * (a zeroed DEVICE buffer of 32 + 32 * capacity bytes, 8-byte aligned,
 * owned by the caller) is set, the grouped-GEMM kernels write one record
 * per tile and role and the small-batch kernel one per CTA and phase into
 * fixed slots of buf (as uint64_t[]): record i at [4 + 4i ..] = {tag, id,
 * t0, t1} with %globaltimer nanoseconds t0 <= t1 and tag = kind << 56 |
 * role << 48 | cta << 16 | sub (unused slots keep tag 0):
 *   kind 1 GEMM1 launch, 2 GEMM2 launch, 3 one-launch GEMM, 4 small-batch;
 *   role 0 producer (t0 tile start, t1 last operand load issued),
 *        1 MMA issuer (t0 accumulator free, t1 last MMA issued),
 *        2 epilogue, first epilogue warp (t0 accumulator full, t1 released),
 *        3 / 4 small-batch phase 1 / grid barrier, 5 act staged on chip,
 *        6 w2 rows on chip, 7 phase 2, 8 phase 2's dot products done
 *        (3-8: id = CTA);
 *   sub: the CTA's rank in its pair (roles 0 and 2); id: the tile number.
 * Each call's records overwrite the previous call's; slots past capacity
 * are dropped.  buf == NULL turns it off (the default).  Not synchronised
 * with running work: set it between calls.  Errors: INVALID_ARG for
 * capacity < 1 or an unaligned buf.
 */
int moe_timeline(void *buf, int64_t capacity);

/*
 * Per-kernel timing for benchmarks.  While enabled, moe_route/moe_forward/
 * moe_permute record a CUDA event pair around each kernel launch on the
 * caller's stream.  moe_profile_read SYNCHRONISES the device, then for each
 * kernel name (up to max_names) writes its launch count, total milliseconds
 * and name, and returns how many names exist.  moe_profile_reset clears.
 * Independently of this switch, every kernel launch of every entry point
 * sits inside an NVTX range named after its stage ("route", "group_gather",
 * "gemm_fused", "small_t", ...), pushed and popped on the calling thread;
 * with no NVTX tool attached to the process those calls do nothing.
 */
int moe_profile_enable(int on);
int moe_profile_reset(void);
int moe_profile_read(int max_names, char (*names)[64], int64_t *launches,
                     double *total_ms);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
