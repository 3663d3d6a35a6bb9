/*
 * statekv.h — C ABI of the StateKV per-frame streaming-prefill library
 * (libstatekv.so, sm_100a).
 *
 * Method: "Linear Scaling Video VLMs for Long Video Understanding" (StateKV).
 * Citations name the summary page by title and the section on it:
 *   P1  "线性扩展视频视觉语言模型用于长视频理解 Linear Scaling Video VLMs for Long
 *       Video Understanding" (Chinese summary), section 方法步骤详情 (method steps).
 *   P2  "Linear Scaling Video VLMs for Long Video Understanding" (section
 *       summary), section 3.2 Method Overview, 3.3 Per-frame cache-builder
 *       forward pass, Appendix A "Protocol", A.3 "Kernel considerations".
 *   P3  "Technische Samenvatting: Lineair Schalende Video VLMs voor Lange Video
 *       Begrip (StateKV)", section 2 "Architectuur en Mechanisme".
 *
 * Conventions for every call:
 *   - Return 0 (STATEKV_OK) on success, a negative statekv_status on error.  On
 *     error nothing is enqueued and the handle's state is unchanged;
 *     statekv_last_error() holds a message.  No kernel traps on bad input: the
 *     host validates first.
 *   - "device pointer" arguments point to GPU global memory of the current
 *     device, row-major and contiguous, with at least 16-byte alignment.  The
 *     caller owns them; the library never frees or retains them past the call.
 *   - "stream" is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls only enqueue work on it and never synchronise the host, except
 *     where stated (allocation on first use of a layer).
 *   - Shapes: S = n_streams (1 unless created batched), Hq query heads, Hkv KV
 *     heads (Hq % Hkv == 0, query head h reads KV head h / (Hq/Hkv)), head
 *     dimension d in {64, 128}, T tokens per frame, B the capacity of the
 *     compressed state.
 *   - Element type: STATEKV_BF16 (bfloat16, the graded path, tensor cores) or
 *     STATEKV_F32 (float32, CUDA-core path).  Arithmetic is float32 in both.
 */
#ifndef STATEKV_H
#define STATEKV_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct statekv_handle* statekv_t;

typedef enum { STATEKV_BF16 = 0, STATEKV_F32 = 1 } statekv_dtype;

/* Mask inside the current frame.  FRAME_CAUSAL (default): frame query i sees
 * frame tokens t <= i (the backbone LLM is causal, P1 section 自注意力复杂度);
 * FRAME_BIDIR: every frame token.  Entries of the compressed state are always
 * visible. */
typedef enum { STATEKV_MASK_FRAME_CAUSAL = 0, STATEKV_MASK_FRAME_BIDIR = 1 } statekv_mask;

/* Selection granularity.  GLOBAL (default): one score per candidate summed over
 * all query heads, one kept set per layer.  PER_KV_HEAD: scores summed over
 * the query heads of each KV head, a kept set per KV head (P2 Appendix A
 * "Protocol": sinks are kept per layer and KV head).  RECENCY: the pages'
 * comparison baseline (P2 Appendix A.3, recency-based retention): C_n keeps the
 * B candidates with the largest positions (the last B tokens), one set per
 * layer; scores are still computed and reported as in GLOBAL mode.  Positions
 * must be non-negative in this mode. */
typedef enum {
  STATEKV_SELECT_GLOBAL = 0,
  STATEKV_SELECT_PER_KV_HEAD = 1,
  STATEKV_SELECT_RECENCY = 2
} statekv_select;

typedef enum {
  STATEKV_OK = 0,
  STATEKV_ERR_INVALID_ARG = -1, /* null pointer, bad shape, bad enum          */
  STATEKV_ERR_UNSUPPORTED = -2, /* d not in {64,128}, unsupported combination  */
  STATEKV_ERR_CAPACITY = -3,    /* more frames than max_frames on a layer     */
  STATEKV_ERR_OOM = -4,         /* device allocation failed                   */
  STATEKV_ERR_CUDA = -5         /* a CUDA launch or runtime call failed       */
} statekv_status;

/* Create a handle for one video stream (S = 1).
 * Per-layer state (C, D and the layer's own step scratch) is allocated on a
 * layer's first prefill_frame call (or by statekv_reserve_layers).
 * max_frames bounds the frames per layer (D holds max_frames*T tokens).
 * B >= 0 (B = 0: no cross-frame context).  Errors: INVALID_ARG, UNSUPPORTED,
 * OOM, CUDA.  *h is set only on success. */
int statekv_create(statekv_t* h, int Hq, int Hkv, int d, int T, int B, int max_frames,
                   int dtype, int mask_mode, int select_mode);

/* Same as statekv_create for n_streams independent video streams processed
 * together: every tensor below gains a leading [S] dimension and each stream
 * keeps its own C and D.  All streams advance one frame per call. */
int statekv_create_batched(statekv_t* h, int n_streams, int Hq, int Hkv, int d, int T,
                           int B, int max_frames, int dtype, int mask_mode,
                           int select_mode);

/* Allocate the state of layers 0..n_layers-1 now (synchronous; device memory
 * zero-filled).  Call before capturing prefill calls in a CUDA graph. */
int statekv_reserve_layers(statekv_t h, int n_layers);

/* One StateKV cache-builder step for one layer and the next frame
 * (P1 section 方法步骤详情; P2 section 3.3; P3 section 2 "Het Proces"):
 *   1. out = softmax(q [C_{n-1}; k]^T / sqrt(d)) [C_{n-1}; v]  (mask_mode);
 *   2. D <- D || (k, v, pos);
 *   3. score_j = sum over the frame's queries i (and heads) of P_ij for every
 *      candidate j of the pool C_{n-1} followed by the frame's tokens;
 *   4. C_n = the B best candidates by (score desc, position asc), stored in
 *      ascending position order (all candidates while m + T <= B).
 * Inputs (device pointers, element type = dtype):
 *   q   [S][T][Hq][d]   queries, RoPE already applied at absolute positions
 *   k,v [S][T][Hkv][d]  keys (RoPE applied) and values
 *   pos [S][T] int32    absolute ("virtual") positions (P2 section 3.3); they
 *                       must increase along the stream: every frame's positions
 *                       ascending and above all earlier frames' positions.
 *                       The library stores them and never re-rotates.
 * Output (device pointer): out [S][T][Hq][d] (dtype).
 * Frame n of a layer must follow frame n-1 of that layer in stream order;
 * layers may interleave.  Steps of different layers share no device memory
 * (each layer has its own C, D and step scratch), so they may also run
 * concurrently on different streams, e.g. frame n+1 of layer l beside frame n
 * of layer l+1 (order each layer's frames with events).  Calls on one handle
 * must come from one host thread at a time.  Errors: INVALID_ARG, CAPACITY,
 * OOM (first use of a layer), CUDA. */
int statekv_prefill_frame(statekv_t h, int layer, const void* q, const void* k,
                          const void* v, const int32_t* pos, void* out, void* stream);

/* statekv_prefill_frame with HOST buffers: q, k, v, pos are read from and out
 * is written to host memory (same layouts; page-locked memory makes the copies
 * asynchronous, pageable memory is accepted).  The call copies the inputs into
 * one of two library-owned staging sets on a library-owned copy stream, runs
 * the step on a library-owned compute stream once they have arrived, and
 * makes `stream` wait for the step and copy out back.  So the copies of call
 * n+1 and the copy-out of call n overlap the steps.  When `stream` has reached
 * the end of the call, the inputs have been read and out is complete
 * (synchronise the stream before reading out or reusing the input buffers).
 * A layer's frames may come through both entry points: the library orders a
 * layer's step after its previous one (a host-buffer step after device-buffer
 * steps enqueued on `stream` before it).  The first call creates the staging
 * buffers, the two streams and their events (synchronous).  Errors: as
 * statekv_prefill_frame. */
int statekv_prefill_frame_host(statekv_t h, int layer, const void* q, const void* k,
                               const void* v, const int32_t* pos, void* out, void* stream);

/* Decode attention over the detailed state D of a layer: the n_text tokens
 * that follow the video (a question, or generated text) attend to every
 * video token D holds and causally to each other (P1 section 方法步骤详情: the
 * frame's KV pairs go to the detailed cache; P2 section 3.2: the second cache
 * keeps full per-frame detail for the final generation).
 *   q   [S][n_text][Hq][d]   text queries (device, dtype), RoPE applied
 *   k,v [S][n_text][Hkv][d]  text keys and values (device, dtype)
 *   out [S][n_text][Hq][d]   (device, dtype)
 *   lse [S][Hq][n_text]      float32 natural-log log-sum-exp (device) or NULL
 * Text token i sees D tokens [0, frames*T) of the layer and text tokens 0..i.
 * D is read, not modified.  bf16 runs on the tensor cores with the G query
 * heads of a KV group stacked in one tile, so each D tile crosses HBM once
 * per KV head; float32 runs on the CUDA cores.  Split scratch is allocated on
 * the first call that needs more than before (synchronous), then reused.
 * Errors: INVALID_ARG (unknown layer, bad pointer), OOM, CUDA. */
int statekv_decode(statekv_t h, int layer, const void* q, const void* k, const void* v, int n_text,
                   void* out, float* lse, void* stream);

/* Borrow the compressed state C_n of a layer (device pointers owned by the
 * library; valid until the next prefill_frame on that layer or destroy):
 *   k,v   [S][Hkv][B][d] (dtype), rows [0, len) valid, ascending position
 *   pos   [S][Hkv][B] int32, score [S][Hkv][B] float32 (the score each kept
 *         entry earned in the frame that selected it).  In GLOBAL mode the Hkv
 *         rows of pos/score are identical.
 *   len   current length m = min(B, frames*T).
 * Any output pointer may be NULL.  Errors: INVALID_ARG (unknown layer). */
int statekv_get_compressed(statekv_t h, int layer, const void** k, const void** v,
                           const int32_t** pos, const float** score, int* len);

/* Borrow the detailed state D of a layer (P2 section 3.2: every frame token,
 * kept for decoding):
 *   k,v [S][Hkv][max_frames*T][d] (dtype), tokens [0, len) valid, in arrival
 *   order; pos [S][max_frames*T] int32.  len = frames*T.
 * Valid until destroy.  Errors: INVALID_ARG. */
int statekv_get_detailed(statekv_t h, int layer, const void** k, const void** v,
                         const int32_t** pos, int* len);

/* Borrow the per-row statistics of the most recent prefill_frame call (of
 * whichever layer it was):
 *   lse        [S][Hq][T] float32, natural-log log-sum-exp of each query row;
 *   pool_score [S][Hkv][B+T] float32, the score of every pool candidate
 *              (C entries first, then frame tokens); entries [0, pool_len)
 *              valid.  In GLOBAL and RECENCY modes only row 0 of each stream
 *              is written.
 * Valid until the next prefill_frame on that layer.  Any output pointer may be
 * NULL.  Errors: INVALID_ARG (no step has run yet). */
int statekv_get_step_stats(statekv_t h, const float** lse, const float** pool_score,
                           int* pool_len);

/* Kernel stages of one step, for statekv_profile_read. */
typedef enum {
  STATEKV_STAGE_ATTENTION = 0,         /* (a) attention main kernel            */
  STATEKV_STAGE_ATTENTION_COMBINE = 1, /* (a) merge of key-split partials      */
  STATEKV_STAGE_SCORE = 2,             /* (b) score pass                       */
  STATEKV_STAGE_SELECT = 3,            /* (c) top-B select                     */
  STATEKV_STAGE_GATHER = 4,            /* (d) gather into C_n + append to D    */
  STATEKV_STAGE_DECODE = 5,            /* statekv_decode attention             */
  STATEKV_STAGE_DECODE_COMBINE = 6,    /* statekv_decode merge of key splits   */
  STATEKV_STAGE_ATTENTION_CHAINED = 7, /* (a) attention and its split merge,   */
                                       /*     one event pair (profiling mode 2) */
  STATEKV_N_STAGES = 8
} statekv_stage;

/* Per-stage device timing.  on = 1: every later prefill_frame records a CUDA
 * event pair around each kernel on the call's stream (a few microseconds of
 * extra enqueue cost; leave off in production), and the merge of the
 * attention's key splits, which otherwise rides in the select launch, runs as
 * its own launch so that its time is recorded under ATTENTION_COMBINE.
 * on = 2: the same, except that the attention and its merge share one event
 * pair, recorded under ATTENTION_CHAINED, with the merge launched right behind
 * the attention as a programmatic dependent launch (as the step chains its
 * kernels), so that the pair times both kernels without a launch gap between
 * them.  on = 0 turns timing off and drops unread records; any other value is
 * STATEKV_ERR_INVALID_ARG. */
int statekv_profile_enable(statekv_t h, int on);

/* Accumulated device time and launch count per stage since the last read:
 * ms[STATEKV_N_STAGES] milliseconds, launches[STATEKV_N_STAGES] (either may be
 * NULL).  Waits for the recorded events (host synchronisation), then resets. */
int statekv_profile_read(statekv_t h, double* ms, long long* launches);

/* Number of kernels this handle has launched since it was created. */
long long statekv_kernel_launches(statekv_t h);

/* Device-side status of the handle's kernels: *code = 0, or the first error a
 * kernel recorded since the last call (a pipeline wait that exceeded its time
 * limit; the kernel then abandoned its tile and exited cleanly, so results of
 * that step are invalid).  Synchronises the device, then resets the word. */
int statekv_device_status(statekv_t h, int* code);

/* Time limit of the pipeline waits inside the handle's tensor-core kernels
 * (ns <= 0 restores the default of 0.5 s).  A wait that runs past it makes
 * the kernel record a code that statekv_device_status reports, drain its own
 * copies and MMAs and exit; the results of that step are invalid, and later
 * steps run normally.  Meant for testing that failure path: a limit of a few
 * nanoseconds makes the waits give up on an otherwise healthy step. */
int statekv_set_wait_limit(statekv_t h, long long ns);

/* Frames processed so far on a layer (0 for a layer never called). */
int statekv_frames(statekv_t h, int layer);

/* Release all device memory of the handle (synchronises the device first). */
int statekv_destroy(statekv_t h);

/* Message of the handle's last error ("" if none); h may be NULL for errors of
 * calls that had no handle (create, full_causal_prefill). */
const char* statekv_last_error(statekv_t h);

/* Full causal self-attention over n_tokens tokens: the quadratic comparator
 * (P2 section 4 "Compute scaling"; P2 A.3: the full-attention baseline).
 *   q [n_tokens][Hq][d], k,v [n_tokens][Hkv][d] (device, dtype);
 *   out [n_tokens][Hq][d] (device, dtype);
 *   lse [Hq][n_tokens] float32 natural-log (device) or NULL.
 * Token i attends to tokens 0..i.  Scratch is allocated by the library on
 * first use and kept (grown as needed) until process exit.
 * Errors: INVALID_ARG, UNSUPPORTED, OOM, CUDA. */
int full_causal_prefill(const void* q, const void* k, const void* v, int n_tokens, int Hq,
                        int Hkv, int d, int dtype, void* out, float* lse, void* stream);

/* full_causal_prefill over n_seq independent sequences of n_tokens each:
 * every tensor gains a leading [n_seq] dimension (lse: [n_seq][Hq][n_tokens]). */
int full_causal_prefill_batched(const void* q, const void* k, const void* v, int n_seq,
                                int n_tokens, int Hq, int Hkv, int d, int dtype, void* out,
                                float* lse, void* stream);

/* One StateKV step (same computation as statekv_prefill_frame for S = 1) that
 * allocates no device memory.  The paper has no counterpart: this is a
 * deployment variant for callers that cannot call cudaMalloc when they run the
 * step, e.g. a server that has already reserved nearly all GPU memory for its
 * own pool, or a latency-critical loop that cannot afford cudaMalloc's
 * implicit device-wide synchronisation.
 *
 * Arithmetic: for both element types the attention and score passes run on
 * the CUDA cores (float32 FMA), not on the tensor cores that
 * statekv_prefill_frame uses for bf16.  bf16 results therefore agree with
 * statekv_prefill_frame within the parity tolerances, not bit for bit (a
 * candidate within 1e-4 relative of the B-th score may be kept by one and
 * not the other), and at the 8B-class shape this entry point is many times
 * slower; it is not the timed path.
 *
 * The caller owns every tensor (device pointers, 16-byte aligned):
 *   q [T][Hq][d], k,v [T][Hkv][d], pos [T]        the frame (as prefill_frame);
 *   kc,vc [Hkv][B][d], posc [Hkv][B], m            C_{n-1}: its first m rows;
 *   out [T][Hq][d]                                 attention output;
 *   kc_new,vc_new [Hkv][B][d], posc_new, scorec_new [Hkv][B]
 *                                                  C_n (min(B, m+T) rows); must
 *                                                  not alias kc/vc;
 *   kd,vd [Hkv][max_tok][d], posd [max_tok]        D; the frame is appended at
 *                                                  token d_len (d_len+T <= max_tok).
 * pos, posc, posc_new, scorec_new and posd need 4-byte alignment.  Every
 * output range (out, C_n, D) must be disjoint from every input range and from
 * the other outputs; overlapping buffers are refused with INVALID_ARG.
 * Per-step scratch lives in one file-scope device array of 1 MiB per device
 * (lse [Hq][T], partial and pool scores [Hkv][B+T], kept list [Hkv][B], each
 * rounded up to 256 bytes); shapes that need more are rejected with
 * STATEKV_ERR_UNSUPPORTED and a message naming the size.  Nothing in the
 * scratch must start at zero (each call writes what it reads).  The array is
 * shared by every call on the device and keeps the last call's contents, so
 * calls whose work overlaps on the GPU (different streams, or threads using
 * this entry point concurrently) race; order them on one stream.  The first
 * call on each device looks up the array's device address (with that device
 * current); make that first call before any stream capture.
 * Errors (message in statekv_last_error(NULL)): INVALID_ARG, UNSUPPORTED,
 * CAPACITY, CUDA. */
int statekv_step_noalloc(int Hq, int Hkv, int d, int T, int B, int dtype, int mask_mode,
                         int select_mode, const void* q, const void* k, const void* v,
                         const int32_t* pos, const void* kc, const void* vc,
                         const int32_t* posc, int m, void* out, void* kc_new, void* vc_new,
                         int32_t* posc_new, float* scorec_new, void* kd, void* vd,
                         int32_t* posd, int d_len, int max_tok, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* STATEKV_H */
