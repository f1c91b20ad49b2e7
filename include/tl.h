/*
 * tl.h -- C ABI of the B200 (sm_100a) looped INT4 transformer library.
 *
 * The library computes the forward pass of a weight-shared looped transformer:
 *   tokens -> embed -> pre blocks -> one shared loop block run L times
 *          -> output norm -> head
 * (TinyLoop README, "Why TinyLoop Exists"), with every block linear stored as
 * group-wise INT4 weights with zero points, w = (q - z) * s, group 128 along K
 * (TinyLoop README, "Status", INT4 loop / pre linears with zero points).  The
 * loop count L is an argument of every call (TinyLoop docs, "Async API",
 * "Scoring" and "Generation": loops= on score / generate).
 *
 * General conventions
 * -------------------
 * - Every pointer named d_* is DEVICE memory on the model's / call's device;
 *   every pointer named h_* is HOST memory.  The caller owns all buffers it
 *   passes; the library never frees them and keeps no pointer to them after
 *   the call returns, except where a function says otherwise.
 * - fp16 values travel as uint16_t bit patterns (IEEE binary16).
 * - Arguments are validated synchronously before anything is enqueued; a call
 *   that returns an error has enqueued nothing (apart from TL_ERR_CUDA, which
 *   reports a failed launch).  tl_last_error() returns a one-line reason for
 *   the last error of the calling thread.
 * - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *   legacy default stream).  Results are ready when the stream reaches them.
 * - One model handle must not be used by two host threads at the same time
 *   (TinyLoop docs, "Async API", "Concurrency model": the model is not
 *   thread-safe and callers serialise).  Calls on one handle must be ordered
 *   on one stream.
 * - Data-dependent device-side faults (a token id outside [0, vocab)) do not
 *   trap: the kernel substitutes token 0, records the fault in a device flag,
 *   and tl_check_device_error() reports it.
 */
#ifndef TL_H_
#define TL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TL_OK = 0,
  TL_ERR_INVALID_ARG = 1,    /* a NULL pointer, size or shape out of range */
  TL_ERR_OOM = 2,            /* device allocation failed */
  TL_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed */
  TL_ERR_CONTEXT_FULL = 4,   /* the lane has no room for more tokens */
  TL_ERR_LOOPS_MISMATCH = 5, /* decode loops differ from the lane's prefill */
  TL_ERR_NOT_PREFILLED = 6,  /* decode on a lane that holds no prompt */
  TL_ERR_DEVICE_FLAG = 7,    /* a kernel recorded a data fault (see above) */
  TL_ERR_UNSUPPORTED = 8     /* a shape the kernels are not built for */
} tl_status;

/* Static description of a model (TinyLoop docs, "Async API", "Constructor":
 * max_seq_len; the dimensions are those of the Llama-family block that the
 * README's "Status" list names: RoPE with configurable theta, GQA). */
typedef struct {
  int d_model;      /* hidden size; multiple of 128 */
  int n_q_heads;    /* query heads */
  int n_kv_heads;   /* key/value heads; divides n_q_heads (GQA) */
  int head_dim;     /* 64 or 128; n_q_heads * head_dim is a multiple of 128 */
  int ffn_dim;      /* SwiGLU inner size F; multiple of 128 */
  int vocab;        /* vocabulary size; multiple of 16 */
  int n_pre;        /* number of distinct pre blocks (>= 0) */
  int max_loops;    /* largest L any call may use (>= 1) */
  int max_ctx;      /* tokens per lane (prompt + generated), <= 8192 */
  int max_lanes;    /* decode lanes, 1..16 */
  float rms_eps;    /* RMSNorm epsilon */
  float rope_theta; /* RoPE base */
  int kv_mode;      /* TL_KV_FP16 (0) or TL_KV_INT8, see below */
  int weight_bits;  /* block linears: 4 (or 0) INT4, 2 the INT2 body, see tl_int4_linear */
} tl_config;

/* KV cache storage (TinyLoop README, "Python API reference", KV cache modes:
 * "FP16 KV" and "INT8 KV"; the pages give no INT8 format, so this is the
 * plainest reading).  TL_KV_FP16 stores the rotated keys and the values as
 * fp16.  TL_KV_INT8 stores each key or value vector (one position, one kv
 * head: head_dim elements) as int8 codes with one fp32 scale, scale =
 * max|x| / 127 and code = round-half-even(x / scale) in fp32 (an all-zero
 * vector has scale 0); attention reads code * scale.  INT8 halves the cache's
 * bytes.  Both per-op decode forms (tl_model_set_clustered_decode) read and
 * write it; every prefill attention pass runs on the 16-query tile kernel;
 * the single-kernel decode path (TL_DECODE_FUSED) is FP16 only. */
enum { TL_KV_FP16 = 0, TL_KV_INT8 = 1 };

/* One INT4 linear with K inputs and N outputs, HOST memory, storage format
 * (with tl_config.weight_bits = 2 / tl_linear_create_int2, the INT2 body of
 * TinyLoop README, "Current Runtime Snapshot", whose format the pages do not
 * give, read as the same layout with 2-bit fields: qweight uint32
 * [N][K/16] with element k in bits 2*(k%16)..+1 of word k/16, qzeros uint32
 * [N][ceil(K/2048)] with sixteen 2-bit zero points per word, q and z in
 * 0..3; the decode kernels then read half the weight bytes, the prefill GEMM
 * widens the codes to its 4-bit tile layout at load):
 *   qweight uint32 [N][K/8]        element k of row n is bits 4*(k%8)..+3 of
 *                                  word k/8 (low nibble first)
 *   scales  fp16   [N][K/128]      scale of (row, group)
 *   qzeros  uint32 [N][ceil(K/1024)] the K/128 zero points of the row, eight
 *                                  per word, same nibble order, unused = 0
 * The dequantized weight is W[n][k] = (q - z) * s with no offset on z. */
typedef struct {
  const uint32_t *qweight;
  const uint16_t *scales;
  const uint32_t *qzeros;
} tl_int4_linear;

/* One transformer block (pre-norm, Llama family).
 *   qkv:     N = (n_q_heads + 2 n_kv_heads) * head_dim, K = d_model; rows are
 *            the q heads, then the k heads, then the v heads, head-major
 *   o:       N = d_model, K = n_q_heads * head_dim
 *   gate_up: N = 2 ffn_dim, K = d_model; rows [0, F) gate, [F, 2F) up
 *   down:    N = d_model, K = ffn_dim
 *   attn_norm, ffn_norm: fp16 [d_model] RMSNorm gains */
typedef struct {
  const uint16_t *attn_norm;
  const uint16_t *ffn_norm;
  tl_int4_linear qkv, o, gate_up, down;
} tl_block;

/* All weights, HOST memory.  embed and head are fp16 [vocab][d_model] (the
 * head is its own matrix), out_norm fp16 [d_model], pre[n_pre] the distinct
 * pre blocks, loop the one block shared by every loop iteration. */
typedef struct {
  const uint16_t *embed;
  const uint16_t *out_norm;
  const uint16_t *head;
  const tl_block *pre;
  const tl_block *loop;
} tl_weights;

typedef struct tl_model tl_model;
typedef struct tl_linear tl_linear;

/* ------------------------------------------------------------------------
 * Model API
 * ------------------------------------------------------------------------ */

/* Copy the host weights to `device`, re-lay them out for the kernels and
 * allocate the KV cache (max_lanes lanes x (n_pre + max_loops) layers x K/V x
 * n_kv_heads x max_ctx x head_dim fp16, one slice per effective layer, so that
 * every loop iteration keeps its own keys and values; TinyLoop README,
 * "Status", GQA item) and all workspaces.  The host arrays may be freed when
 * this returns.  On success *out owns all device memory of the model. */
tl_status tl_model_create(const tl_config *cfg, const tl_weights *w, int device,
                          tl_model **out);

/* Free all device memory of the model.  NULL is a no-op.  The caller must make
 * sure no work of the model is still pending on any stream. */
void tl_model_destroy(tl_model *m);

/* Run a prompt on `lane` (0 <= lane < max_lanes): n_tokens ids at positions
 * 0..n_tokens-1 through n_pre + loops effective layers, writing each layer's
 * keys and values to the lane's cache slices.  Any earlier content of the lane
 * is discarded; the lane's loop count becomes `loops`.
 *   d_tokens        int32 [n_tokens], 1 <= n_tokens <= max_ctx
 *   loops           1 <= loops <= max_loops
 *   d_last_logits   fp32 [vocab] logits of the last position, or NULL to skip
 *                   the output norm and head ("no logits", TinyLoop README,
 *                   "Current Runtime Snapshot")
 *   d_last_argmax   int32 [1] greedy token of the last position (lowest index
 *                   on ties), or NULL; needs the head, like the logits. */
tl_status tl_prefill(tl_model *m, int lane, const int32_t *d_tokens, int n_tokens,
                     int loops, float *d_last_logits, int32_t *d_last_argmax,
                     void *stream);

/* One cached decode step for n_lanes lanes at once (TinyLoop docs, "Async
 * API", "Batch generation": per-lane loops).  Lane i feeds token d_tokens[i]
 * at position length(lane) and attends over its own cache; each lane runs
 * exactly its own n_pre + loops layers, and its result does not depend on
 * which other lanes share the step.
 *   h_lane_ids  int32 [n_lanes], distinct, each prefilled
 *   d_tokens    int32 [n_lanes]
 *   h_loops     int32 [n_lanes], must equal each lane's prefill loops
 *               (else TL_ERR_LOOPS_MISMATCH)
 *   d_logits    fp32 [n_lanes][vocab] or NULL
 *   d_argmax    int32 [n_lanes] greedy tokens, or NULL.  May alias d_tokens:
 *               the tokens are read before the argmax is written.
 * Returns TL_ERR_CONTEXT_FULL if a lane already holds max_ctx tokens. */
tl_status tl_decode_step(tl_model *m, int n_lanes, const int32_t *h_lane_ids,
                         const int32_t *d_tokens, const int32_t *h_loops,
                         float *d_logits, int32_t *d_argmax, void *stream);

/* Append n_tokens tokens to a prefilled lane: positions length(lane) ..
 * length(lane) + n_tokens - 1 through the lane's n_pre + loops layers,
 * attending to everything the lane holds (a chunk of a longer prompt --
 * TinyLoop docs, "Async API", "Constructor": prefill_chunk -- or the verify
 * pass of speculative decoding).  The lane's length grows by n_tokens.
 *   d_tokens  int32 [n_tokens]
 *   d_logits  fp32 [n_tokens][vocab] logits of EVERY appended position, or NULL
 *   d_argmax  int32 [n_tokens] greedy token of every position, or NULL
 * Per-position outputs need n_tokens <= 16 (else TL_ERR_UNSUPPORTED);
 * TL_ERR_NOT_PREFILLED for an empty lane, TL_ERR_CONTEXT_FULL past max_ctx. */
tl_status tl_extend(tl_model *m, int lane, const int32_t *d_tokens, int n_tokens, float *d_logits,
                    int32_t *d_argmax, void *stream);

/* Counters of one tl_generate_speculative call. */
typedef struct {
  int rounds;    /* draft + verify rounds */
  int drafted;   /* draft tokens proposed */
  int accepted;  /* draft tokens the verifier agreed with */
} tl_spec_stats;

/* Greedy self-speculative generation on a prefilled lane (TinyLoop docs,
 * "Async API", "Speculative decode": draft_loops, verify_loops, draft_ahead;
 * TinyLoop README, "Why TinyLoop Exists", item 3: draft and verify reuse the
 * same weights; "Quick CLI Tour", Speculate).  The verifier runs the lane's
 * prefill loops; the draft model is the same network cut after draft_loops
 * loop iterations, so its keys and values are the verifier's first slices.
 * Each round: k = min(draft_ahead, tokens still to produce) cached greedy
 * draft steps with draft_loops from the next input token, then one pass of
 * those k inputs through all the lane's loops (tl_extend's computation)
 * giving the verifier's greedy token at each; drafts are accepted while they
 * equal the verifier's tokens, the verifier's token replaces the first
 * rejected draft, and the lane's length is rolled back to the accepted
 * positions.  The output therefore equals max_tokens plain greedy decode
 * steps at the lane's loops (up to rounding at near-ties).
 *   d_first_token  int32 [1] the token fed at position length(lane), as for
 *                  tl_decode_step
 *   max_tokens     tokens to produce (>= 1, length(lane) + max_tokens <= max_ctx)
 *   draft_loops    1 <= draft_loops <= the lane's loops
 *   draft_ahead    1 <= draft_ahead <= 16
 *   d_out_tokens   int32 [max_tokens] the generated tokens
 *   h_stats        HOST, or NULL
 * On return the lane holds length + max_tokens positions, as after
 * max_tokens decode steps.  Synchronises `stream` once per round (the
 * accepted count decides the next round on the host). */
tl_status tl_generate_speculative(tl_model *m, int lane, const int32_t *d_first_token, int max_tokens,
                                  int draft_loops, int draft_ahead, int32_t *d_out_tokens,
                                  tl_spec_stats *h_stats, void *stream);

/* Stateless uncached forward (TinyLoop docs, "Async API", "Scoring",
 * score_last): logits [vocab] of the last of n_tokens tokens.  Touches no
 * lane (it uses a private scratch slice).  d_logits must not be NULL;
 * d_argmax may be NULL. */
tl_status tl_score_last(tl_model *m, const int32_t *d_tokens, int n_tokens, int loops,
                        float *d_logits, int32_t *d_argmax, void *stream);

/* Logit lens (TinyLoop docs, "Async API", "Scoring", score_logit_lens:
 * [loops, vocab]): a stateless uncached forward like tl_score_last that
 * applies the output norm and head to the last position after EVERY loop
 * iteration.  Row i of d_logits (fp32 [loops][vocab]) holds the logits after
 * iteration i + 1, which equal tl_score_last with loops = i + 1; d_argmax
 * (int32 [loops], or NULL) their greedy tokens. */
tl_status tl_score_logit_lens(tl_model *m, const int32_t *d_tokens, int n_tokens, int loops,
                              float *d_logits, int32_t *d_argmax, void *stream);

/* Token-stable early exit (TinyLoop README, "Runtime Flags",
 * TINYLOOP_TOKEN_EXIT=N): a stateless uncached forward of the last position
 * that stops iterating the loop block once the greedy token after the last
 * stable_n iterations has been the same, or after max_loops iterations.
 * d_logits fp32 [vocab] (and d_argmax int32 [1], or NULL) receive the
 * logits of the exit iteration, which equal tl_score_last with that many
 * loops; *h_loops_used (HOST) the iterations run.  Synchronises `stream`
 * after every iteration. */
tl_status tl_score_early_exit(tl_model *m, const int32_t *d_tokens, int n_tokens, int max_loops,
                              int stable_n, float *d_logits, int32_t *d_argmax, int *h_loops_used,
                              void *stream);

/* Prefix cache (TinyLoop README, "Python Quick Start": build_prefix_cache /
 * generate_from_prefix_cache; "Python API reference", Prefix cache): copy
 * the keys and values of positions 0 .. n_tokens - 1 of every slice of
 * src_lane (n_pre + its loops layers) into dst_lane, which then holds
 * n_tokens positions with src_lane's loops, as if it had been prefilled with
 * the same first n_tokens tokens.  A lane prefilled with a shared prompt is
 * the prefix cache; forks continue from it without recomputing it.
 * 1 <= n_tokens <= length(src_lane); the lanes differ. */
tl_status tl_lane_fork(tl_model *m, int src_lane, int dst_lane, int n_tokens, void *stream);

/* Snapshot of one lane's KV slice `layer` (0 <= layer < n_pre + the lane's
 * loops), positions [0, n_tokens), copied out of the cache as stored (the
 * prefix cache's snapshot of a lane's slices; same pages as tl_lane_fork):
 *   FP16 cache: d_k, d_v fp16 [n_kv_heads][n_tokens][head_dim] (rotated keys,
 *               values); d_k_scales / d_v_scales are not touched (may be NULL)
 *   INT8 cache: d_k, d_v int8 codes [n_kv_heads][n_tokens][head_dim] and
 *               d_k_scales, d_v_scales fp32 [n_kv_heads][n_tokens]
 * Device pointers, stream-ordered after the calls that wrote the lane.
 * TL_ERR_NOT_PREFILLED for an empty lane, TL_ERR_INVALID_ARG for a layer or
 * n_tokens out of range (n_tokens <= the lane's length) or a NULL pointer. */
tl_status tl_lane_kv_export(const tl_model *m, int lane, int layer, int n_tokens, void *d_k, void *d_v,
                            float *d_k_scales, float *d_v_scales, void *stream);

/* Tokens currently held by a lane (0 if never prefilled). */
tl_status tl_lane_length(const tl_model *m, int lane, int *h_length);

/* Device bytes held by the model: weights (as laid out for the kernels), KV
 * cache, and all other workspaces.  Any pointer may be NULL. */
tl_status tl_model_info(const tl_model *m, size_t *weight_bytes, size_t *kv_bytes,
                        size_t *workspace_bytes);

/* Synchronise `stream`, read and clear the model's device fault flag.
 * Returns TL_OK, TL_ERR_DEVICE_FLAG (a kernel saw a token id outside
 * [0, vocab) and used token 0 instead), or TL_ERR_CUDA. */
tl_status tl_check_device_error(tl_model *m, void *stream);

/* Kernel families, for the per-kernel profiler. */
typedef enum {
  TL_KERNEL_EMBED = 0,        /* embedding gather */
  TL_KERNEL_QKV = 1,          /* RMSNorm + QKV INT4 linear + RoPE + KV write (+ attention: clustered kernel) */
  TL_KERNEL_ATTN_DECODE = 2,  /* single-query cached-decode attention */
  TL_KERNEL_O_PROJ = 3,       /* O INT4 linear + residual */
  TL_KERNEL_GATE_UP = 4,      /* RMSNorm + gate_up INT4 linear + SwiGLU */
  TL_KERNEL_DOWN = 5,         /* down INT4 linear + residual */
  TL_KERNEL_HEAD = 6,         /* output norm + head + greedy argmax */
  TL_KERNEL_ATTN_PREFILL = 7, /* tiled causal prefill attention */
  TL_KERNEL_GEMM_TC = 8,      /* tensor-core INT4 GEMM (prefill linears) */
  TL_KERNEL_NORM = 9,         /* stand-alone RMSNorm */
  TL_KERNEL_SETUP = 10,       /* per-call row bookkeeping */
  TL_KERNEL_DECODE_FUSED = 11,/* a whole decode step in one persistent kernel */
  TL_KERNEL_CLASSES = 12
} tl_kernel_class;

/* Per-kernel timing (the counterpart of the pages' phase timings, TinyLoop
 * README, "Quick CLI Tour", Benchmark with TINYLOOP_CUDA_PROFILE=1): from
 * this call on, every launch of the model whose class bit is set in
 * class_mask (bit c = class c) is bracketed by two CUDA events on its stream,
 * up to 16384 launches.  Events between launches serialise them, so profiled
 * runs are slower than unprofiled ones. */
tl_status tl_model_profile_start(tl_model *m, unsigned class_mask);

/* Stop profiling; waits for the recorded events and writes, per class,
 * the number of timed launches and their summed duration in ms.
 *   h_launches int [TL_KERNEL_CLASSES] or NULL, h_total_ms float [..] or NULL */
tl_status tl_model_profile_stop(tl_model *m, int *h_launches, float *h_total_ms);

/* Decode steps run as one captured CUDA graph per row pattern (lanes and
 * loop counts) by default; enable = 0 launches their kernels one by one
 * (same kernels, same results; useful under a kernel profiler). */
tl_status tl_model_set_graphs(tl_model *m, int enable);

/* How tl_decode_step runs a step (the same computation either way: the
 * cached single-token forward of TinyLoop README, "Architecture"):
 *   TL_DECODE_LAYERED  one kernel per projection / attention / head
 *                      (replayed as a CUDA graph unless disabled above);
 *   TL_DECODE_FUSED    the whole step as ONE persistent cooperative kernel
 *                      (one CTA per SM, grid-wide barriers between the
 *                      phases, weights streamed through shared memory);
 *                      steps it cannot take return TL_ERR_UNSUPPORTED;
 *   TL_DECODE_AUTO     (default) the faster of the two as measured on
 *                      B200 for the 400M model at batch 1: LAYERED.
 * FUSED needs <= 4 lanes per step, head_dim 64 or 128, n_pre <= 8,
 * d_model, n_q_heads * head_dim and ffn_dim <= 5760, and a device with
 * cooperative launch; set_decode_path returns TL_ERR_UNSUPPORTED for a model
 * it cannot run. */
typedef enum {
  TL_DECODE_AUTO = 0,
  TL_DECODE_LAYERED = 1,
  TL_DECODE_FUSED = 2
} tl_decode_path;
tl_status tl_model_set_decode_path(tl_model *m, int path);

/* Which per-op (TL_DECODE_LAYERED) step a model takes: enable = 1 runs each
 * layer's RMSNorm + QKV + RoPE + KV write + attention as ONE clustered kernel
 * (a thread-block cluster per kv head, <= 2 rows per launch); enable = 0 runs
 * the QKV GEMV and the split-KV attention kernel (every row in one launch
 * each; with an INT8 cache a quantising pass between them).  The default,
 * chosen at creation: clustered for max_lanes <= 2, otherwise the GEMV +
 * split-KV form (faster from 3 lanes on).  It is per model, so a lane's
 * results never depend on which lanes share a step.  Synchronises the device
 * and drops captured decode graphs when it changes the form.
 * TL_ERR_UNSUPPORTED: enable = 1 where the clustered kernel does not fit the
 * shapes or device. */
tl_status tl_model_set_clustered_decode(tl_model *m, int enable);

/* Phase timeline of single-kernel decode steps (the counterpart of the pages'
 * per-phase timings, TinyLoop README, "Quick CLI Tour", Benchmark with
 * TINYLOOP_CUDA_PROFILE=1).  While d_buf (device memory, n_entries uint64,
 * owned by the caller) is set, every TL_DECODE_FUSED step writes %globaltimer
 * nanoseconds there, G = tl_model_trace_grid(m) entries per event (slot s
 * = entries [s G, (s + 1) G), one per CTA): slot 0 kernel start; for grid
 * barrier k (5 per effective layer: after QKV, attention, O, gate_up, down)
 * slot 1 + 5k arrival and 2 + 5k release, and for the GEMV phase before it
 * 3 + 5k activations staged, 4 + 5k first weight item arrived (not written
 * by CTAs without items), 5 + 5k items consumed (none of the three for
 * attention); after B barriers, slot 1 + 5B head activations staged,
 * 2 + 5B head tiles done, 3 + 5B end.  Entries past n_entries are skipped.
 * d_buf = NULL turns it off.  Steps overwrite the same entries.  Head-only
 * launches of the layered path (output norm + head + argmax) write slots 0
 * (start), 1 (activations staged), 2 (head tiles done), 3 (end).  Each layer
 * launch of a layered step (per effective layer: QKV (+ attention), O,
 * gate_up, down, in launch order; launch i) writes 12 entries from
 * 4 G + 12 i, each an atomic maximum over its CTAs (thread 0), so the caller
 * zeroes them before the step: 0 the earliest CTA start, stored complemented
 * (~t); 1 the latest CTA start; 2 the latest return from the wait for the
 * previous kernel; 3 and 4 GEMV: weights arrived, main loop done; clustered
 * QKV + attention: q/k/v exchanged, attention partials exchanged; 5 the
 * latest CTA end; 6 and 7 GEMV: activations staged, unused; clustered:
 * arrival at the q/k/v and at the partials exchange barrier; 8 to 11
 * clustered only: rows normalised, weights arrived, GEMV reduced, cached
 * keys arrived.  A decode graph captured while a buffer is set keeps
 * writing to that buffer. */
tl_status tl_model_set_trace(tl_model *m, unsigned long long *d_buf, long long n_entries);
int tl_model_trace_grid(const tl_model *m);

/* Test hook with no counterpart in the pages: exercises the bounded waits.
 * With extra_arrivals = 1, every grid barrier of the following
 * TL_DECODE_FUSED steps waits for one CTA more than the step launches, so
 * the first barrier's wait runs out after its time limit (0.5 s of
 * %globaltimer), the CTA that gives up tells the others to stop waiting, the
 * step finishes with invalid results and tl_check_device_error() returns
 * TL_ERR_DEVICE_FLAG ("a kernel's bounded wait gave up").  The barrier words
 * are reset at the end of the launch as usual, so after
 * tl_model_set_wait_test(m, 0) the next steps are correct again (re-prefill
 * the lanes whose caches the invalid step wrote).  Other paths ignore it. */
tl_status tl_model_set_wait_test(tl_model *m, int extra_arrivals);

/* Measurement and tuning control with no counterpart in the pages: causal
 * prefill attention (prefill, tl_extend, tl_op_gqa_prefill) runs on the
 * tcgen05 kernel (128-query tiles, TMEM accumulators) for passes of at least
 * min_queries queries and on 16-query mma.sync tiles below that.  Process
 * wide; default 1024 (measured: below it the 16-query tiles are faster on
 * B200, from it the tcgen05 kernel).  Both kernels compute the same
 * attention. */
tl_status tl_set_prefill_attention_tc_min(int min_queries);

/* Number of kernels this library has launched in the process so far. */
unsigned long long tl_kernel_launch_count(void);

/* ------------------------------------------------------------------------
 * Op API: the hot-path kernels on caller-provided tensors
 * ------------------------------------------------------------------------ */

/* An INT4 linear (storage format above, HOST memory) copied to `device` and
 * re-laid out for the kernels.  K is a multiple of 128 and 128 <= K <= 16384;
 * 1 <= N <= 65536.  The host arrays may be freed when this returns. */
tl_status tl_linear_create(const tl_int4_linear *w, int K, int N, int device,
                           tl_linear **out);
/* tl_linear_create for an INT2 linear (the 2-bit storage described above). */
tl_status tl_linear_create_int2(const tl_int4_linear *w, int K, int N, int device,
                                tl_linear **out);
void tl_linear_destroy(tl_linear *l);

/* Kernel family used by tl_linear_forward. */
typedef enum {
  TL_PATH_AUTO = 0,   /* GEMV for M <= 16, tensor-core GEMM otherwise */
  TL_PATH_GEMV = 1,   /* INT4 GEMV on mma.sync, any M (16 rows per launch) */
  TL_PATH_TC = 2      /* INT4 GEMM on tcgen05 tensor cores, any M */
} tl_path;

/* y = x W^T with fp32 accumulation (dequantisation w = (q - z) * s).
 *   d_x  fp16 [M][K] row-major, d_y fp16 [M][N] row-major, M >= 1.
 * Returns TL_ERR_UNSUPPORTED if `path` is not built for this shape. */
tl_status tl_linear_forward(tl_linear *l, const uint16_t *d_x, int M, uint16_t *d_y,
                            int path, void *stream);

/* RMSNorm (tiny-llm feature list, "Root Mean Square Normalizations"):
 * y[r][i] = fp16(x[r][i] / sqrt(mean_i(x[r][i]^2) + eps) * g[i]).
 *   d_x fp32 [rows][d], d_g fp16 [d], d_y fp16 [rows][d]; d a multiple of 8. */
tl_status tl_op_rmsnorm(const float *d_x, const uint16_t *d_g, int rows, int d, float eps,
                        uint16_t *d_y, void *stream);

/* In-place rotary embedding of Q or K (TinyLoop README, "Status", RoPE, fused
 * in-place Q/K rotation with configurable theta).  Token t, head h starts at
 * d_x + t*token_stride + h*head_stride (fp16 elements); element j and
 * j + head_dim/2 rotate by angle pos[t] * theta^(-2j/head_dim).
 *   d_positions int32 [n_tokens], each >= 0; head_dim even, <= 256. */
tl_status tl_op_rope(uint16_t *d_x, int n_tokens, int n_heads, int head_dim,
                     long long token_stride, long long head_stride,
                     const int32_t *d_positions, float theta, void *stream);

/* Single-query cached-decode GQA attention (TinyLoop README, "Current Runtime
 * Snapshot", direct single-query decode kernel; "Status", GQA).  For batch
 * entry b the keys and values are the planes
 *   K_b = d_k + b*batch_stride, V_b = d_v + b*batch_stride,
 * each laid out [n_kv_heads][ctx_stride][head_dim] fp16 and already rotated;
 * query b (fp16 [n_q_heads][head_dim] at d_q + b*n_q_heads*head_dim, already
 * rotated) attends to keys 0..n_keys[b]-1.  q head h reads kv head
 * h / (n_q_heads/n_kv_heads); scale 1/sqrt(head_dim).
 *   h_n_keys  int32 [B] HOST, 1 <= n_keys[b] <= ctx_stride
 *   d_out     fp16 [B][n_q_heads][head_dim]
 * Uses a library-owned device workspace (allocated on first use, grown as
 * needed) for the split-KV partial results. */
tl_status tl_op_gqa_decode(const uint16_t *d_q, const uint16_t *d_k, const uint16_t *d_v,
                           long long batch_stride, int ctx_stride, const int32_t *h_n_keys,
                           int B, int n_q_heads, int n_kv_heads, int head_dim,
                           uint16_t *d_out, void *stream);

/* tl_op_gqa_decode without any allocation.  The pages have no counterpart to
 * this entry point; it exists for callers that cannot call cudaMalloc, such as
 * a serving host that plans every device byte up front and owns the
 * allocator, or a plug-in running inside another runtime whose allocator owns
 * the device memory.
 * Same arguments, layout and result as tl_op_gqa_decode, but its scratch (row
 * descriptors, split-KV partial results and merge tickets) lives in one
 * fixed 4 MiB device array that every GPU loading this library reserves until
 * the process exits; nothing is allocated or freed by the call.
 *   Limits: 1 <= B <= 32, B * n_kv_heads <= 4096, and
 *   B * n_kv_heads * 32 * (n_q_heads/n_kv_heads) * (head_dim + 4) * 4 bytes
 *   + 17 KiB <= 4 MiB (e.g. B = 8, 16/4 heads of 128 needs about 2.1 MiB);
 *   beyond them it returns TL_ERR_UNSUPPORTED and enqueues nothing.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it for the
 * life of the process (a cudaDeviceReset makes the cached address stale; do
 * not call this entry point on a device after resetting it).  All calls
 * share the one array and it
 * keeps the last call's contents (each call re-zeroes what must start at
 * zero), so calls whose work overlaps on the GPU (different streams without
 * ordering between them) race and corrupt each other's results: order them on
 * one stream or with events. */
tl_status tl_op_gqa_decode_noalloc(const uint16_t *d_q, const uint16_t *d_k, const uint16_t *d_v,
                                   long long batch_stride, int ctx_stride, const int32_t *h_n_keys,
                                   int B, int n_q_heads, int n_kv_heads, int head_dim,
                                   uint16_t *d_out, void *stream);

/* Causal tiled prefill GQA attention (TinyLoop README, "Current Runtime
 * Snapshot", tiled prefill path; tiny-llm feature list, "Tiled Online
 * Softmax", "Causal Masking").  Queries d_q fp16 [B][T][n_q_heads][head_dim]
 * (rotated) at positions pos0..pos0+T-1 attend to keys 0..pos0+t of the planes
 * described as in tl_op_gqa_decode.  d_out fp16 [B][T][n_q_heads][head_dim].
 * pos0 + T <= ctx_stride. */
tl_status tl_op_gqa_prefill(const uint16_t *d_q, const uint16_t *d_k, const uint16_t *d_v,
                            long long batch_stride, int ctx_stride, int T, int pos0, int B,
                            int n_q_heads, int n_kv_heads, int head_dim, uint16_t *d_out,
                            void *stream);

/* The INT8 KV quantisation of tl_config.kv_mode = TL_KV_INT8, as the model's
 * prefill writes it: n vectors of head_dim fp32 elements
 *   d_x fp32 [n][head_dim] -> d_codes int8 [n][head_dim], d_scales fp32 [n]
 * with scale = max|x| / 127 and code = round-half-even(x / scale) (0 for an
 * all-zero vector), both in fp32.  head_dim 64 or 128; n >= 0 (0 enqueues
 * nothing).  Device pointers; TL_ERR_INVALID_ARG for a NULL pointer or n < 0,
 * TL_ERR_UNSUPPORTED for another head_dim. */
tl_status tl_op_kv_quant_int8(const float *d_x, int n, int head_dim, int8_t *d_codes, float *d_scales,
                              void *stream);

/* ------------------------------------------------------------------------
 * Misc
 * ------------------------------------------------------------------------ */

/* Static string naming a status. */
const char *tl_status_string(tl_status s);

/* One-line reason for the last non-OK status returned on the calling thread
 * (empty string if none).  Valid until the next call on that thread. */
const char *tl_last_error(void);

/* Library version, e.g. "0.1.0". */
const char *tl_version(void);

/* Measurement helper with no counterpart in the pages: read bandwidth of a
 * device buffer.  One launch (one CTA per SM x 4, 512 threads, 8 independent
 * 16-byte loads in flight per thread, loads that skip L1) sweeps the `bytes`
 * (a multiple of 16, >= 16) of d_buf `reps` times (1..100000), after one
 * untimed launch of 3 sweeps, on `stream`; it is timed with CUDA events and
 * *h_gbs = bytes x reps / time in GB/s; the stream is synchronised.  Because
 * the sweeps repeat inside one launch, launch overhead does not count.  A
 * buffer of about half the L2 size measures L2 read bandwidth, one well over
 * it HBM read bandwidth.  The buffer is only read. */
tl_status tl_probe_read_bandwidth(const void *d_buf, size_t bytes, int reps, void *stream,
                                  double *h_gbs);

#ifdef __cplusplus
}
#endif
#endif /* TL_H_ */
