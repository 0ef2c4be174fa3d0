/*
 * dec.h -- C ABI of the B200 (sm_100a) greedy decode-step library (libdec.so).
 *
 * The library computes one autoregressive greedy decode step of a Qwen3-style
 * decoder for a batch of sequences: embedding, RMSNorm, QKV projection,
 * per-head q/k RMSNorm, rotary embedding, KV-cache append, grouped-query
 * attention over the cached context, o_proj + residual, SwiGLU MLP + residual,
 * final norm, lm_head and argmax.  The pages this follows:
 *   - "Qwen3-ASR -- Latency & Bottleneck Analysis", 03 Decode (module list and
 *     the 18.58 ms/token split), 07 Root causes (q/k/v projections, repeat_kv,
 *     QK^T, mask, fp32 softmax, AV, o_proj; RMSNorm fp32 up-cast).
 *   - "Can CTC make Qwen3-ASR faster?", 03 Greedy exactness (emit the argmax)
 *     and 11 Phase A step 1 (a one-token decode exposing the cache, its
 *     length and the logits).
 *   - faster-qwen-asr GB10 benchmark record, notes.configuration (the token,
 *     mask and position are fed back on the device: out_ids may alias the
 *     next step's token_ids).
 *   - Baseten Qwen3-ASR article, "Minimizing host-to-device syncs" (sequence
 *     lengths are owned by the host; no step reads device data back) and
 *     "KV cache quantization" (an FP8 cache, attention math in full
 *     precision).
 *   - faster-qwen-asr GB10 benchmark record, "cuda_graph_int8" entries
 *     (int8 weight-only text decoder and lm_head: dec_init_int8).
 *
 * Conventions.  Every pointer is a DEVICE pointer unless its comment says
 * "host".  `stream` is a cudaStream_t (NULL = the legacy default stream).
 * Calls that take a stream are asynchronous on it unless noted.  Return values
 * are DEC_OK (0) or a negative dec_status; nothing is written on error.
 * A handle is not thread-safe: calls on one handle must be serialised (one
 * stream at a time).  The caller owns every buffer it passes (weights, KV,
 * token/position/output arrays) and keeps them alive while the handle or an
 * enqueued step uses them; the library owns only the handle and its
 * workspace.
 *
 * Numerics: bf16 weights and cache, fp32 activations and accumulation, fp32
 * softmax; RMSNorm eps and rope theta from dec_shape.  Readings of the pages
 * taken by this library (the pages are silent on them):
 *   - q/k RMSNorm per head after the projection, before the rotation; one
 *     gain vector [head_dim] shared by all heads;
 *   - rotate-half RoPE pairing (i, i + head_dim/2) with
 *     inv_freq_i = theta^(-2i/head_dim) and angle p * inv_freq_i in fp32
 *     (for a text decode step the three MRoPE sections share the position);
 *   - query head h reads KV head floor(h * n_kv_heads / n_q_heads) (each KV
 *     head serves n_q_heads/n_kv_heads consecutive query heads);
 *   - attention scale 1/sqrt(head_dim), causal over rows 0..p inclusive (the
 *     new token attends to itself), no biases, no sliding window;
 *   - argmax ties go to the lowest token id;
 *   - FP8 cache: OCP E4M3 codes with one fp32 scale per (layer, K/V, sequence,
 *     KV head, token): scale = max(amax, 2^-126)/448, code = RNE-satfinite of
 *     x/scale, both in fp32;
 *   - int8 weights: one fp32 scale per output row, scale = amax/127,
 *     code = round-half-even(w/scale), both in fp32, clamped to [-127, 127].
 */
#ifndef DEC_H
#define DEC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ */
/* Status codes                                                        */
/* ------------------------------------------------------------------ */
typedef enum dec_status {
  DEC_OK = 0,
  DEC_ERR_NULL = -1,          /* a required pointer is NULL */
  DEC_ERR_SHAPE = -2,         /* unsupported or inconsistent shape */
  DEC_ERR_BATCH = -3,         /* batch < 1 or > max_batch / kv batch */
  DEC_ERR_KV_SIZE = -4,       /* KV buffer smaller than dec_kv_bytes() */
  DEC_ERR_DTYPE = -5,         /* unsupported KV dtype */
  DEC_ERR_ALIGN = -6,         /* pointer not aligned as documented */
  DEC_ERR_CUDA = -7,          /* a CUDA runtime call failed (dec_last_cuda_error) */
  DEC_ERR_DEVICE = -8,        /* the current device is not sm_100 or lacks resources */
  DEC_ERR_ARG = -9,           /* other invalid argument */
  DEC_ERR_TOO_LARGE = -10,    /* problem exceeds dec_attention_noalloc's fixed scratch */
  /* device-detected conditions, returned (OR-ed as a positive bit set) by
   * dec_check(); the step that saw them wrote -1 to every out_ids entry */
  DEC_DEV_BAD_POSITION = 1,   /* a position < 0 or >= max_ctx */
  DEC_DEV_BAD_TOKEN = 2,      /* a token id < 0 or >= vocab */
  DEC_DEV_TIMEOUT = 4         /* a bounded device wait ran out (see dec_set_timeout_ns) */
} dec_status;

/* ------------------------------------------------------------------ */
/* Model description                                                   */
/* ------------------------------------------------------------------ */
typedef struct dec_shape {
  int n_layers;      /* 1..64 (28 for the 0.6B / 1.7B decoders) */
  int hidden;        /* multiple of 256 */
  int n_q_heads;     /* multiple of n_kv_heads */
  int n_kv_heads;
  int head_dim;      /* 64 or 128 */
  int ffn;           /* multiple of 256 */
  int vocab;
  float rms_eps;     /* 1e-6 */
  float rope_theta;  /* 1e6 */
  int max_batch;     /* largest batch dec_step will be called with, 1..64.
                      * Batches of 1..4 run the single persistent kernel; a
                      * handle with max_batch > 4 also plans the batched
                      * (tensor-core) step for batches of 5..max_batch, which
                      * needs n_q_heads*head_dim and n_kv_heads*head_dim to be
                      * multiples of 128, ffn a multiple of 64 and at most 4
                      * query heads per KV head (else DEC_ERR_SHAPE) */
} dec_shape;

/* Order of the per-layer weight pointers in dec_weights.layers. */
typedef enum dec_layer_weight {
  DEC_LW_IN_NORM = 0,  /* bf16 [hidden]                    input RMSNorm gain  */
  DEC_LW_Q,            /* bf16 [n_q_heads*head_dim, hidden]  row-major, y = W x */
  DEC_LW_K,            /* bf16 [n_kv_heads*head_dim, hidden]                    */
  DEC_LW_V,            /* bf16 [n_kv_heads*head_dim, hidden]                    */
  DEC_LW_Q_NORM,       /* bf16 [head_dim]                  per-head q gain     */
  DEC_LW_K_NORM,       /* bf16 [head_dim]                  per-head k gain     */
  DEC_LW_O,            /* bf16 [hidden, n_q_heads*head_dim]                     */
  DEC_LW_POST_NORM,    /* bf16 [hidden]                    post-attn RMSNorm   */
  DEC_LW_GATE,         /* bf16 [ffn, hidden]                                    */
  DEC_LW_UP,           /* bf16 [ffn, hidden]                                    */
  DEC_LW_DOWN,         /* bf16 [hidden, ffn]                                    */
  DEC_LW_COUNT
} dec_layer_weight;

typedef struct dec_weights {
  const void *embed;        /* bf16 [vocab, hidden] */
  const void *lm_head;      /* bf16 [vocab, hidden]; may equal embed (tied) */
  const void *final_norm;   /* bf16 [hidden] */
  /* HOST array of n_layers * DEC_LW_COUNT device pointers, layer-major in
   * dec_layer_weight order; copied by dec_init, may be freed afterwards.
   * Every weight pointer must be 16-byte aligned. */
  const void *const *layers;
} dec_weights;

typedef struct dec_handle dec_handle;

/* Create a handle for the current CUDA device (the pages define no API: this
 * call, like dec_kv_bytes, dec_kv_alloc and dec_check, is the library's own
 * boundary around the step they describe).  Validates the shape, copies
 * the weight pointer table (not the weights: they stay caller-owned and must
 * stay alive and unchanged), allocates the workspace (activation exchange
 * buffers, attention partials, counters; a few MB) and picks the kernel
 * configuration.  The step time depends by a few per cent on where the
 * workspace lands in device memory, so dec_init times a few batch-1 steps
 * (on a scratch cache of zeros) in each of several candidate workspaces and
 * keeps the fastest: it runs the weights it is given, which must therefore
 * be valid device memory already.  Synchronous.  Returns DEC_ERR_SHAPE for
 * unsupported shapes and DEC_ERR_DEVICE if the device is not compute
 * capability 10.0. */
int dec_init(const dec_shape *shape, const dec_weights *weights, dec_handle **out);

/* Weight-only int8 model (faster-qwen-asr GB10 benchmark record,
 * "cuda_graph_int8" entries of the 0.6B and 1.7B models: int8 weight-only
 * quantisation of the text decoder and lm_head).  The seven projections of
 * every layer (DEC_LW_Q, _K, _V, _O, _GATE, _UP, _DOWN) and lm_head are int8
 * codes [out, in] (row-major, like the bf16 tensors they replace) with one
 * fp32 scale per output row; the weight the step multiplies is code * scale
 * (dec_quantize_int8 makes both from bf16).  The embedding and the norm
 * gains stay bf16. */
typedef struct dec_weights_int8 {
  const void *embed;           /* bf16 [vocab, hidden] */
  const void *lm_head;         /* int8 [vocab, hidden] codes, 16-byte aligned */
  const float *lm_head_scale;  /* fp32 [vocab] */
  const void *final_norm;      /* bf16 [hidden] */
  /* HOST array of n_layers * DEC_LW_COUNT device pointers in dec_layer_weight
   * order: bf16 norm gains, int8 codes for the projections; every pointer
   * 16-byte aligned.  Copied by dec_init_int8. */
  const void *const *layers;
  /* HOST array of n_layers * DEC_LW_COUNT device pointers: the fp32 row
   * scales [out] of each projection (4-byte aligned); the norm slots are
   * ignored (may be NULL).  Copied by dec_init_int8. */
  const float *const *scales;
} dec_weights_int8;

/* dec_init for a weight-only int8 model.  Same ownership, errors and
 * max_batch range (1..64) as dec_init.  Batches of 1..4 run on the single
 * persistent kernel (int8 rows in its ring, CUDA-core dot products); batches
 * of 5..64 on the batched step, whose tensor-core GEMMs stage each int8
 * weight tile by TMA and widen it to a bf16 operand tile in shared memory
 * (codes up to 127 are exact in bf16), with the row scale applied to the
 * fp32 accumulator.  dec_step, dec_step_host, dec_generate and dec_verify
 * work as with bf16 weights. */
int dec_init_int8(const dec_shape *shape, const dec_weights_int8 *weights, dec_handle **out);

/* Weight-only E4M3 model ("Qwen3-ASR -- Latency & Bottleneck Analysis", 08
 * Optimization roadmap: an fp8 lm_head; the same scheme for the
 * projections).  The same dec_weights_int8 layout, with OCP E4M3 codes in
 * place of the int8 codes of the projections and lm_head (dec_quantize_fp8w
 * makes them from bf16); the weight the step multiplies is e4m3(code) *
 * scale.  Same ownership, errors, max_batch range and paths as
 * dec_init_int8. */
int dec_init_fp8w(const dec_shape *shape, const dec_weights_int8 *weights, dec_handle **out);

/* Release the handle and its workspace (synchronises the device first). */
void dec_free(dec_handle *h);

/* ------------------------------------------------------------------ */
/* KV cache                                                            */
/* ------------------------------------------------------------------ */
typedef enum dec_kv_dtype { DEC_KV_BF16 = 0, DEC_KV_FP8_E4M3 = 1 } dec_kv_dtype;

/* A KV cache bound to a caller buffer.  Layout (fixed, so that a caller can
 * prefill it):
 *   bf16: values  [n_layers][2 (K,V)][batch][n_kv_heads][max_ctx][head_dim]
 *   fp8 : codes   [n_layers][2][batch][n_kv_heads][max_ctx][head_dim] (uint8)
 *         then, at byte offset dec_kv_scale_offset(), fp32 scales
 *               [n_layers][2][batch][n_kv_heads][max_ctx]
 * Row p of (layer, K/V, b, head) holds the key / value of the token at
 * position p of sequence b (after q/k norm and rotation for K). */
typedef struct dec_kv {
  void *base;         /* device, 256-byte aligned */
  size_t bytes;
  int batch;
  int max_ctx;
  int dtype;          /* dec_kv_dtype */
} dec_kv;

/* Bytes a cache of this size needs (0 for an invalid request).  No page
 * defines this call; the layout above is the library's own. */
size_t dec_kv_bytes(const dec_handle *h, int batch, int max_ctx, int dtype);

/* Byte offset of the fp32 scale array inside an fp8 cache (0 for bf16). */
size_t dec_kv_scale_offset(const dec_handle *h, int batch, int max_ctx, int dtype);

/* Bind a caller-owned device buffer as a KV cache (no page defines this call;
 * the caller owning the cache follows the Baseten article's host-owned
 * sequence state, "Minimizing host-to-device syncs").  Allocates nothing and
 * does not touch the buffer's contents.  DEC_ERR_KV_SIZE if buf_bytes <
 * dec_kv_bytes(), DEC_ERR_ALIGN unless buf is 256-byte aligned. */
int dec_kv_alloc(dec_handle *h, int batch, int max_ctx, int dtype, void *buf,
                 size_t buf_bytes, dec_kv *out);

/* ------------------------------------------------------------------ */
/* Decode step                                                         */
/* ------------------------------------------------------------------ */

/* One greedy decode step for sequences 0..batch-1 of `kv`.
 *   token_ids  int32 [batch]  the current token of every sequence
 *   positions  int32 [batch]  p_b: the row the new K/V are written to; the
 *                             step attends over rows 0..p_b.  The caller
 *                             (host) owns the lengths: it writes positions
 *                             every step; the library never reads them back.
 *   out_ids    int32 [batch]  argmax token of every sequence; may alias
 *                             token_ids (self-feeding decode).
 *   out_logits fp32 [batch, vocab] or NULL.
 * Asynchronous on `stream`; never synchronises.  Batches of 1..4: one
 * kernel launch.  Batches of 5..64: 5 launches per layer + 3 (programmatic
 * dependent launches, so the caller's stream must not be shared with work
 * that expects the step to be a single kernel).  Invalid positions or
 * tokens are detected on the device: the step then writes -1 to out_ids,
 * leaves the cache unchanged and raises a bit that dec_check() returns. */
int dec_step(dec_handle *h, int batch, const int32_t *token_ids, const int32_t *positions,
             const dec_kv *kv, int32_t *out_ids, float *out_logits, void *stream);

/* n greedy steps on the device, the host out of the loop (faster-qwen-asr
 * GB10 record, notes.configuration: token fed back on the device; Baseten
 * article, "Minimizing host-to-device syncs").
 *   token_ids  int32 [batch] (device)   the current tokens
 *   positions  int32 [batch] (device)   the rows the first step writes;
 *                                       advanced IN PLACE after every step
 *   out_ids    int32 [n_steps][batch]   step i's ids (the input of step i+1)
 *   eos        end-of-sequence id in [0, vocab), or -1 for none.  A sequence
 *              that emits it is retired: its position stays at the row of
 *              that step, its later outputs are eos and no later step writes
 *              its cache.
 * Equivalent to n_steps dec_step calls that feed out_ids back and advance the
 * positions by one.  Batches of 1..4 run as ONE launch of the persistent
 * kernel, which loops over the steps itself; once every sequence has retired
 * it stops early (the remaining out_ids rows are eos).  A sequence whose next
 * position would reach max_ctx stops the loop: DEC_DEV_BAD_POSITION, and the
 * steps that could not run report -1.  Batches of 5..64 launch the batched
 * step once per step with a small bookkeeping kernel in between.
 * Asynchronous (no host read-back inside); other device errors as in dec_step
 * (dec_check). */
int dec_generate(dec_handle *h, int batch, int n_steps, const int32_t *token_ids,
                 int32_t *positions, const dec_kv *kv, int32_t *out_ids, int eos, void *stream);

/* ------------------------------------------------------------------ */
/* Block verification and greedy acceptance (speculative decoding)     */
/* ------------------------------------------------------------------ */

/* Verify a block of k consecutive tokens of ONE cached sequence in a single
 * step ("Can CTC make Qwen3-ASR faster?", §11 Phase A steps 2-3: one target
 * forward over the whole draft block; §03: greedy verification).  A block
 * of one token runs as one launch of the persistent kernel; so do blocks of
 * 2 to 4 (with k * n_q_heads / n_kv_heads <= 8) on a handle without a
 * batched step (max_batch <= 4, and every int8 handle), the committed prefix
 * of the sequence read once for the whole block.  Other blocks run the
 * batched step, as fast or faster than the persistent kernel from 2 tokens
 * on.
 *   token_ids  int32 [k] (device)  t_0 = the last committed token, then the
 *                                  draft tokens t_1 .. t_{k-1}
 *   positions  int32 [k] (device)  p0 + i: row i is written to cache row
 *                                  p0 + i of sequence `seq` and attends rows
 *                                  0 .. p0 + i (so the block is causal among
 *                                  itself)
 *   out_ids    int32 [k]           out_ids[i] = greedy next token after t_i
 *                                  (the prediction that checks t_{i+1});
 *                                  may alias token_ids
 *   out_logits fp32 [k, vocab] or NULL.
 * Results equal k single-sequence steps fed t_0 .. t_{k-1} (up to rounding).
 * Needs 1 <= k <= max_batch; blocks the persistent kernel does not take need
 * a handle created with max_batch > 4 (DEC_ERR_BATCH otherwise).  int8
 * handles verify blocks of up to 4.  Asynchronous; invalid positions /
 * tokens, and positions that are not p0, p0 + 1, ..., behave as in dec_step
 * (DEC_DEV_BAD_POSITION).  Cache rows p0 .. p0 + k - 1 of `seq` are
 * overwritten. */
int dec_verify(dec_handle *h, int k, const int32_t *token_ids, const int32_t *positions,
               int seq, const dec_kv *kv, int32_t *out_ids, float *out_logits, void *stream);

/* Greedy acceptance of a verified block (HOST arrays, no GPU work): the
 * pages' contract ("Can CTC make Qwen3-ASR faster?", §03 and §08) — accept
 * draft token t_{i+1} only while it equals out_ids[i]; at the first mismatch
 * emit out_ids[i] instead and stop; after a full match emit the bonus token
 * out_ids[k-1].  Writes the j + 1 emitted tokens (t_1..t_j, then out_ids[j])
 * to emitted[] (room for k) and j + 1 to *n_emitted.  The cache is valid up
 * to row p0 + j; the host continues at position p0 + j + 1 with token
 * emitted[j] (rows beyond are overwritten by later steps: the crop is the
 * host's position).  DEC_ERR_ARG if out_ids holds -1 (an invalid step). */
int dec_accept_greedy(int k, const int32_t *tokens, const int32_t *out_ids, int32_t *emitted,
                      int *n_emitted);

/* dec_step plus the residual stream after the embedding and after every
 * layer: hidden_out fp32 [n_layers + 1][batch][hidden] (device). */
int dec_step_debug(dec_handle *h, int batch, const int32_t *token_ids,
                   const int32_t *positions, const dec_kv *kv, int32_t *out_ids,
                   float *out_logits, float *hidden_out, void *stream);

/* dec_step with HOST inputs and outputs: copies token_ids / positions (host,
 * int32 [batch]) to the device, runs the step, copies out_ids (host) and, if
 * non-NULL, out_logits (host, fp32 [batch, vocab]) back, and synchronises
 * `stream` before returning. */
int dec_step_host(dec_handle *h, int batch, const int32_t *token_ids_host,
                  const int32_t *positions_host, const dec_kv *kv, int32_t *out_ids_host,
                  float *out_logits_host, void *stream);

/* (No page defines this call: it reports the conditions the device detected
 * without any read-back inside a step.)
 * Synchronise `stream`, then return and clear the device status bits
 * (DEC_DEV_*; 0 when every step since the last check was clean), or a
 * negative dec_status if the synchronisation itself failed. */
int dec_check(dec_handle *h, void *stream);

/* Bound of every device-side wait, in nanoseconds (default 2e9).  A wait
 * that runs out sets DEC_DEV_TIMEOUT, the step drains its copies in flight
 * and returns with out_ids = -1; the context stays usable. */
int dec_set_timeout_ns(dec_handle *h, unsigned long long ns);

/* Test hook: 0 = normal; k > 0 makes CTA k-1 skip publishing its share of the
 * first layer's o_proj output, so that every other CTA's bounded wait on it
 * runs out (exercises the timeout path without any fault). */
int dec_set_debug_stall(dec_handle *h, int cta_plus_one);

/* Human-readable name of a dec_status value or DEC_DEV_* bit set. */
const char *dec_error_string(int code);

/* The last CUDA error code a call on any handle saw (cudaError_t as int). */
int dec_last_cuda_error(void);

/* Kernel configuration chosen by dec_init (for reports): CTAs per step,
 * ring slots per CTA and slot bytes. */
int dec_get_config(const dec_handle *h, int *ctas, int *ring_slots, int *slot_bytes);

/* ------------------------------------------------------------------ */
/* Isolated grouped-query decode attention                             */
/* ------------------------------------------------------------------ */

/* Split-K (flash-decoding) GQA attention of one query token per sequence over
 * its cached rows, fp32 softmax ("Latency & Bottleneck Analysis", 07 Root
 * causes: repeat_kv, QK^T, mask, fp32 softmax, AV in one kernel instead of
 * ~10 launches per layer):
 *   out[b, h, :] = sum_j softmax_j(q[b,h,:] . K[b,g,j,:] / sqrt(head_dim)) V[b,g,j,:],
 *   g = floor(h * n_kv_heads / n_q_heads), j = 0 .. lengths[b]-1.
 *   q          bf16 [batch, n_q_heads, head_dim]
 *   k_cache,
 *   v_cache    bf16 [batch, n_kv_heads, max_len, head_dim] (rows >= lengths[b]
 *              are not read)
 *   lengths    int32 [batch] (device), each in [1, max_len]
 *   out        fp32 [batch, n_q_heads, head_dim]
 *   workspace  device scratch of dec_attention_workspace_bytes() bytes,
 *              256-byte aligned, zero-filled by the caller before its first
 *              use; every completed call leaves it ready for the next one
 *              (calls sharing one workspace must not overlap on the GPU).
 * head_dim 64 or 128; n_q_heads/n_kv_heads <= 8.  Lengths outside [1,
 * max_len] raise DEC_DEV_BAD_POSITION in `status` (device int, may be NULL)
 * and that sequence's output is left untouched. */
size_t dec_attention_workspace_bytes(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                     int max_len);
int dec_attention(int batch, int n_q_heads, int n_kv_heads, int head_dim, const void *q,
                  const void *k_cache, const void *v_cache, int max_len,
                  const int32_t *lengths, float *out, void *workspace,
                  size_t workspace_bytes, int *status, void *stream);

/* dec_attention without a workspace argument: for callers that must not
 * allocate device memory on their call path -- code running inside another
 * framework's execute or enqueue callback, where allocating is not permitted;
 * real-time loops, where cudaMalloc's implicit synchronisation would stall the
 * device; processes whose device memory is owned by another allocator or fixed
 * by a budget.  (The pages have no counterpart: this is a deployment variant
 * of the attention above.)
 * Same inputs, outputs and numerics as dec_attention.  The scratch (per-chunk
 * partial softmax states, per-(sequence, KV head) counters) is a fixed 4 MiB
 * device array inside the library: every GPU that loads the library holds it
 * until the process exits.  Requests needing more than 4 MiB of it (batch *
 * n_q_heads * chunks * (head_dim + 2) * 4 bytes, chunks as dec_attention
 * splits max_len, plus 4 bytes per (sequence, KV head)) return
 * DEC_ERR_TOO_LARGE; nothing is launched.  Allocates nothing: no cudaMalloc,
 * no cudaFree.  The first call on a device looks up the array's device address
 * (with that device current) and should come before any stream capture.  All
 * calls on a device share the array and each clears its counters first, so
 * calls that overlap on the GPU (other streams, or other host threads) race:
 * serialise them. */
int dec_attention_noalloc(int batch, int n_q_heads, int n_kv_heads, int head_dim, const void *q,
                          const void *k_cache, const void *v_cache, int max_len,
                          const int32_t *lengths, float *out, int *status, void *stream);

/* ------------------------------------------------------------------ */
/* int8 weights                                                        */
/* ------------------------------------------------------------------ */

/* Quantise a bf16 weight matrix w [rows, cols] (row-major, device) to int8
 * codes [rows, cols] and one fp32 scale per row (device), the format
 * dec_init_int8 reads: scale = amax/127 (IEEE fp32 division; 0 for a row of
 * zeros), code = round-half-even(w/scale) (IEEE fp32 division), clamped to
 * [-127, 127] (faster-qwen-asr GB10 record, "cuda_graph_int8": int8
 * weight-only, per output row).  cols must be a multiple of 8 (DEC_ERR_ARG);
 * w 16-byte, codes 8-byte and scales 4-byte aligned (DEC_ERR_ALIGN).
 * Asynchronous on `stream`. */
int dec_quantize_int8(const void *w, int rows, int cols, int8_t *codes, float *scales,
                      void *stream);

/* Quantise a bf16 weight matrix w [rows, cols] (row-major, device) to OCP
 * E4M3 codes [rows, cols] and one fp32 scale per row (device), the format
 * dec_init_fp8w reads: the per-row quantiser of the FP8 cache rows applied
 * to the weight row, scale = max(amax, 2^-126)/448 and code =
 * RNE-satfinite(w/scale), both divisions in IEEE fp32 ("Latency & Bottleneck
 * Analysis", 08 Optimization roadmap: fp8 lm_head).  cols must be a multiple
 * of 8 (DEC_ERR_ARG); w 16-byte, codes 8-byte and scales 4-byte aligned
 * (DEC_ERR_ALIGN).  Asynchronous on `stream`. */
int dec_quantize_fp8w(const void *w, int rows, int cols, uint8_t *codes, float *scales,
                      void *stream);

/* ------------------------------------------------------------------ */
/* FP8 cache rows                                                      */
/* ------------------------------------------------------------------ */

/* Quantise `rows` rows of `dim` (64 or 128) fp32 values to OCP E4M3 codes with
 * one fp32 scale per row, exactly as dec_step stores the rows it appends to an
 * FP8 cache (Baseten Qwen3-ASR article, KV cache quantization: FP8 storage,
 * full-precision attention math): scale = max(amax, 2^-126)/448 and
 * code = RNE-satfinite(x/scale), both divisions in IEEE fp32.  Use it to fill
 * an FP8 cache from a bf16/fp32 prefill.  x fp32 [rows, dim], codes uint8
 * [rows, dim], scales fp32 [rows] (all device).  Asynchronous on `stream`. */
int dec_kv_quantize_e4m3(const float *x, int rows, int dim, uint8_t *codes, float *scales,
                         void *stream);

#ifdef __cplusplus
}
#endif
#endif /* DEC_H */
