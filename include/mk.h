/*
 * mk.h -- C ABI of the single-launch decode engine for hybrid
 * Gated-DeltaNet + full-attention language models on NVIDIA B200 (sm_100a).
 *
 * The operation behind every entry point is one token's (or a few tokens')
 * forward pass of the hybrid stack described in the launch post "OS
 * Megakernel that match M5 Max Tok/w at 2x the Throughput on RTX 3090"
 * (paragraph "Why nobody had done this yet?": DeltaNet layers with a
 * learned recurrence interleaved with full-attention layers; the kernel
 * bullet list: one dispatch for the whole forward pass, bf16 weights,
 * fp32 accumulation, fused QKV + RoPE + causal softmax + output
 * projection; the post synchronises the grid between layers, this engine
 * lets each CTA wait for exactly the data it needs instead).  The
 * recurrence is the gated delta rule of "Gated Delta Networks" (Yang,
 * Kautz & Hatamizadeh, ICLR 2025).
 *
 * Conventions shared by all entry points
 *  - Every pointer documented as "device" must point to memory of the CUDA
 *    device that was current when mk_create ran; "host" pointers are read
 *    before the call returns.
 *  - Calls are asynchronous on the stream given to mk_create unless stated.
 *  - Nothing throws across the ABI.  Every call returns an mk_status code;
 *    MK_OK is 0.  A device-side failure (a wait for another CTA's data or
 *    a pipeline wait that ran out of time) is recorded in a device error
 *    word and reported by mk_sync() until mk_reset() clears it; results of
 *    calls made after such an error are undefined until then.  mk_reset()
 *    clears the error, the recurrent state and the KV cache.
 *  - Tensors are row-major.  bf16 values are IEEE bfloat16 bit patterns.
 */
#ifndef MK_H
#define MK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MK_MAX_LAYERS 64

typedef enum {
  MK_OK = 0,
  MK_ERR_ARG = 1,          /* bad argument, shape, alignment or NULL        */
  MK_ERR_CTX_OVERFLOW = 2, /* the call would write past max_ctx             */
  MK_ERR_STATE = 3,        /* call not valid in the engine's current state  */
  MK_ERR_LAUNCH = 4,       /* cooperative launch impossible / failed        */
  MK_ERR_TIMEOUT = 5,      /* a device-side wait gave up (error word set)   */
  MK_ERR_CUDA = 6,         /* another CUDA runtime error                    */
  MK_ERR_UNSUPPORTED = 7,  /* shape outside what the kernels implement      */
  MK_ERR_RANGE = 8         /* a decode partial sum left the fixed-point range
                              of the split-K reduction (|value| >= 8192)     */
} mk_status;

/* Model shape.  Layer l is full attention when layer_is_attn[l] != 0 and a
 * Gated-DeltaNet layer otherwise.  Shapes the decode kernel is built for:
 * hidden % 256 == 0 and <= 2048; conv_k == 4; mlp % 8 == 0 and <= 4096; the embedding
 * tied to the LM head; q_heads == 4 * kv_heads; and (dn_dk == dn_dv,
 * head_dim) one of (64, 64), (128, 128), (128, 256); mlp and
 * q_heads * head_dim divisible by dn_heads (the decode groups' K blocks,
 * each a multiple of 8 and the attention block at most 256 wide); at least
 * one SM per DeltaNet head.  mk_create returns MK_ERR_UNSUPPORTED otherwise
 * (also when a CTA's share of a phase exceeds the kernel's shared-memory
 * staging). */
typedef struct {
  int32_t n_layers;
  uint8_t layer_is_attn[MK_MAX_LAYERS];
  int32_t hidden, vocab, mlp;
  int32_t dn_heads, dn_dk, dn_dv, conv_k;
  int32_t q_heads, kv_heads, head_dim;
  float rope_theta, rms_eps;
  int32_t max_ctx;     /* KV-cache capacity in positions                    */
  int32_t max_verify;  /* most tokens one mk_verify call may carry (<= 8)   */
} mk_config;

/* Device pointers of one layer's weights.  bf16 matrices are [out][in];
 * every pointer must be 16-byte aligned.  Members of the other layer kind
 * are ignored and may be NULL.
 *   attn_norm [H], mlp_norm [H]            pre-mixer / pre-MLP RMSNorm gains
 *   in_proj   [2*nh*dk + 2*nh*dv + 2*nh][H] DeltaNet rows q | k | v | z | b | a
 *   conv_w    [2*nh*dk + nh*dv][conv_k]    causal conv taps of q | k | v
 *   A_log, dt_bias [nh] (float32)          decay parameters
 *   out_norm  [dv]                         gated-RMSNorm gain (shared by heads)
 *   out_proj  [H][nh*dv]                   DeltaNet output projection
 *   w_q [q_heads*hd][H], w_k, w_v [kv_heads*hd][H], w_o [H][q_heads*hd]
 *   w_gate, w_up [mlp][H], w_down [H][mlp] SwiGLU MLP                      */
typedef struct {
  const void *attn_norm;
  const void *in_proj, *conv_w;
  const float *A_log, *dt_bias;
  const void *out_norm, *out_proj;
  const void *w_q, *w_k, *w_v, *w_o;
  const void *mlp_norm;
  const void *w_gate, *w_up, *w_down;
} mk_layer_weights;

/* embed [vocab][H] bf16 (also the LM head: tied), final_norm [H] bf16,
 * layers: host array of n_layers entries. */
typedef struct {
  const void *embed;
  const void *final_norm;
  const mk_layer_weights *layers;
} mk_weights;

typedef struct mk_engine mk_engine;

/* Bytes of device workspace mk_create needs for this config (recurrent
 * state buffers, verify records, KV cache, activations, exchange words, and the
 * decode kernel's copies of the layer weights, see mk_create).
 * Returns 0 for an invalid config. */
size_t mk_workspace_bytes(const mk_config *cfg);

/* Create an engine on the current CUDA device for the hybrid stack of the
 * launch post "OS Megakernel that match M5 Max Tok/w at 2x the Throughput on
 * RTX 3090" (kernel bullet list: the whole forward pass of one token in one
 * dispatch).  `workspace` (device, at
 * least mk_workspace_bytes(cfg) bytes, 256-byte aligned) and the weights
 * stay owned by the caller and must outlive the engine; the engine only
 * keeps pointers.  `cuda_stream` (a cudaStream_t, may be NULL for the
 * legacy stream) is the stream every later call runs on.  Checks that one
 * CTA of the decode kernel fits on every SM (cooperative co-residency) and
 * returns MK_ERR_LAUNCH otherwise.  Copies weights into the workspace in
 * the layouts the decode kernel's CTA groups read (one group per DeltaNet
 * head): each attention layer's w_q, w_k and w_v as one [q|k|v][hidden]
 * matrix, each DeltaNet head's in_proj rows (q|k|v|z|b|a of that head) as
 * one block, and every out_proj, w_o and w_down split into dn_heads column
 * blocks; later changes to the caller's weights need a new engine.  Zeroes
 * the state (as mk_reset). */
int mk_create(const mk_config *cfg, const mk_weights *w, void *workspace,
              size_t ws_bytes, void *cuda_stream, mk_engine **out);

/* Destroy the host handle (NULL is allowed).  Does not free caller memory. */
void mk_destroy(mk_engine *e);

/* Zero the DeltaNet and conv states, empty the KV cache, clear a device
 * error, any pending verify and any accepted positions not yet replayed:
 * the start of a new sequence (launch post,
 * "Why nobody had done this yet?": the DeltaNet layers carry a recurrent
 * state and the attention layers a KV cache from token to token).  Weights
 * are untouched. */
int mk_reset(mk_engine *e);

/* Run n prompt tokens (host array, values in [0, vocab)) through the stack
 * at positions pos .. pos+n-1 and leave the state and KV cache as n decode
 * steps would, up to rounding (launch post "OS Megakernel that match M5 Max
 * Tok/w at 2x the Throughput on RTX 3090", results table: prompt processing
 * "pp520" beside decode).  When n-1 >= 8 the first n-1 positions run as
 * chunks of up to 1024 positions: every projection one tensor-core GEMM
 * (bf16 weights; each fp32 activation as a bf16 hi + lo pair; fp32
 * accumulation), the causal conv and gated delta rule scanned position by
 * position, causal attention over cache + chunk.  The last position is
 * always one decode step, so its logits and greedy argmax come from the
 * decode kernel.  If logits_out (device, float32 [vocab]) is not NULL it
 * receives the logits of the last prompt position.  n == 0 is a no-op.
 * The host array is copied before the call returns (pageable copies
 * synchronise with the stream).  Errors: MK_ERR_ARG (token out of range),
 * MK_ERR_CTX_OVERFLOW when pos+n > max_ctx, MK_ERR_STATE while a verify is
 * pending, MK_ERR_LAUNCH / MK_ERR_CUDA on launch failures. */
int mk_prefill(mk_engine *e, const int32_t *tokens_host, int n,
               float *logits_out);

/* One decode step: the whole forward pass of `token` at the current
 * position in one cooperative launch of the persistent kernel (launch post
 * "OS Megakernel that match M5 Max Tok/w at 2x the Throughput on RTX 3090",
 * kernel bullet list: one dispatch per token instead of ~100 launches).
 * logits_out (device, float32 [vocab]) may be NULL.  The greedy argmax of
 * the step is kept on the device (see mk_generate) and can be read with
 * mk_last_argmax.  Does not synchronise the host.  Errors: MK_ERR_ARG
 * (token out of range), MK_ERR_CTX_OVERFLOW at max_ctx, MK_ERR_STATE while
 * a verify is pending, MK_ERR_LAUNCH / MK_ERR_CUDA on launch failures. */
int mk_decode_step(mk_engine *e, int32_t token, float *logits_out);

/* Greedy generation with no host round trip between tokens (the tg128
 * decode of the launch post's results table): n decode launches, the first
 * fed `first_token` (or, when first_token == -1, the device-side argmax of
 * the last decode launch, which must be at the current position: the last
 * prefill position or the last decode / generate step; MK_ERR_STATE after
 * mk_create, mk_reset, mk_set_state or mk_verify), each later one fed the
 * device-side argmax of the launch before it.  tokens_out (device, int32 [n]) receives the n argmax tokens;
 * logits_out (device, float32 [n][vocab]) may be NULL.  Other errors as
 * mk_decode_step. */
int mk_generate(mk_engine *e, int32_t first_token, int n, int32_t *tokens_out,
                float *logits_out);

/* Verify n tokens at once (1 <= n <= max_verify), the speculative-decoding
 * shape (several draft tokens checked by one forward pass, with the
 * recurrent state kept recoverable for rollback; the follow-up post
 * "업데이트: 단일 RTX 3090에서 Qwen 3.8 27B를 140 tok/s로 구동 (Megakernel:
 * KL divergence", speed list: four draft tokens checked for the cost of one
 * forward pass, greedy output unchanged): the stack runs over positions
 * pos .. pos+n-1 as one chunk -- every projection one pass over its weights
 * for the n positions, the conv and the gated delta rule advanced position
 * by position -- and writes the logits of every position to logits_out
 * (device, float32 [n][vocab], not NULL) and K/V of the n positions to the
 * cache.  Instead of the state after every position it records, per
 * DeltaNet layer and position, the normalised key, the value, alpha, beta
 * and the conv inputs (a few KB).  Positions kept by the previous
 * mk_accept are applied to the state first, inside this call.  Results
 * equal n decode steps up to rounding.  The position does not advance until
 * mk_accept.  MK_ERR_STATE while a verify is pending. */
int mk_verify(mk_engine *e, const int32_t *tokens_host, int n,
              float *logits_out);

/* Keep the first n_keep (1..n) positions of the last mk_verify and advance
 * the position by n_keep (the rollback of rejected draft tokens that exact
 * greedy speculative decoding needs; same follow-up post, accuracy
 * paragraph: greedy output stays the main model's greedy choice).  No work
 * is launched: the next call that reads the state (verify, decode,
 * generate, prefill, mk_get_state) first replays the n_keep recorded
 * positions on it, so the state after a rejected position is never
 * written.  (Without the chunk path, mk_verify falls back to one decode
 * launch per position with a full state copy after each, and mk_accept
 * selects the copy.)  MK_ERR_STATE if no verify is pending. */
int mk_accept(mk_engine *e, int n_keep);

/* Current position (number of tokens consumed). */
int mk_position(const mk_engine *e);

/* Synchronise the stream and report a recorded device-side error. */
int mk_sync(mk_engine *e);

/* Host copy of the packed argmax of the last decode/generate step:
 * the token id, or -1.  Synchronises the stream. */
int32_t mk_last_argmax(mk_engine *e);

/* Engine state I/O (checkpoint / resume and tests).  All buffers are device
 * pointers in these layouts:
 *   dn_state   [n_dn][dn_heads][dv][dk] float32
 *   conv_state [n_dn][2*nh*dk + nh*dv][conv_k-1] float32
 *   k_cache, v_cache [n_attn][kv_heads][pos][head_dim] bf16
 * mk_set_state installs a state as if `pos` tokens had been consumed;
 * mk_get_state copies the current one out (k/v caches may be NULL). */
int mk_set_state(mk_engine *e, int pos, const float *dn_state,
                 const float *conv_state, const void *k_cache,
                 const void *v_cache);
int mk_get_state(mk_engine *e, float *dn_state, float *conv_state,
                 void *k_cache, void *v_cache);

/* Residual stream after every layer for the last position processed by a
 * decode, generate or prefill call: device float32 [n_layers][hidden]. */
int mk_get_hidden(mk_engine *e, float *hidden_out);

/* Launch statistics: number of kernels the engine launched so far. */
int64_t mk_launch_count(const mk_engine *e);

/* Debug: device-side wait limit in nanoseconds (default 2e9).  A pipeline
 * wait or a wait for another CTA's data that exceeds it records
 * MK_ERR_TIMEOUT and the kernel returns early.  `fail_phase` >= 0 makes the
 * next decode launch wait, in that phase (0-based index of the launch's
 * phase sequence: five phases per layer, then the LM head), for data
 * tagged with a value no phase ever writes (or a split-K sum with one
 * contribution more than any phase adds), so the wait must run out (tests
 * of the timeout path only). */
int mk_debug_set_wait_limit(mk_engine *e, int64_t limit_ns, int fail_phase);

/* ------------------------------------------------------------------------
 * Isolated gated delta-rule step (no engine).  One launch advances B
 * sequences x heads of the recurrence by one token, in place:
 *   S <- alpha S (I - beta k k^T) + beta v k^T ,   o = S q
 * (Gated Delta Networks, the gated delta rule).
 *   S     device float32 [B][heads][dv][dk]   state, read and written
 *   q, k  device bf16    [B][heads][dk]       used as given (no renorm)
 *   v     device bf16    [B][heads][dv]
 *   alpha, beta device float32 [B][heads]
 *   o     device float32 [B][heads][dv]
 * dk == dv in {64, 128}.  `stream` is a cudaStream_t (may be NULL). */
int mk_delta_step(float *S, const void *q, const void *k, const void *v,
                  const float *alpha, const float *beta, float *o, int B,
                  int heads, int dk, int dv, void *stream);

/* The gated delta rule over a whole sequence of T positions in the
 * chunkwise-parallel form the prompt path uses ("Gated Delta Networks",
 * the WY / UT representation of a chunk of delta-rule updates: chunks of 64
 * positions prepared independently, then one pass over the chunks per slice
 * of state rows), no engine.  Results equal T consecutive steps of
 * mk_delta_step up to rounding.
 *   S      device float32 [heads][dv][dk], read and written
 *   q, k   device float32 [heads][T][dk], used as given (no renormalisation)
 *   v      device float32 [heads][T][dv]
 *   alpha, beta device float32 [heads][T]
 *   o      device float32 [heads][T][dv]   (o_t = S_t q_t)
 *   workspace device scratch, 16-byte aligned, at least
 *          mk_delta_chunked_ws_bytes(T, heads, dk) bytes (caller-owned)
 * dk == dv in {64, 128} (else MK_ERR_UNSUPPORTED); MK_ERR_ARG on NULL,
 * misaligned or short arguments.  Asynchronous on `stream`. */
size_t mk_delta_chunked_ws_bytes(int T, int heads, int dk);
int mk_delta_chunked(float *S, const float *q, const float *k, const float *v,
                     const float *alpha, const float *beta, float *o, int T,
                     int heads, int dk, int dv, void *workspace, size_t ws_bytes,
                     void *stream);

/* Debug: the prompt path's tensor-core GEMM on its own, asynchronous on
 * `stream` (a cudaStream_t, may be NULL):
 *   C[t][n] = sum_k (X_hi[t][k] + X_lo[t][k]) * W[n][k]
 *   W device bf16 [n_out][K]; X device bf16 [2][T][K], the hi operands of
 *   the activations then their lo residuals (an fp32 x is split as
 *   hi = bf16(x), lo = bf16(x - hi)); C device float32 [T][n_out]; all
 *   16-byte aligned, K a multiple of 64.
 * MK_ERR_ARG on bad sizes, MK_ERR_UNSUPPORTED if the TMA descriptors cannot
 * be encoded.  The first call on a device allocates a 4-byte device word
 * (kept for the life of the process) where a device-side wait that runs
 * out is recorded.  Every call clears that word first (stream-ordered), and
 * if a tile's wait runs out, all of C is set to NaN: the call returns
 * before the GPU runs it, so a timed-out call shows in its output, never as
 * silently wrong values. */
int mk_debug_gemm(const void *W, const void *X, float *C, int n_out, int T,
                  int K, void *stream);

/* The same GEMM as mk_debug_gemm, for callers that must not allocate device
 * memory (the pages have no counterpart): a process whose device memory is
 * fully budgeted up front, or a host loop that may not call cudaMalloc or an
 * allocating library between steps.  It allocates nothing: K is split over
 * the SMs and the ranges' partial sums go to a static device scratch array
 * of 2^21 floats (8 MiB) inside libmk.so, then are summed in a fixed order
 * into C.  T * n_out must not exceed 2^21 (else MK_ERR_ARG); other argument
 * rules and layouts as mk_debug_gemm.  The first call on a device (made
 * with that device current) looks up the scratch address with
 * cudaGetSymbolAddress; make that first call before any stream capture.
 * No partial needs to start at zero: every partial is written before it is
 * read.  The private wait-error word (also static) is cleared by every call
 * with cudaMemsetAsync before its kernels; if a range's wait runs out it is
 * set, and the reduction writes NaN to all of C instead of the sums.  Calls
 * share the scratch, so calls that overlap (other streams or threads
 * without ordering) race; serialise them. */
int mk_debug_gemm_noalloc(const void *W, const void *X, float *C, int n_out,
                          int T, int K, void *stream);

/* ---- 4-bit weights ------------------------------------------------------
 * The tag page "RTX 3090" (item on a custom engine for a 27B-class model
 * on one RTX 3090: 4-bit weights with 16-bit activations, "W4A16") credits
 * 4-bit weights for its speed, since a batch-1 decoder streams every weight
 * once per token.  Format (the page names none; this is the plain
 * group-wise symmetric reading): groups of 64 consecutive weights of a row
 * share one fp32 scale s = max|w| / 7 (0 for an all-zero group); each weight
 * is stored as the nibble q + 8 with q = clamp(rint(w / s), -7, 7) (IEEE
 * fp32 division, round half to even); weight k of a row lives in byte k / 2
 * of the row, the even weight in the low nibble.  A row of `cols` weights
 * takes cols / 2 bytes of codes and cols / 16 bytes of scales. */

/* Quantise W (device, bf16 [rows][cols], 16-byte aligned) into codes
 * (device, uint8 [rows][cols / 2], 16-byte aligned) and scales (device,
 * float32 [rows][cols / 64], 16-byte aligned).  cols must be a multiple of
 * 64 (else MK_ERR_ARG).  Asynchronous on `stream` (a cudaStream_t or NULL);
 * nothing is allocated. */
int mk_quantize_w4(const void *W, int rows, int cols, void *codes, float *scales,
                   void *stream);

/* y[t][n] = sum_k s(n, k / 64) * q(n, k) * x[t][k] for t < T, with fp32
 * activations and fp32 accumulation: every code row is read once for all T
 * rows of x.  codes / scales as mk_quantize_w4 writes them; x (device,
 * float32 [T][cols], 16-byte aligned); y (device, float32 [T][rows]).
 * 1 <= T <= 8 and cols a multiple of 64 (else MK_ERR_ARG); T * cols * 4
 * bytes must fit in 220 KB of shared memory (else MK_ERR_UNSUPPORTED).
 * Asynchronous on `stream`; allocates nothing.  The first call per device
 * and T (and any call that needs more shared memory than the earlier ones)
 * raises the kernel's shared-memory limit: serialise those calls when
 * several host threads use the library. */
int mk_gemv_w4(const void *codes, const float *scales, const float *x, int T,
               int rows, int cols, float *y, void *stream);

/* Human-readable text of a status code. */
const char *mk_strerror(int status);

#ifdef __cplusplus
}
#endif
#endif /* MK_H */
