/*
 * ttt.h — C ABI of libttt.so, the fast-weight (test-time-training) chunk scan on one
 * NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources are the pages' titles and sections):
 *
 *  In-Place rule ("In-Place Test-Time Training", §2, §3, §4, §6). The fast weight is the
 *  gated MLP's down projection Wdown [d_model x d_ff]. The sequence is cut into chunks of
 *  C tokens. For chunk c, first O_c = Z_c · W_cᵀ with the weight from before this chunk
 *  (chunk 0 uses the pretrained W0), then W_{c+1} = W_c + η · V̂_cᵀ · Z_c. The target is
 *  either given (V̂) or produced as V̂ = Conv1D(X0) · Wtarget with depthwise taps at token
 *  offsets 0, +1, +2 that read zero past the end of the token's chunk.
 *
 *  TTT-Linear rule ("テスト時学習（Test-Time Training）とは", the TTT layers page: the
 *  hidden state is a linear model updated by one self-supervised gradient step). Per
 *  (sequence, head), for each inner mini-batch i of b tokens: O_i = Q_i · W_i,
 *  R_i = K_i · W_i − V_i, L_t = ‖R_i[t]‖², W_{i+1} = W_i − (η/b) · K_iᵀ · R_i.
 *
 *  Richer inner models (the TTT layers page: TTT-Linear and TTT-MLP are its two instances,
 *  and by its DeltaNet remark the full TTT-Linear carries a LayerNorm and a residual
 *  connection). The inner model is f(x) = x + LN(g(x)) with g(x) = x · W (rule
 *  TTT_RULE_LINEAR_LN_GD) or g(x) = GELU(x · W1) · W2 (TTT_RULE_MLP_GD, hidden width 256,
 *  GELU(x) = x·Φ(x)); LN normalises a token's 64 values by their mean and population variance
 *  (ε under the square root) and applies the per-head gain γ and bias β, which the inner step
 *  does not change. Per mini-batch of 16 tokens: O_i = f(Q_i; θ_i), E_i = f(K_i; θ_i) − V_i,
 *  L_t = ‖E_i[t]‖², θ_{i+1} = θ_i − η · ∇ℓ_i(θ_i) with ℓ_i = ‖E_i‖² / (2·16). With per-token
 *  weights (token_weights = 1, the TTT layer's mini-batch form) output t instead uses the
 *  weights after the gradient steps of the mini-batch's tokens up to t, all taken at θ_i.
 *
 *  Surprisal gate ("SR-TTT: Surprisal-Aware Residual Test-Time Training", §2.1). Per
 *  (sequence, head) and chunk of 64 losses: p95 = 61st smallest; τ = p95 for the first
 *  chunk, else τ = fl32(fl32(0.9·τ) + fl32(0.1·p95)); the chunk passes if
 *  5·S ≥ 256·τ with S the double sum of its losses in index order; a token of a passing
 *  chunk is routed if L_t > τ. Routed (sequence, head, t) triples are appended in
 *  increasing t to that (sequence, head)'s cache until it is full; later ones are counted
 *  as dropped.
 *
 * Conventions shared by every entry point:
 *  - Every pointer argument marked "device" must point to memory of the CUDA device that
 *    was current when the state was created, be 16-byte aligned and be densely packed in
 *    the row-major layout stated for it. The caller owns all such buffers; the library
 *    never frees or retains them beyond the call.
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default
 *    stream). Calls that synchronise: ttt_state_poll(), ttt_chunk_scan_host(),
 *    ttt_chunk_scan_docs() (it uploads the document layout from host memory) and
 *    ttt_state_destroy() always; ttt_state_create(), the first ttt_chunk_scan() of an
 *    In-Place BF16 state (it builds and uploads its tile schedules) and a scan that must
 *    grow a state-owned scratch buffer (longer T than before, or the first host call) may,
 *    through cudaMalloc, cudaFree and cudaMemcpy. Steady-state scans of unchanged sizes
 *    enqueue only.
 *  - Everything a call reads and advances from one call to the next (the weights, the index
 *    of the In-Place bf16 weight copy in use, the gate's threshold, cache and token position)
 *    lives in device memory, and the fp32 In-Place weight ends every call in the same buffer.
 *    So a steady-state scan (ttt_chunk_scan, ttt_surprisal_route, ttt_cache_attention,
 *    ttt_state_reset) can be captured into a CUDA graph once and replayed any number of
 *    times, each replay continuing the state where the last left it, with the caller copying
 *    each segment's inputs into the captured buffers before the replay.
 *  - A call returns TTT_OK or an error status and never aborts the process. The message
 *    of the last error on the calling thread is returned by ttt_last_error_string().
 *  - Every call that takes a state must be made with the state's device current
 *    (else INVALID_ARG). Calls on one state must not run concurrently from several host
 *    threads; different states are independent.
 *  - Failures detected on the device (a bounded wait that ran out, a failed device-side
 *    check, an argument check against a count that only the device holds) are recorded in
 *    the state's status word and returned by the next call of ttt_state_poll().
 */
#ifndef TTT_H_
#define TTT_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so this header needs no CUDA include. */
typedef struct CUstream_st* ttt_stream;

typedef enum {
  TTT_OK = 0,
  TTT_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, T not a multiple of the chunk */
  TTT_ERR_UNSUPPORTED = 2, /* a valid configuration this library does not implement */
  TTT_ERR_OOM = 3,         /* device or pinned host allocation failed */
  TTT_ERR_CUDA = 4,        /* a CUDA runtime or driver call failed */
  TTT_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out (from ttt_state_poll) */
  TTT_ERR_DEVICE = 6       /* a device-side consistency check failed (from ttt_state_poll) */
} ttt_status;

typedef enum {
  TTT_RULE_INPLACE_HEBBIAN = 0,
  TTT_RULE_LINEAR_GD = 1,     /* TTT-Linear: linear inner model, no normalisation */
  TTT_RULE_LINEAR_LN_GD = 2,  /* TTT-Linear with LayerNorm and residual */
  TTT_RULE_MLP_GD = 3         /* TTT-MLP: two-layer GELU MLP (hidden 256) with LayerNorm and residual */
} ttt_rule;
typedef enum { TTT_F32 = 0, TTT_BF16 = 1 } ttt_dtype;

typedef struct {
  int32_t rule;           /* ttt_rule */
  int32_t io_dtype;       /* ttt_dtype of keys, targets, queries and out. The weight state is
                             always fp32. In-Place: F32 (SIMT FFMA) or BF16 (tensor cores).
                             TTT-Linear: BF16. */
  int32_t batch, heads;   /* TTT-Linear: sequences and heads per sequence. In-Place: 1 and 1. */
  int32_t d_key;          /* In-Place: d_ff = f, columns of Wdown. TTT-Linear: head width (64). */
  int32_t d_val;          /* In-Place: d_model = d, rows of Wdown. TTT-Linear: head width (64). */
  int32_t chunk;          /* In-Place: chunk C. TTT-Linear: inner mini-batch b (16, 32 or 64;
                             other values are UNSUPPORTED at ttt_state_create). */
  float eta;              /* learning rate η */
  int32_t target_mode;    /* In-Place only. 0: targets are V̂ [T, d]. 1: targets are X0 [T, d]
                             and V̂ = Conv1D(X0)·Wtarget is produced inside the scan (BF16). */
  int32_t conv_pad_mode;  /* 0: taps read zero past the token's chunk end (default).
                             1: taps read zero past the end of the call's tokens only. */
  int32_t conv_taps;      /* number of future taps (offsets 0 .. conv_taps-1); 3 */
  int32_t gate_enable;    /* TTT-Linear only: run the surprisal gate on the scan's losses */
  int32_t gate_chunk;     /* tokens per gate chunk; 64 */
  int32_t cache_capacity; /* residual cache entries per (sequence, head); 256 */
  float gate_pct;         /* percentile of the threshold (nearest rank); 0.95 */
  float gate_ema_old;     /* weight on the previous τ; 0.9f */
  float gate_ema_new;     /* weight on the chunk's percentile; 0.1f */
  int32_t gate_mean_num;  /* the mean test is S/gate_chunk >= (num/den)·τ; 4 */
  int32_t gate_mean_den;  /* 5 */
  float ln_eps;           /* TTT_RULE_LINEAR_LN_GD and TTT_RULE_MLP_GD: LayerNorm ε; 1e-6 */
  int32_t token_weights;  /* TTT-Linear family: 0 (default): the outputs of a
                             mini-batch use its starting weights θ_i. 1: per-token weights, output t
                             uses θ_i − (η/b)·Σ_{s ≤ t} ∇½‖f(k_s; θ_i) − v_s‖² over the mini-batch's
                             tokens s up to t (the last token sees θ_{i+1}); losses and the weight
                             update are unchanged. Also TTT_RULE_LINEAR_GD with mini-batch 16 and no
                             gate (the dual form of the plain rule). In-Place: must be 0. */
} ttt_config;

typedef struct ttt_state ttt_state; /* opaque; owns all of its device memory */

/* ABI version of this header (incremented on any incompatible change). */
int32_t ttt_abi_version(void);

/* Fill *cfg with the defaults of `rule` (the values noted above, eta = 1, chunk 16 for the
 * TTT-Linear and TTT-MLP rules, 1024 for In-Place, BF16). INVALID_ARG if cfg is NULL or rule
 * unknown. The rules with LayerNorm and the MLP take only batch, heads, eta and ln_eps: head
 * width 64, mini-batch 16, BF16 io, no gate (else UNSUPPORTED at ttt_state_create). */
ttt_status ttt_config_init(ttt_config* cfg, int32_t rule);

/* Create a scan state on the current device and copy the initial weights into it.
 *   W0       device. In-Place: fp32 [d_val, d_key] (Wdown, row-major).
 *                    TTT-Linear (with or without LayerNorm): fp32 [batch, heads, d_key, d_key],
 *                    applied as x·W.
 *                    TTT-MLP: fp32 [batch, heads, 64·256 + 256·64]: per (sequence, head) W1
 *                    [64, 256] then W2 [256, 64], row-major, applied as GELU(x·W1)·W2.
 *            The LayerNorm rules start with γ = 1 and β = 0 (ttt_state_set_layernorm).
 *   Wtarget  device, In-Place with target_mode 1 only (else NULL): bf16 [d_val, d_val],
 *            [in, out], V̂[t, j] = Σ_i conv[t, i]·Wtarget[i, j].
 *   convw    device, target_mode 1 only (else NULL): fp32 [d_val, conv_taps].
 * W0, Wtarget and convw are copied; the caller may free them after the call returns
 * (stream-ordered). On success *out receives the state; on error *out is NULL and
 * nothing is leaked. Errors: INVALID_ARG (bad sizes or pointers), UNSUPPORTED (shape or
 * mode not implemented, see the message), OOM, CUDA. The state starts at the pretrained
 * weight ("In-Place Test-Time Training", §2: the MLP's own Wdown is the fast weight; the TTT
 * layers page: the inner model's weight is the hidden state). */
ttt_status ttt_state_create(const ttt_config* cfg, const void* W0, const void* Wtarget,
                            const float* convw, ttt_stream stream, ttt_state** out);

/* Continue the scan over the next T tokens (successive calls form one scan).
 *   In-Place:   keys = Z [T, d_key]; targets = V̂ [T, d_val] (target_mode 0) or X0 [T, d_val]
 *               (target_mode 1); queries must be NULL; out = O [T, d_val] (required);
 *               loss_out must be NULL. T must be a multiple of chunk.
 *   TTT-Linear, TTT-MLP: keys = K, targets = V, queries = Q (or NULL), all
 *               [batch, heads, T, d_key];
 *               out = O [batch, heads, T, d_key] (NULL iff queries is NULL);
 *               loss_out = L [batch, heads, T] fp32 (or NULL; required when the gate is
 *               enabled). T must be a multiple of chunk (and of gate_chunk with the gate).
 * All inputs are read-only; outputs are written with the io dtype (loss fp32). Inputs and
 * outputs must not overlap. T = 0 is a no-op. Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 * Defined by "In-Place Test-Time Training", §3 (each chunk is applied with the weight from
 * before it, then the weight is updated from that chunk) and §4 (the next-token-aligned
 * target Conv1D(X0)·Wtarget, with padding at chunk boundaries from §6), and by the TTT
 * layers page (one self-supervised gradient step of the inner linear model per mini-batch;
 * with b = 1 and no normalisation it is the delta rule). */
ttt_status ttt_chunk_scan(ttt_state* st, const void* keys, const void* targets,
                          const void* queries, int64_t T, void* out, float* loss_out,
                          ttt_stream stream);

/* ttt_chunk_scan with HOST buffers of the same shapes, returning when the outputs are in
 * host memory. T is cut into segments of about T/4 tokens (whole chunks; whole gate chunks
 * with the gate; one segment for the fused target in conv_pad_mode 1, whose taps reach past
 * the call's end, and for the TTT-Linear family when the outputs are less than a fifth of the
 * inputs), each scanned as a separate ttt_chunk_scan call would be, so the results are those
 * of one call. A segment's inputs are copied to one of two sets of device staging
 * buffers owned by the state (grown on demand) on a copy stream of the state's, its scan runs
 * on `stream`, its outputs come back on a second copy stream: the copies of neighbouring
 * segments overlap each scan, in both directions at once. All three streams are synchronised
 * before the call returns, on errors too. Host buffers should be pinned: copies from or to
 * pageable memory do not overlap. */
ttt_status ttt_chunk_scan_host(ttt_state* st, const void* keys, const void* targets,
                               const void* queries, int64_t T, void* out, float* loss_out,
                               ttt_stream stream);

/* Packed sequences for In-Place BF16 states: `keys` Z (device, bf16 [T, d_key]) and `targets`
 * (device, bf16 [T, d_val]: V̂ with target_mode 0, X0 with target_mode 1) hold documents laid end
 * to end; `doc_starts` (HOST, int64 [ndocs]) lists each document's first token: 0 first,
 * strictly increasing, below T. Each document is scanned as if alone: the weight starts from
 * the pretrained W0, its chunks are counted from its first token (its last chunk may be
 * shorter: T need not be a multiple of chunk), and with clip_norm > 0 each chunk's delta
 * η·V̂_cᵀ·Z_c is scaled to Frobenius norm clip_norm when its norm is larger (0: no clipping).
 * With target_mode 1 each document's targets Conv1D(X0)·Wtarget are made from its own rows:
 * the taps stop at its end (and in conv_pad_mode 0 at the end of each of its chunks, counted
 * from its first token).
 * Writes `out` (device, bf16 [T, d_val]); afterwards the state holds the last document's
 * final weight. Runs in the context-parallel form (all chunk deltas, their norms, sums that
 * restart at each document, all outputs), with state-owned scratch for the padded layout and
 * the deltas (grown on demand). Errors: INVALID_ARG (a malformed doc_starts, negative or NaN
 * clip_norm, misaligned buffers), UNSUPPORTED (other states), CUDA. Defined by "In-Place
 * Test-Time Training", §6 and the implementation notes after it (the weight goes back to its
 * pretrained value at each independent document; the Frobenius norm of the update delta is
 * clipped). */
ttt_status ttt_chunk_scan_docs(ttt_state* st, const void* keys, const void* targets, int64_t T, void* out,
                               const int64_t* doc_starts, int32_t ndocs, float clip_norm, ttt_stream stream);

/* Packed sequences for the TTT-Linear family (plain, LayerNorm and MLP rules; mini-batch 16, no
 * gate): sequence b of the batch holds docs_per_seq[b] documents laid end to end, whose first
 * tokens are the next docs_per_seq[b] entries of doc_starts (host memory, sequence after
 * sequence; each sequence's list starts at 0, increases strictly and stays below T). Each
 * document is scanned as if alone: the weights of every head start from the pretrained W0,
 * mini-batches are counted from its first token, and its last mini-batch may be shorter: with
 * b' < 16 tokens it takes the step of its own loss (η/b' for the plain rule). T need not be a
 * multiple of 16. keys, targets, queries (or NULL), out (NULL iff queries is NULL) and loss_out
 * (or NULL) are laid out as for ttt_chunk_scan, [batch, heads, T, ...]; afterwards the state holds
 * each sequence's last document's final weights. Per-token weights (token_weights = 1) apply
 * within every mini-batch. Runs one scan launch over a padded copy (state-owned scratch grown
 * on demand, with gather and scatter launches around it) and synchronises (the layout goes up
 * from host memory). Errors: INVALID_ARG (malformed document lists, misaligned buffers),
 * UNSUPPORTED (In-Place states, other mini-batches, the gate), CUDA. Defined by "In-Place
 * Test-Time Training", §6 and the notes after it (the weights go back to their pretrained value
 * at each independent document) and the TTT layers page (the hidden state is the inner model's
 * weight, so a new sequence starts it afresh). */
ttt_status ttt_chunk_scan_packed(ttt_state* st, const void* keys, const void* targets, const void* queries, int64_t T,
                                 void* out, float* loss_out, const int64_t* doc_starts, const int32_t* docs_per_seq,
                                 ttt_stream stream);

/* Run the surprisal gate alone on a loss array `loss` (device, fp32 [batch, heads, T]),
 * advancing the state's τ, cache and token position exactly as a gated scan would.
 * TTT-Linear states only; T must be a multiple of gate_chunk. The token position (stored
 * in the cache as int32) may not pass 2^31 − 1 between resets: a gated call that would take
 * it there (this one or ttt_chunk_scan with the gate on) returns UNSUPPORTED, or, when only
 * the device's count shows it (replays of a captured call), the next ttt_state_poll does. Defined by
 * "SR-TTT: Surprisal-Aware Residual Test-Time Training", §2.1 (the loss gate's two
 * conditions and the residual cache). */
ttt_status ttt_surprisal_route(ttt_state* st, const float* loss, int64_t T, ttt_stream stream);

/* Document boundary: W ← W0, τ unset, cache emptied (entries -1, counts 0), token
 * position 0. Defined by "In-Place Test-Time Training", §6 (implementation notes: when an
 * independent document ends, the fast weight goes back to its pretrained value so that no
 * information leaks from one document into the next; §8 repeats that the fast weight lives
 * only within a document). The gate's threshold and cache are per-document state of the
 * same scan ("SR-TTT", §2.1), so they restart with it. */
ttt_status ttt_state_reset(ttt_state* st, ttt_stream stream);

/* Copy the current fp32 weights out of / into the state (device buffers shaped like W0).
 * set_weights also refreshes the In-Place bf16 copy used by the apply. The weight is the
 * scan's whole recurrent state (the TTT layers page: the hidden state is the inner model's
 * weight; "In-Place Test-Time Training", §2: Wdown is that weight), so saving it and setting
 * it back resumes a scan exactly at a chunk boundary. */
ttt_status ttt_state_get_weights(const ttt_state* st, float* W, ttt_stream stream);
ttt_status ttt_state_set_weights(ttt_state* st, const float* W, ttt_stream stream);

/* y ← y + alpha·x over n fp32 elements (device buffers of the current device; y and x may
 * not overlap unless equal), enqueued on `stream`. The context-parallel form across devices
 * combines weights with it: the In-Place update η·V̂ᵀ·Z does not depend on W, so the weight a
 * device's first chunk starts from is the weight before the sequence plus the sums of the
 * deltas of the devices before it ("In-Place Test-Time Training", §6, context parallelism: an
 * exclusive prefix sum of the chunk deltas). Errors: INVALID_ARG (NULL with n > 0, n < 0),
 * CUDA. */
ttt_status ttt_add_f32(float* y, const float* x, float alpha, int64_t n, ttt_stream stream);

/* Set the LayerNorm gain and bias of the inner model (TTT_RULE_LINEAR_LN_GD and
 * TTT_RULE_MLP_GD states; UNSUPPORTED otherwise): gamma and beta (device) fp32 [heads, 64],
 * shared by every sequence. They are parameters of the outer model: the scan reads them and
 * never updates them (copied; the caller keeps ownership). A state starts with γ = 1, β = 0.
 * Defined by the TTT layers page (the full TTT-Linear's inner model carries a LayerNorm, which
 * DeltaNet drops). */
ttt_status ttt_state_set_layernorm(ttt_state* st, const float* gamma, const float* beta, ttt_stream stream);

/* Copy out the residual cache: entries (device) int32 [batch, heads, cache_capacity, 3]
 * holding (sequence, head, t) with t counted from the last reset, unused entries -1;
 * counts (device) int32 [batch, heads, 2] = (tokens routed, routed tokens dropped).
 * Either pointer may be NULL. The cache is the fixed-capacity store of the tokens the gate
 * finds incompressible ("SR-TTT: Surprisal-Aware Residual Test-Time Training", §2.1,
 * "Residual Cache"); this library keeps the first cache_capacity of them in token order and
 * counts the rest as dropped. */
ttt_status ttt_cache_read(const ttt_state* st, int32_t* entries, int32_t* counts,
                          ttt_stream stream);

/* Copy out the gate thresholds: tau (device) fp32 [batch, heads]; tau_set (device) int32
 * [batch, heads], 1 once a chunk has set τ. Either pointer may be NULL. τ is the
 * EMA-smoothed 95th percentile of the per-token losses ("SR-TTT", §2.1, the gate's first
 * condition). */
ttt_status ttt_gate_read(const ttt_state* st, float* tau, int32_t* tau_set, ttt_stream stream);

/* Read path of the residual cache ("SR-TTT: Surprisal-Aware Residual Test-Time Training", §2.1,
 * "Residual Cache" and "Alpha Fusion"): the layer's output is the TTT output plus the cache's
 * attention output weighted by the gate vector α, clamped to [0, 1]:
 *   out[b,h,t] = o_ttt[b,h,t] + clamp(α[h], 0, 1) ⊙ Σ_j softmax_j(q_t·k_j / √64)·v_j
 * over the cache entries j of (b, h) that token t may see: those whose 64-token gate chunk lies
 * before t's (a token's routing is known once its gate chunk has been scanned). The keys and
 * values of an entry are the scanned K and V rows of its token. A query that sees no entry adds
 * nothing (out = o_ttt).
 *   queries, keys, values, o_ttt  device bf16 [batch, heads, T, 64]: the Q, K and V of all T
 *            tokens scanned since the last reset (T must equal that count: a T below the
 *            count of the calls made on the host returns INVALID_ARG; any other mismatch is
 *            found by the kernel, which holds the count, and the next ttt_state_poll returns
 *            INVALID_ARG) and the scan's outputs.
 *   alpha    device fp32 [heads, 64].
 *   out      device bf16 [batch, heads, T, 64]; may be o_ttt itself (updated in place).
 * TTT-Linear states with the gate, cache_capacity ≤ 256. The cache is read as the gate left it
 * on the stream. Errors: INVALID_ARG (sizes, pointers, T), UNSUPPORTED, CUDA. */
ttt_status ttt_cache_attention(const ttt_state* st, const void* queries, const void* keys, const void* values,
                               const void* o_ttt, const float* alpha, int64_t T, void* out, ttt_stream stream);

/* Target generation V̂ = Conv1D(X0)·Wtarget for T tokens without allocating device memory.
 * The pages have no counterpart of this entry point: it exists for callers that cannot call
 * cudaMalloc where they need the work done — their device memory is owned by another
 * allocator that has reserved the GPU, or they run a loop that must not allocate after
 * start-up (cudaMalloc can block and synchronise the device). It computes the same values
 * as the fused target of an In-Place state with target_mode 1 (same kernels), but keeps its
 * scratch (the conv rows and the tile schedule) in one fixed array of device memory inside
 * the library image (about 8.1 MB) instead of state memory, and calls no cudaMalloc, cudaFree
 * or allocating routine.
 *   X0       device bf16 [T, d_model], the token embeddings.
 *   convw    device fp32 [d_model, conv_taps], depthwise taps at token offsets 0..taps-1.
 *   Wtarget  device bf16 [d_model, d_model], [in, out].
 *   chunk    taps read zero past the end of each chunk of this many tokens (conv_pad_mode 0)
 *            or past token T only (conv_pad_mode 1).
 *   Vhat_out device bf16 [T, d_model], written.
 *   status   device int32 or NULL. If given, the call first sets it to 0 (stream-ordered)
 *            and a bounded device-side wait that runs out sets it to TTT_ERR_TIMEOUT (then
 *            Vhat_out is incomplete); read it after the stream's work has finished.
 * Limits: T a multiple of 128, d_model a multiple of 8, T·d_model ≤ 4,194,304; larger inputs
 * are rejected with TTT_ERR_INVALID_ARG and a message naming the limit. The fixed array is
 * created on a device when the library's module is first loaded there: with lazy module
 * loading (the CUDA default) that is this entry point's first call on the device, with
 * CUDA_MODULE_LOADING=EAGER it is library load; from then on the device holds it until the
 * process exits. The first call on each device therefore may need about 8 MB of free device
 * memory and may synchronise: it looks up the array's device address (cudaGetSymbolAddress
 * with that device current). Make that first call before any stream capture. All calls share
 * the array and it keeps the last call's contents: calls whose GPU work overlaps (other
 * streams, other host threads) race on it. */
ttt_status ttt_target_values_noalloc(const void* X0, const float* convw, const void* Wtarget, int64_t T,
                                     int32_t d_model, int32_t chunk, int32_t conv_taps, int32_t conv_pad_mode,
                                     void* Vhat_out, int32_t* status, ttt_stream stream);

/* Options of a state, set after creation (ttt_state_set_option). */
typedef enum {
  /* TTT-Linear with b = 16: how many inner mini-batches the scan groups into one chunk.
   * 1 runs the mini-batch steps one after another. 2 or 4 run the chunked form: inside a
   * chunk every product with W uses the weight from the chunk's start, and each mini-batch's
   * residual is corrected by those of the mini-batches before it through the Gram blocks
   * K_i·K_jᵀ (and Q_i·K_jᵀ for the outputs). That is the same sequence of weights and outputs
   * as the step-by-step rule, regrouped (rounding differs); results are bit-identical between
   * a single call and calls split at multiples of 16·value tokens. 0 selects the default (1,
   * the fastest on B200: the chunked forms issue more tensor-core work per token and the
   * step chain is not what bounds this kernel). Other rules and mini-batch sizes ignore it. */
  TTT_OPT_LINEAR_CHUNK = 1,
  /* Limit of every spin-wait of this state's kernels, in nanoseconds of the GPU's global
   * timer: a wait that lasts longer records TTT_ERR_TIMEOUT (read by ttt_state_poll), the
   * kernel drains its own copies and tensor-core work in flight (each with the same limit),
   * releases its tensor memory and returns. Range [1000, 60e9]; default 2e9 (2 s). */
  TTT_OPT_WAIT_LIMIT_NS = 2,
  /* Fault injection for tests of the path above, value 1: the next scan that can (an In-Place
   * BF16 scan of two or more chunks, or a TTT-Linear b = 16 scan longer than 64 tokens) makes
   * one of its bounded waits wait for something that never comes — an In-Place APPLY tile of
   * the second chunk waits for one more finished UPDATE tile than exists; the TTT-Linear scan
   * never loads its second 64-token tile — so that the wait runs out. The outputs of that scan
   * are incomplete. 0 cancels a pending injection. */
  TTT_OPT_INJECT_STALL = 3,
  /* In-Place BF16 states with given targets (target_mode 0), value 1: run each scan call in the
   * context-parallel form ("In-Place Test-Time Training", §6: the chunk updates are additive, so
   * every chunk's ΔW_j is computed in parallel, an exclusive prefix sum gives each chunk its
   * cumulative update, and every chunk's outputs are computed in parallel with
   * W_c = W_start + η·Σ_{j<c} ΔW_j). Same outputs and final weight as the sequential form, up
   * to rounding (each η·ΔW_j is rounded to fp32 before it is added). The call keeps n fp32
   * deltas and n bf16 weights of d_val x d_key in state-owned scratch (grown on demand, n =
   * T / chunk). 0 returns to the sequential form. UNSUPPORTED for other states. */
  TTT_OPT_INPLACE_PREFIX = 4,
  /* In-Place BF16 states, sequential form: 1 (default) runs the tensor-core scan on pairs of
   * SMs (clusters of two CTAs, tcgen05 MMAs of 256 x 256 tiles issued for both) wherever the
   * chunk and d_val are multiples of 256, and on single SMs (128 x 256 tiles) otherwise; 0
   * always uses single SMs. Both give the same results up to the order of fp32 additions
   * inside the tensor cores. Changing it rebuilds the state's tile schedules on the next scan
   * (the call synchronises the device). Other states ignore it. */
  TTT_OPT_SM_PAIR = 5,
  /* Tests of the device-side check of the gate's token position: sets the count of tokens
   * gated since the reset, held on the device per (sequence, head), to `value` for every
   * (sequence, head), leaving the host's own count alone, as replays of a captured call do.
   * Range [0, 2^31 − 1]; synchronises the device. TTT-Linear states only (UNSUPPORTED
   * otherwise). */
  TTT_OPT_GATE_TOKENS = 6
} ttt_option;

/* Set option `option` of state `st` to `value`. Takes effect from the next call that
 * enqueues work. Errors: INVALID_ARG (unknown option or value out of range). */
ttt_status ttt_state_set_option(ttt_state* st, int32_t option, int64_t value);

/* Synchronise the device and return the first device-side failure recorded since the
 * last poll, or TTT_OK; clears the record. TTT_ERR_TIMEOUT: a bounded wait ran out, and
 * ttt_last_error_string() names it: an mbarrier (by its shared-memory offset in the
 * kernel's layout) or a progress counter (by the low bits of its address). INVALID_ARG: the
 * T given to ttt_cache_attention was not the count of tokens gated since the reset.
 * UNSUPPORTED: the gate's token position passed 2^31 − 1. TTT_ERR_DEVICE: another
 * device-side check failed. The message names the (sequence, head) of the last two. */
ttt_status ttt_state_poll(ttt_state* st);

/* Number of kernels this state has launched since creation. */
int64_t ttt_state_launch_count(const ttt_state* st);

/* Synchronise the device and free everything the state owns. NULL is a no-op. */
ttt_status ttt_state_destroy(ttt_state* st);

/* Message of the last error returned on the calling thread ("" if none). */
const char* ttt_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* TTT_H_ */
