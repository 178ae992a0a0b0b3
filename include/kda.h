/*
 * kda.h - C ABI of libkda.so: the Kimi Delta Attention (KDA) layer hot path on
 * NVIDIA B200 (sm_100a).
 *
 * The layer (llama.cpp PR #27754 "model: add GLM-5-Next", KDA commit) is, per
 * head h of width d (d_k = d_v = d), for each token t of a sequence:
 *
 *   prep   x~ = depthwise causal conv over q|k|v (one kernel, K taps), then SiLU
 *          q = q~ / max(||q~||, l2_eps),  k = k~ / max(||k~||, l2_eps),  v = v~
 *          log a_t = lb * sigmoid(exp(A_log[h]) * (f_t + dt_bias[h]))   (per key channel;
 *                    or -exp(A_log[h]) * softplus(f_t + dt_bias[h]), enum kda_gate)
 *          b_t = sigmoid(beta_logit_t)
 *   state  S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T   (S is d_k x d_v,
 *          decay on the key axis; order: decay, delta update, read)
 *   out    o_t = q_scale * S_t^T q_t
 *          y_t = o_t / sqrt(mean(o_t^2) + norm_eps) * w * sigmoid(g_t)
 *
 * plus speculative verify (a block of draft tokens run from one state, with a
 * per-step state tape) and rollback to any accepted prefix (dflash-mlx issue
 * #63, "What the backend needs": rollback for the KDA recurrent state; PR
 * #27754: the conv state is one contiguous block so it can be snapshotted).
 *
 * Conventions for every entry point
 *  - Returns KDA_OK (0) or a kda_status code.  Every argument is checked on the
 *    host BEFORE anything is launched; on an error nothing is launched and no
 *    output is touched.
 *  - Every pointer is caller-owned DEVICE memory (any allocator), except `cfg`
 *    which is host memory.  The library allocates nothing and frees nothing;
 *    between calls it keeps only the per-thread measurement hooks below
 *    (phase events, launch count, last CUDA error message) and the fixed
 *    scratch of kda_prefill_noalloc.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and the call returns without synchronising.  Launch failures are
 *    reported as KDA_ERR_CUDA.
 *  - Tensors are dense, row-major (last index fastest), with the shapes given
 *    below.  Activations (x, f, beta_logit, g, y, conv state/window) have the
 *    element type cfg->dtype; the prep outputs q, k, v, log decay and beta,
 *    the parameters, the recurrent states and the tapes are fp32 (rounding the
 *    normalised q/k/v to bf16 would cost more accuracy than every later bf16
 *    operand of the chunked prefill together).
 *  - Every pointer must be 16-byte aligned (KDA_ERR_MISALIGNED otherwise).
 *  - Packed (varlen) batches use cu_seqlens: int32 [n_seqs + 1], device,
 *    non-decreasing, cu_seqlens[0] = 0, cu_seqlens[n_seqs] = total_tokens.
 *    Sequence s owns token rows [cu_seqlens[s], cu_seqlens[s+1]).  The kernels
 *    clamp every index they derive from it to [0, total_tokens], so a
 *    malformed array cannot make them access memory out of bounds (its results
 *    are then undefined).
 *  - state_slots (optional, int32 [n_seqs], device) maps sequence s to row
 *    state_slots[s] of a state pool of pool_size rows; NULL means row s.
 *    Sequences whose slot lies outside [0, pool_size) are skipped.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

typedef struct CUstream_st* kda_stream_t; /* == cudaStream_t */

enum kda_status {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad enum */
  KDA_ERR_MISALIGNED = 2,   /* a pointer is not 16-byte aligned */
  KDA_ERR_UNSUPPORTED = 3,  /* valid but not built: e.g. head_dim not in {16,32,64,128} */
  KDA_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
  KDA_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up (see kda_workspace_status) */
  KDA_ERR_WORKSPACE = 6,    /* workspace missing or smaller than kda_prefill_workspace_size */
  KDA_ERR_SCRATCH_LIMIT = 7 /* problem needs more scratch than kda_prefill_noalloc has */
};

enum kda_dtype { KDA_F32 = 0, KDA_BF16 = 1 };

enum kda_conv_mode {
  KDA_CONV_COMMIT = 0, /* conv_state <- last K-1 pre-conv rows of [conv_state; x] */
  KDA_CONV_TAPE = 1    /* conv_state read only; conv_window <- [conv_state; x] */
};

/*
 * Decay gate (per key channel, A = exp(A_log[h])).  PR #27754, "Metadata and tensor
 * loading" commit: the bounded-sigmoid branch is selected by the gate_lower_bound key
 * and, when the key is absent, a softplus branch (a separate function):
 *   KDA_GATE_BOUNDED_SIGMOID  log a = lb * sigmoid(A (f + dt_bias)),  lb in [-5, 0)
 *   KDA_GATE_SOFTPLUS         log a = -A * softplus(f + dt_bias)      (lb ignored)
 * The softplus gate has no lower bound, so a chunk's cumulative decay can span far
 * more than fp32's exponent range; the tensor-core prefill passes rely on the bound
 * (their exponent split keeps every factor within e^80) and a softplus layer runs on
 * the SIMT prefill passes, whose gram takes one exponential per (pair, channel)
 * inside each 16-token block instead of splitting it.
 */
enum kda_gate { KDA_GATE_BOUNDED_SIGMOID = 0, KDA_GATE_SOFTPLUS = 1 };

/*
 * Launch flags (kda_config.launch_flags).  The token-step kernels (kda_decode,
 * kda_verify, kda_verify_compact, the kda_layer_* step calls) and
 * kda_rollback_replay are launched as programmatic dependents of the kernel before
 * them on the stream: they may be scheduled while that kernel finishes, and wait for
 * it (its completion and its memory) before they read any input.  With
 * KDA_LAUNCH_EARLY_STATE they instead start streaming the recurrent state (the rows
 * named by state_slots) BEFORE that wait, overlapping the state read with the tail of
 * the previous kernel.  Set it only when the kernel issued just before the call on
 * the same stream writes neither `state` nor `state_slots` (kda_prep, kda_verify_compact
 * before kda_rollback_replay, the projection GEMM); everything else the call reads is
 * read after the wait.  Any other bit is KDA_ERR_INVALID_ARG.  Flags are ignored by
 * entry points that do not take a recurrent state from a previous call.
 *
 * The tensor-core prefill (bf16, d = 128, chunk 64, bounded gate) runs as ONE
 * cooperative launch when the head count lies between a fifth and a quarter of the SMs
 * (32 heads on a B200) and the sequences average at least 4 chunks: H CTAs carry the
 * inter-chunk chains, one per head over every sequence of the batch, while the others
 * run the intra-chunk pass, and each chain waits (bounded) for its chunk's tiles through
 * ready words in the workspace.  KDA_LAUNCH_SEPARATE_PASSES runs the two passes as
 * separate launches instead (the form used otherwise); the results agree bit for bit.
 */
enum kda_launch_flag { KDA_LAUNCH_EARLY_STATE = 1, KDA_LAUNCH_SEPARATE_PASSES = 2 };

/* Layer configuration (host memory, read during the call only). */
typedef struct kda_config {
  int32_t num_heads;      /* H >= 1 */
  int32_t head_dim;       /* d = d_k = d_v in {16, 32, 64, 128} */
  int32_t conv_size;      /* K taps of the short conv, 1..8 (4 in GLM-5.3-Flash) */
  int32_t dtype;          /* enum kda_dtype of the activations */
  int32_t chunk_size;     /* prefill chunk length in {16, 32, 64} */
  float gate_lower_bound; /* lb of the bounded-sigmoid decay, in [-5, 0) (GLM-5.3-Flash:
                             -5); ignored by the softplus gate */
  float l2_eps;           /* q/k L2 eps, 1e-6 (a constant in PR #27754) */
  float norm_eps;         /* output RMSNorm eps, 1e-5 (rms_norm_eps, glm53-flash-mlx README) */
  float q_scale;          /* multiplies o = S^T q; 1.0 */
  int32_t gate_kind;      /* enum kda_gate: which decay-gate function (see above) */
  int32_t launch_flags;   /* bitwise OR of enum kda_launch_flag (see above); 0 by default */
} kda_config;

/* Human-readable name of a kda_status code (static string, never NULL). */
KDA_API const char* kda_status_string(int status);

/* ABI version of this header; bumped on any incompatible change. */
KDA_API int kda_abi_version(void);

/*
 * kda_prep - fused short conv + SiLU + q/k L2 norm + decay gate + beta.
 * PR #27754, KDA commit: q|k|v convolved as ONE depthwise kernel, SiLU after
 * the conv, L2 eps exactly 1e-6 with max(sqrt(sum), eps), bounded-sigmoid
 * decay with dt_bias per channel and per-head A broadcast; f and beta come
 * from the pre-conv hidden states (separate inputs here).
 *
 *  max_seqlen  host hint: an upper bound on every sequence length, or 0 if
 *              unknown.  When 1 <= max_seqlen <= 16 (decode, verify blocks) a
 *              kernel for short sequences runs (one CTA per sequence and head,
 *              every input requested at once; still correct for longer
 *              sequences).  Otherwise the tiled kernel runs; when max_seqlen <= 64
 *              it commits the conv state itself, else a second small kernel does.
 *              There, a wrong non-zero hint leaves the conv state of longer
 *              sequences undefined (never out of bounds).
 *  x           [total_tokens, H, 3d]  pre-conv q|k|v, per head q(d) k(d) v(d)
 *  f           [total_tokens, H, d]   decay-gate input
 *  beta_logit  [total_tokens, H]
 *  conv_w      fp32 [H, 3d, K]        tap K-1 multiplies the current token
 *  A_log       fp32 [H]
 *  dt_bias     fp32 [H, d]
 *  conv_state  [pool_size, K-1, H, 3d] pre-conv history, oldest row first, or
 *              NULL (history = zeros; then nothing is written back).  Rows of
 *              sequence s are at state_slots[s] (or s).  In COMMIT mode it is
 *              updated to the last K-1 rows of [history; x_s].
 *  conv_mode   enum kda_conv_mode
 *  conv_window TAPE mode only: [total_tokens + n_seqs*(K-1), H, 3d]; sequence s
 *              occupies rows [cu[s] + s*(K-1), cu[s+1] + (s+1)*(K-1)) and gets
 *              [history; x_s].  Ignored (may be NULL) in COMMIT mode.
 *  q, k, v     out fp32 [total_tokens, H, d]  normalised q, k and SiLU'd v
 *  log_a       out fp32 [total_tokens, H, d]
 *  beta        out fp32 [total_tokens, H]
 */
KDA_API int kda_prep(const kda_config* cfg, int32_t n_seqs, int32_t total_tokens,
             const int32_t* cu_seqlens, int32_t max_seqlen, const void* x, const void* f,
             const void* beta_logit, const float* conv_w, const float* A_log,
             const float* dt_bias, void* conv_state, const int32_t* state_slots,
             int32_t pool_size, int32_t conv_mode, void* conv_window, void* q,
             void* k, void* v, float* log_a, float* beta, kda_stream_t stream);

/*
 * Workspace bytes kda_prefill needs for this problem (0 on invalid arguments).
 * The workspace holds the intra-chunk products handed from the chunk-parallel
 * pass to the serial inter-chunk pass.
 */
KDA_API size_t kda_prefill_workspace_size(const kda_config* cfg, int32_t n_seqs,
                                  int32_t total_tokens);

/*
 * kda_prefill - chunkwise-parallel prefill of packed sequences (chunk length
 * cfg->chunk_size).  llama.cpp PR #27754, KDA commit: prefill on backends without
 * the fused delta-net operator runs the layer as a chunked fallback graph; this
 * is that algorithm class, written for sm_100a.  An intra-chunk pass, parallel
 * over (sequence, head, chunk), builds the UT/WY form of each chunk with a
 * triangular solve; a
 * serial inter-chunk pass carries the fp32 state on chip through the chunks
 * of each sequence and applies the gated RMSNorm epilogue.  The result equals
 * the token-by-token recurrence up to rounding.
 *
 *  q, k, v, log_a, beta   prep outputs (layouts as in kda_prep)
 *  g          [total_tokens, H, d]   output-gate input (post projection)
 *  norm_w     fp32 [d]               RMSNorm weight, shared by the heads
 *  state_in   fp32 [pool_size, H, d, d] initial states (key axis = rows), or
 *             NULL for zeros.  Row of sequence s: state_slots[s] (or s).
 *  state_out  fp32 [pool_size, H, d, d] final states, or NULL to skip; may
 *             equal state_in (updated in place).
 *  y          out [total_tokens, H, d]
 *  workspace  device scratch of at least kda_prefill_workspace_size() bytes,
 *             256-byte aligned; its contents on entry do not matter.
 */
KDA_API int kda_prefill(const kda_config* cfg, int32_t n_seqs, int32_t total_tokens,
                const int32_t* cu_seqlens, const void* q, const void* k,
                const void* v, const float* log_a, const float* beta,
                const void* g, const float* norm_w, const float* state_in,
                float* state_out, const int32_t* state_slots, int32_t pool_size,
                void* y, void* workspace, size_t workspace_bytes,
                kda_stream_t stream);

/*
 * kda_layer_prefill - the whole layer over packed sequences in one call: prep
 * (conv + SiLU + L2 + gate + beta), chunked prefill and gated RMSNorm, from the
 * raw inputs.  For bf16, d = 128, chunk 64, K = 4 the prep runs inside the
 * tensor-core intra-chunk pass (q/k/v stay on chip in fp32); other
 * configurations run kda_prep into the workspace, then the chunked prefill.
 * Results equal kda_prep followed by kda_prefill up to rounding.
 *
 *  x, f, beta_logit, conv_w, A_log, dt_bias, max_seqlen   as in kda_prep
 *  g, norm_w, state_in, state_out, y                      as in kda_prefill
 *  conv_state  [pool_size, K-1, H, 3d] history (NULL = zeros), updated to the
 *              last K-1 pre-conv rows of each sequence (COMMIT)
 *  state_slots / pool_size index both the conv state and the recurrent state.
 *  workspace   at least kda_layer_prefill_workspace_size() bytes, 256-aligned.
 */
KDA_API size_t kda_layer_prefill_workspace_size(const kda_config* cfg, int32_t n_seqs,
                                                int32_t total_tokens);
KDA_API int kda_layer_prefill(const kda_config* cfg, int32_t n_seqs, int32_t total_tokens,
                              const int32_t* cu_seqlens, int32_t max_seqlen, const void* x,
                              const void* f, const void* beta_logit, const void* g,
                              const float* conv_w, const float* A_log, const float* dt_bias,
                              const float* norm_w, void* conv_state, const float* state_in,
                              float* state_out, const int32_t* state_slots, int32_t pool_size,
                              void* y, void* workspace, size_t workspace_bytes,
                              kda_stream_t stream);

/*
 * kda_decode - one token for each of `batch` sequences (the fused operator
 * path of PR #27754: no chunking).  Streams each head's d x d fp32 state once:
 * decay, both column reductions S^T k and S^T q in one pass, rank-1 update,
 * one store, gated RMSNorm.
 *
 *  q, k, v fp32 [batch, H, d]; g [batch, H, d]; log_a fp32 [batch, H, d];
 *  beta fp32 [batch, H]
 *  state      fp32 [pool_size, H, d, d], updated in place (row state_slots[b] or b)
 *  y          out [batch, H, d]
 */
KDA_API int kda_decode(const kda_config* cfg, int32_t batch, const void* q,
               const void* k, const void* v, const float* log_a,
               const float* beta, const void* g, const float* norm_w,
               float* state, const int32_t* state_slots, int32_t pool_size,
               void* y, kda_stream_t stream);

/*
 * kda_layer_decode - one token for each of `batch` sequences from the raw layer
 * inputs: the prep of kda_prep (COMMIT mode: depthwise causal conv against the conv
 * state, which is advanced in place; SiLU; q, k L2 norms; the decay gate; beta) and
 * the step of kda_decode, in one kernel.  Same result as kda_prep + kda_decode.
 *
 *  x [batch, H, 3d] (pre-conv q|k|v); f, g [batch, H, d]; beta_logit [batch, H]
 *    (all in cfg->dtype); conv_w fp32 [H, 3d, K]; A_log fp32 [H]; dt_bias fp32 [H, d]
 *  conv_state [pool_size, K-1, H, 3d] (cfg->dtype), NULL for zeros (then not updated)
 *  state      fp32 [pool_size, H, d, d], updated in place (row state_slots[b] or b)
 *  y          out [batch, H, d]
 */
KDA_API int kda_layer_decode(const kda_config* cfg, int32_t batch, const void* x,
                             const void* f, const void* beta_logit, const void* g,
                             const float* conv_w, const float* A_log, const float* dt_bias,
                             const float* norm_w, void* conv_state, float* state,
                             const int32_t* state_slots, int32_t pool_size, void* y,
                             kda_stream_t stream);

/*
 * kda_layer_verify - kda_prep in TAPE mode and kda_verify in one kernel: a block of
 * `block_len` (1..16) draft tokens per sequence from the raw layer inputs.  The conv
 * state and the recurrent state are only read; the tape and the conv window (history
 * then the block's x rows, for kda_rollback) are written.  Same result as kda_prep
 * (TAPE) + kda_verify.
 *
 *  x [batch, block_len, H, 3d]; f, g [batch, block_len, H, d];
 *  beta_logit [batch, block_len, H]; conv_w, A_log, dt_bias, norm_w as kda_layer_decode
 *  conv_state [pool_size, K-1, H, 3d] or NULL (zeros); state fp32 [pool_size, H, d, d]
 *  tape       out fp32 [batch, block_len, H, d, d]
 *  conv_window out [batch, K-1+block_len, H, 3d] (cfg->dtype)
 *  y          out [batch, block_len, H, d]
 */
KDA_API int kda_layer_verify(const kda_config* cfg, int32_t batch, int32_t block_len,
                             const void* x, const void* f, const void* beta_logit,
                             const void* g, const float* conv_w, const float* A_log,
                             const float* dt_bias, const float* norm_w,
                             const void* conv_state, const float* state,
                             const int32_t* state_slots, int32_t pool_size, float* tape,
                             void* conv_window, void* y, kda_stream_t stream);

/*
 * kda_verify - speculative verify of a block of `block_len` draft tokens per
 * sequence (1..16; the DFlash2 drafter of dflash-mlx issue #63 uses 8).  Runs
 * the decode step block_len times from one load of each state, keeps the live
 * state untouched, and writes the state after every step to the tape, so that
 * rollback to any accepted prefix is a copy.
 *
 *  q, k, v fp32 [batch, block_len, H, d]; g [batch, block_len, H, d];
 *  log_a fp32 [batch, block_len, H, d];
 *  beta fp32 [batch, block_len, H]
 *  state      fp32 [pool_size, H, d, d], read only
 *  tape       out fp32 [batch, block_len, H, d, d]: tape[b, j] = state after draft j
 *  y          out [batch, block_len, H, d]
 */
KDA_API int kda_verify(const kda_config* cfg, int32_t batch, int32_t block_len,
               const void* q, const void* k, const void* v, const float* log_a,
               const float* beta, const void* g, const float* norm_w,
               const float* state, const int32_t* state_slots, int32_t pool_size,
               float* tape, void* y, kda_stream_t stream);

/*
 * kda_rollback - commit the accepted prefix of a verified block.
 * For sequence b with L = accepted[b] (device int32 [batch], clamped to
 * [0, block_len]): L = 0 leaves state and conv state untouched; otherwise
 * state <- tape[b, L-1] and conv_state <- conv_window rows [L, L+K-1) of
 * sequence b.  Bit-exact copies.  conv_window is kda_prep's TAPE output for
 * the block ([batch, K-1+block_len, H, 3d]); conv_state / conv_window may be
 * NULL together to roll back only the recurrent state.
 */
KDA_API int kda_rollback(const kda_config* cfg, int32_t batch, int32_t block_len,
                 const int32_t* accepted, const float* tape,
                 const void* conv_window, float* state, void* conv_state,
                 const int32_t* state_slots, int32_t pool_size,
                 kda_stream_t stream);

/*
 * Compact verify tape and rollback by replay.  dflash-mlx issue #63, "What the backend
 * needs": the KDA recurrent state is to roll back the way the GatedDeltaNet
 * tape-replay path does.  Each verify step changes the state by
 *   S_j = Diag(a_j) S_{j-1} + k_j u_j^T,   u_j = b_j (v_j - (Diag(a_j) S_{j-1})^T k_j),
 * so the step is recorded as the three d-vectors (k_j, u_j, a_j) instead of the
 * d x d state (3d floats: 1.5 KB instead of 64 KB per head at d = 128), and rollback
 * to L accepted drafts replays L such updates from the live state, which verify left
 * untouched.  The replay performs the step kernel's own operations on each element
 * (a multiply by a, then one fused multiply-add of k u), so the rolled-back state is
 * bit-identical to the full tape's entry tape[L-1].
 *
 *  tape_kua  fp32 [batch, block_len, H, 3, d]: per step and head k, u, a (a = e^{log a})
 *
 * kda_verify_compact       - kda_verify writing tape_kua instead of the full tape.
 * kda_layer_verify_compact - kda_layer_verify writing tape_kua instead of the full tape.
 * kda_rollback_replay      - kda_rollback from tape_kua: for L = accepted[b] >= 1 the
 *                            state row is replaced by L replayed steps (in place) and
 *                            the conv state by conv_window rows [L, L+K-1); L = 0 leaves
 *                            both untouched.  Run it on the state verify read, before
 *                            anything else changes that state.
 */
KDA_API int kda_verify_compact(const kda_config* cfg, int32_t batch, int32_t block_len,
                               const void* q, const void* k, const void* v,
                               const float* log_a, const float* beta, const void* g,
                               const float* norm_w, const float* state,
                               const int32_t* state_slots, int32_t pool_size, float* tape_kua,
                               void* y, kda_stream_t stream);
KDA_API int kda_layer_verify_compact(const kda_config* cfg, int32_t batch, int32_t block_len,
                                     const void* x, const void* f, const void* beta_logit,
                                     const void* g, const float* conv_w, const float* A_log,
                                     const float* dt_bias, const float* norm_w,
                                     const void* conv_state, const float* state,
                                     const int32_t* state_slots, int32_t pool_size,
                                     float* tape_kua, void* conv_window, void* y,
                                     kda_stream_t stream);
KDA_API int kda_rollback_replay(const kda_config* cfg, int32_t batch, int32_t block_len,
                                const int32_t* accepted, const float* tape_kua,
                                const void* conv_window, float* state, void* conv_state,
                                const int32_t* state_slots, int32_t pool_size,
                                kda_stream_t stream);

/*
 * kda_proj_gemm - the layer's projections: C = A B^T on the tensor cores, bf16 operands,
 * fp32 accumulation, bf16 results.  glm53-flash-mlx README, quantization recipe: the
 * runtime fuses the six KDA input projections into one matmul; llama.cpp PR #27754, KDA
 * commit: the output gate is low rank, g_b(g_a(x)).  With A the hidden states and B the
 * fused input weight, one call produces q|k|v (pre-conv), f, the beta logit and g_a,
 * each written to its own dense tensor by the output ranges below; a second call with
 * A = g_a and B = the g_b weight produces g.
 *
 *  A       bf16 [M, K] row-major (one row per token)
 *  B       bf16 [N, K] row-major (the weight, one row per output column)
 *  outs    host array of n_outs (1..4) ranges: columns [col_begin, col_end) of C go to
 *          out[row * ld + (col - col_begin)], bf16, device memory.  col_begin, col_end
 *          and ld are multiples of 8, 0 <= col_begin < col_end <= N, ld >= the range's
 *          width, and the ranges do not overlap; columns outside every range are dropped.
 *  status  optional device int32 the caller clears: set to KDA_ERR_TIMEOUT if a bounded
 *          device wait gave up (read it with kda_workspace_status), or NULL.
 *  M >= 0, N >= 0 (a multiple of 8), K >= 8 (a multiple of 8); M = 0 or N = 0 launches
 *  nothing.
 */
typedef struct kda_proj_out {
  void* out;
  int64_t ld;
  int32_t col_begin, col_end;
} kda_proj_out;
KDA_API int kda_proj_gemm(int32_t M, int32_t N, int32_t K, const void* A, const void* B,
                          const kda_proj_out* outs, int32_t n_outs, void* status,
                          kda_stream_t stream);

/*
 * kda_workspace_status - synchronises `stream`, then reads the status word
 * the prefill kernels keep at the start of `workspace`.  Returns KDA_OK, or
 * KDA_ERR_TIMEOUT when a bounded device wait of the last kda_prefill on this
 * workspace gave up (its outputs are then invalid).
 */
KDA_API int kda_workspace_status(const void* workspace, kda_stream_t stream);

/*
 * kda_prefill_noalloc - kda_prefill for callers that cannot allocate device
 * memory.  The pages have no counterpart to this entry point.
 *
 * Some callers cannot call cudaMalloc: code embedded in a host framework that owns
 * every byte of device memory (a serving engine that reserves the whole HBM for
 * its own pools up front), or a path that must not pay cudaMalloc's latency and
 * device-wide synchronisation.  This entry point takes the same inputs and
 * outputs as kda_prefill (the caller still passes and owns them) but keeps its
 * scratch in one fixed array of KDA_NOALLOC_SCRATCH_BYTES (64 MiB) of device
 * memory inside the library, so it allocates nothing and frees nothing.
 *
 *  - Limit: problems whose kda_prefill_workspace_size() exceeds
 *    KDA_NOALLOC_SCRATCH_BYTES are rejected with KDA_ERR_SCRATCH_LIMIT before
 *    anything is launched (at H = 32, d = 128, chunk 64, bf16 a single sequence
 *    of about 1,000 tokens fits).
 *  - Memory: every GPU that loads the library holds the 64 MiB until the process
 *    exits.
 *  - Set-up: every call looks up the array's device address on the current
 *    device (nothing is cached, so the address stays right after a
 *    cudaDeviceReset); the first call on a device also loads the library's
 *    device code there, so make that first call before any stream capture.
 *  - Sharing: every call on a device uses the same array, which keeps the last
 *    call's contents.  Calls that overlap on the GPU (different streams, or
 *    different host threads) race on it and give undefined results; order them.
 *  - Status: kda_workspace_status cannot see this scratch; a bounded-wait
 *    timeout here leaves the outputs invalid without a readable status word.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
KDA_API int kda_prefill_noalloc(const kda_config* cfg, int32_t n_seqs, int32_t total_tokens,
                                const int32_t* cu_seqlens, const void* q, const void* k,
                                const void* v, const float* log_a, const float* beta,
                                const void* g, const float* norm_w, const float* state_in,
                                float* state_out, const int32_t* state_slots,
                                int32_t pool_size, void* y, kda_stream_t stream);

/*
 * kda_selftest_wait_timeout - failure-detection self-test.  Enqueues one warp
 * that waits, with the same bounded wait the prefill pipeline uses, on a
 * barrier nothing ever completes; after about a quarter of a second it gives up
 * and records KDA_ERR_TIMEOUT in the status word at the start of `workspace`
 * (>= 256 bytes, 256-byte aligned, device memory), which it clears first.  A
 * following kda_workspace_status returns KDA_ERR_TIMEOUT and the context stays
 * usable.  No trap, no fault, no unbounded wait.
 */
KDA_API int kda_selftest_wait_timeout(void* workspace, kda_stream_t stream);

/*
 * kda_set_phase_events - measurement hook (the pages have no counterpart).
 * `events` holds n <= 3 cudaEvent_t handles (created by the caller, owned by
 * the caller, may be NULL entries); while set, every kda_prefill,
 * kda_prefill_noalloc and kda_layer_prefill issued from THIS host thread
 * records events[0] after the intra-chunk pass, events[1] after the
 * inter-chunk pass and events[2] after the output norm, on the call's stream.
 * The kernels are unchanged.  n = 0 (events may be NULL) clears the hook.
 * Returns KDA_ERR_INVALID_ARG for n outside [0, 3] or events NULL with n > 0.
 */
KDA_API int kda_set_phase_events(void* const* events, int32_t n);

/*
 * kda_launch_count - measurement hook (the pages have no counterpart): the number
 * of kernels the library has launched from THIS host thread since it was loaded
 * (cumulative; take differences around the calls of interest).  Launches only:
 * cudaMemsetAsync and other runtime calls are not counted.
 */
KDA_API long long kda_launch_count(void);

/*
 * kda_last_cuda_error - the CUDA runtime's message for the error behind the most
 * recent KDA_ERR_CUDA returned to THIS host thread ("no error" if there was none).
 * Static string; do not free.
 */
KDA_API const char* kda_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
