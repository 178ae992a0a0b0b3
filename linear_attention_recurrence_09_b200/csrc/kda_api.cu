// C ABI of libkda.so (declarations and contracts in include/kda.h).
// Host-side validation happens before any launch; nothing here allocates.
#include <cmath>
#include <cstdint>

#include "../../include/kda.h"
#include "kda_launch.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_cfg(const kda_config* c) {
  if (c == nullptr) return KDA_ERR_INVALID_ARG;
  if (c->num_heads < 1 || c->conv_size < 1 || c->conv_size > kda::prep_kmax())
    return KDA_ERR_INVALID_ARG;
  if (c->dtype != KDA_F32 && c->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (c->head_dim != 16 && c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128)
    return KDA_ERR_UNSUPPORTED;
  if (c->chunk_size != 16 && c->chunk_size != 32 && c->chunk_size != 64)
    return KDA_ERR_UNSUPPORTED;
  if (c->gate_kind != KDA_GATE_BOUNDED_SIGMOID && c->gate_kind != KDA_GATE_SOFTPLUS)
    return KDA_ERR_INVALID_ARG;
  // lb >= -5 keeps a 16-token sub-chunk's decay span <= 80 (< fp32 exp overflow); the
  // softplus gate ignores lb
  if (c->gate_kind == KDA_GATE_BOUNDED_SIGMOID &&
      (!std::isfinite(c->gate_lower_bound) || c->gate_lower_bound < -5.0f ||
       c->gate_lower_bound >= 0.0f))
    return KDA_ERR_UNSUPPORTED;
  if (!(c->l2_eps > 0.0f) || !std::isfinite(c->l2_eps)) return KDA_ERR_INVALID_ARG;
  if (!(c->norm_eps >= 0.0f) || !std::isfinite(c->norm_eps)) return KDA_ERR_INVALID_ARG;
  if (!std::isfinite(c->q_scale)) return KDA_ERR_INVALID_ARG;
  if ((c->launch_flags & ~(KDA_LAUNCH_EARLY_STATE | KDA_LAUNCH_SEPARATE_PASSES)) != 0)
    return KDA_ERR_INVALID_ARG;
  return KDA_OK;
}

// every non-null pointer 16-byte aligned; required ones non-null
int check_ptrs(std::initializer_list<const void*> required,
               std::initializer_list<const void*> optional) {
  for (const void* p : required) {
    if (p == nullptr) return KDA_ERR_INVALID_ARG;
    if (!aligned16(p)) return KDA_ERR_MISALIGNED;
  }
  for (const void* p : optional)
    if (p != nullptr && !aligned16(p)) return KDA_ERR_MISALIGNED;
  return KDA_OK;
}

int check_pool(const int32_t* slots, int32_t pool_size, int32_t n) {
  if (pool_size < 0) return KDA_ERR_INVALID_ARG;
  if (slots == nullptr && pool_size < n) return KDA_ERR_INVALID_ARG;
  if (slots != nullptr && n > 0 && pool_size < 1) return KDA_ERR_INVALID_ARG;
  return KDA_OK;
}

cudaError_t& last_cuda_error() {
  static thread_local cudaError_t e = cudaSuccess;
  return e;
}
int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return KDA_OK;
  last_cuda_error() = e;
  return KDA_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* kda_status_string(int status) {
  switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: null pointer, bad size or bad enum";
    case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED: a pointer is not 16-byte aligned";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: configuration not built";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA launch or runtime call failed";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device wait gave up";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
    case KDA_ERR_SCRATCH_LIMIT:
      return "KDA_ERR_SCRATCH_LIMIT: problem exceeds the fixed scratch of kda_prefill_noalloc";
  }
  return "unknown kda status";
}

int kda_abi_version(void) { return 2; }

int kda_prep(const kda_config* cfg, int32_t n_seqs, int32_t total_tokens,
             const int32_t* cu_seqlens, int32_t max_seqlen, const void* x, const void* f,
             const void* beta_logit, const float* conv_w, const float* A_log,
             const float* dt_bias, void* conv_state, const int32_t* state_slots,
             int32_t pool_size, int32_t conv_mode, void* conv_window, void* q, void* k,
             void* v, float* log_a, float* beta, kda_stream_t stream) {
  int st = check_cfg(cfg);
  if (st) return st;
  if (n_seqs < 0 || total_tokens < 0 || max_seqlen < 0) return KDA_ERR_INVALID_ARG;
  if (conv_mode != KDA_CONV_COMMIT && conv_mode != KDA_CONV_TAPE) return KDA_ERR_INVALID_ARG;
  if (n_seqs == 0) return KDA_OK;
  if ((st = check_ptrs({cu_seqlens, conv_w, A_log, dt_bias}, {conv_state, state_slots})))
    return st;
  if (conv_state != nullptr && (st = check_pool(state_slots, pool_size, n_seqs))) return st;
  if (conv_mode == KDA_CONV_TAPE && (st = check_ptrs({conv_window}, {}))) return st;
  if (total_tokens > 0 &&
      (st = check_ptrs({x, f, beta_logit, q, k, v, log_a, beta}, {})))
    return st;
  kda::PrepArgs a{};
  a.cu = cu_seqlens; a.n_seqs = n_seqs; a.total = total_tokens;
  a.H = cfg->num_heads; a.D = cfg->head_dim; a.K = cfg->conv_size;
  a.bf16 = cfg->dtype == KDA_BF16;
  a.x = x; a.f = f; a.beta_logit = beta_logit;
  a.conv_w = conv_w; a.A_log = A_log; a.dt_bias = dt_bias;
  // without a conv state there is no pool to index: every sequence is processed
  a.conv_state = conv_state;
  a.slots = conv_state ? state_slots : nullptr;
  a.pool_size = conv_state ? pool_size : n_seqs;
  a.mode = conv_mode;
  a.commit_in_kernel = (max_seqlen >= 1 && max_seqlen <= kda::prep_tile()) ? 1 : 0;
  a.short_tb = max_seqlen < 1 ? 0 : max_seqlen == 1 ? 1 : max_seqlen <= 8 ? 8
             : max_seqlen <= 16 ? 16 : 0;
  a.window = conv_window;
  a.q = static_cast<float*>(q); a.k = static_cast<float*>(k); a.v = static_cast<float*>(v);
  a.loga = log_a; a.beta = beta;
  a.lb = cfg->gate_lower_bound; a.l2_eps = cfg->l2_eps;
  a.gate_softplus = cfg->gate_kind == KDA_GATE_SOFTPLUS;
  return cuda_status(kda::launch_prep(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t kda_prefill_workspace_size(const kda_config* cfg, int32_t n_seqs, int32_t total_tokens) {
  if (check_cfg(cfg) != KDA_OK || n_seqs < 0 || total_tokens < 0) return 0;
  return kda::prefill_layout(n_seqs, total_tokens, cfg->num_heads, cfg->head_dim,
                             cfg->chunk_size, cfg->dtype == KDA_BF16).total;
}

int kda_prefill(const kda_config* cfg, int32_t n_seqs, int32_t total_tokens,
                const int32_t* cu_seqlens, const void* q, const void* k, const void* v,
                const float* log_a, const float* beta, const void* g, const float* norm_w,
                const float* state_in, float* state_out, const int32_t* state_slots,
                int32_t pool_size, void* y, void* workspace, size_t workspace_bytes,
                kda_stream_t stream) {
  int st = check_cfg(cfg);
  if (st) return st;
  if (n_seqs < 0 || total_tokens < 0) return KDA_ERR_INVALID_ARG;
  if (n_seqs == 0) return KDA_OK;
  if ((st = check_ptrs({cu_seqlens, norm_w}, {state_in, state_out, state_slots}))) return st;
  if ((state_in != nullptr || state_out != nullptr) &&
      (st = check_pool(state_slots, pool_size, n_seqs)))
    return st;
  if (total_tokens > 0 && (st = check_ptrs({q, k, v, log_a, beta, g, y}, {}))) return st;
  const kda::PrefillLayout L =
      kda::prefill_layout(n_seqs, total_tokens, cfg->num_heads, cfg->head_dim,
                          cfg->chunk_size, cfg->dtype == KDA_BF16);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < L.total)
    return KDA_ERR_WORKSPACE;
  kda::PrefillArgs a{};
  a.cu = cu_seqlens; a.n_seqs = n_seqs; a.total = total_tokens;
  a.H = cfg->num_heads; a.D = cfg->head_dim; a.C = cfg->chunk_size;
  a.bf16 = cfg->dtype == KDA_BF16;
  a.q = static_cast<const float*>(q); a.k = static_cast<const float*>(k);
  a.v = static_cast<const float*>(v);
  a.loga = log_a; a.beta = beta; a.g = g; a.norm_w = norm_w;
  // without states there is no pool to index: every sequence is processed
  const bool pooled = state_in != nullptr || state_out != nullptr;
  a.state_in = state_in; a.state_out = state_out;
  a.slots = pooled ? state_slots : nullptr;
  a.pool_size = pooled ? pool_size : n_seqs;
  a.y = y; a.ws = static_cast<char*>(workspace); a.L = L;
  a.norm_eps = cfg->norm_eps; a.q_scale = cfg->q_scale; a.lb = cfg->gate_lower_bound;
  a.gate_softplus = cfg->gate_kind == KDA_GATE_SOFTPLUS;
  a.separate_passes = (cfg->launch_flags & KDA_LAUNCH_SEPARATE_PASSES) != 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(a.ws + L.status, 0, L.zeroed - L.status, s) != cudaSuccess) return KDA_ERR_CUDA;
  return cuda_status(kda::launch_prefill(a, s));
}

// Bytes the fallback of kda_layer_prefill (separate prep, then the chunked
// prefill) needs on top of the prefill workspace: fp32 q, k, v, log a and beta.
static size_t layer_prep_bytes(const kda_config* c, int32_t total) {
  const size_t th = (size_t)total * c->num_heads;
  return ((th * c->head_dim * 4 * 4 + th * 4) + 255) & ~(size_t)255;
}

// prep inside the tcgen05 intra-chunk pass: bf16, d = 128, chunk 64, K = 4, bounded gate
static bool layer_fused(const kda_config* c) {
  return c->dtype == KDA_BF16 && c->head_dim == 128 && c->chunk_size == 64 &&
         c->conv_size == 4 && c->gate_kind == KDA_GATE_BOUNDED_SIGMOID;
}

size_t kda_layer_prefill_workspace_size(const kda_config* cfg, int32_t n_seqs,
                                        int32_t total_tokens) {
  const size_t base = kda_prefill_workspace_size(cfg, n_seqs, total_tokens);
  if (base == 0) return 0;
  return layer_fused(cfg) ? base : base + layer_prep_bytes(cfg, total_tokens);
}

int kda_layer_prefill(const kda_config* cfg, int32_t n_seqs, int32_t total_tokens,
                      const int32_t* cu_seqlens, int32_t max_seqlen, const void* x,
                      const void* f, const void* beta_logit, const void* g,
                      const float* conv_w, const float* A_log, const float* dt_bias,
                      const float* norm_w, void* conv_state, const float* state_in,
                      float* state_out, const int32_t* state_slots, int32_t pool_size, void* y,
                      void* workspace, size_t workspace_bytes, kda_stream_t stream) {
  int st = check_cfg(cfg);
  if (st) return st;
  if (n_seqs < 0 || total_tokens < 0 || max_seqlen < 0) return KDA_ERR_INVALID_ARG;
  if (n_seqs == 0) return KDA_OK;
  if ((st = check_ptrs({cu_seqlens, conv_w, A_log, dt_bias, norm_w},
                       {conv_state, state_in, state_out, state_slots})))
    return st;
  const bool pooled = conv_state != nullptr || state_in != nullptr || state_out != nullptr;
  if (pooled && (st = check_pool(state_slots, pool_size, n_seqs))) return st;
  if (total_tokens > 0 && (st = check_ptrs({x, f, beta_logit, g, y}, {}))) return st;
  const size_t need = kda_layer_prefill_workspace_size(cfg, n_seqs, total_tokens);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < need)
    return KDA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const kda::PrefillLayout L =
      kda::prefill_layout(n_seqs, total_tokens, cfg->num_heads, cfg->head_dim,
                          cfg->chunk_size, cfg->dtype == KDA_BF16);
  const int32_t* slots = pooled ? state_slots : nullptr;
  const int32_t pool = pooled ? pool_size : n_seqs;

  // prep arguments: the commit of the conv state (fused path) or the whole prep (fallback)
  kda::PrepArgs p{};
  p.cu = cu_seqlens; p.n_seqs = n_seqs; p.total = total_tokens;
  p.H = cfg->num_heads; p.D = cfg->head_dim; p.K = cfg->conv_size;
  p.bf16 = cfg->dtype == KDA_BF16;
  p.x = x; p.f = f; p.beta_logit = beta_logit;
  p.conv_w = conv_w; p.A_log = A_log; p.dt_bias = dt_bias;
  p.conv_state = conv_state; p.slots = conv_state ? slots : nullptr;
  p.pool_size = conv_state ? pool : n_seqs;
  p.mode = KDA_CONV_COMMIT;
  p.lb = cfg->gate_lower_bound; p.l2_eps = cfg->l2_eps;
  p.gate_softplus = cfg->gate_kind == KDA_GATE_SOFTPLUS;

  kda::PrefillArgs a{};
  a.cu = cu_seqlens; a.n_seqs = n_seqs; a.total = total_tokens;
  a.H = cfg->num_heads; a.D = cfg->head_dim; a.C = cfg->chunk_size;
  a.bf16 = cfg->dtype == KDA_BF16;
  a.g = g; a.norm_w = norm_w;
  a.state_in = state_in; a.state_out = state_out;
  a.slots = slots; a.pool_size = pool;
  a.y = y; a.ws = static_cast<char*>(workspace); a.L = L;
  a.norm_eps = cfg->norm_eps; a.q_scale = cfg->q_scale; a.lb = cfg->gate_lower_bound;
  a.l2_eps = cfg->l2_eps; a.K = cfg->conv_size;
  a.gate_softplus = cfg->gate_kind == KDA_GATE_SOFTPLUS;
  a.separate_passes = (cfg->launch_flags & KDA_LAUNCH_SEPARATE_PASSES) != 0;
  if (cudaMemsetAsync(a.ws + L.status, 0, L.zeroed - L.status, s) != cudaSuccess) return KDA_ERR_CUDA;

  if (layer_fused(cfg)) {
    // prep runs inside the intra-chunk pass; the conv state is committed afterwards
    a.x = x; a.f = f; a.beta_logit = beta_logit;
    a.conv_w = conv_w; a.A_log = A_log; a.dt_bias = dt_bias; a.conv_state = conv_state;
    if ((st = cuda_status(kda::launch_prefill(a, s)))) return st;
    p.commit_in_kernel = 0;
    return cuda_status(kda::launch_conv_commit(p, s));
  }
  // fallback: prep into the tail of the workspace, then the chunked prefill
  const size_t th = (size_t)total_tokens * cfg->num_heads;
  float* q = reinterpret_cast<float*>(a.ws + L.total);
  float* k = q + th * cfg->head_dim;
  float* v = k + th * cfg->head_dim;
  float* la = v + th * cfg->head_dim;
  float* be = la + th * cfg->head_dim;
  p.q = q; p.k = k; p.v = v; p.loga = la; p.beta = be;
  p.commit_in_kernel = (max_seqlen >= 1 && max_seqlen <= kda::prep_tile()) ? 1 : 0;
  if ((st = cuda_status(kda::launch_prep(p, s)))) return st;
  a.q = q; a.k = k; a.v = v; a.loga = la; a.beta = be;
  return cuda_status(kda::launch_prefill(a, s));
}

long long kda_launch_count(void) { return kda::launch_counter(); }

const char* kda_last_cuda_error(void) { return cudaGetErrorString(last_cuda_error()); }

int kda_set_phase_events(void* const* events, int32_t n) {
  if (n < 0 || n > 3 || (n > 0 && events == nullptr)) return KDA_ERR_INVALID_ARG;
  kda::PhaseEvents& pe = kda::phase_events();
  for (int i = 0; i < 3; ++i) pe.ev[i] = (i < n) ? static_cast<cudaEvent_t>(events[i]) : nullptr;
  return KDA_OK;
}

static int step_common(const kda_config* cfg, int32_t batch, int32_t T, const void* q,
                       const void* k, const void* v, const float* log_a, const float* beta,
                       const void* g, const float* norm_w, const float* state_in,
                       float* state_out, float* tape, float* tape_kua, const int32_t* slots,
                       int32_t pool_size, void* y, kda_stream_t stream) {
  int st = check_cfg(cfg);
  if (st) return st;
  if (batch < 0) return KDA_ERR_INVALID_ARG;
  if (batch == 0) return KDA_OK;
  if ((st = check_ptrs({q, k, v, log_a, beta, g, norm_w, state_in, y}, {slots}))) return st;
  if ((st = check_pool(slots, pool_size, batch))) return st;
  kda::StepArgs a{};
  a.B = batch; a.T = T; a.H = cfg->num_heads; a.D = cfg->head_dim;
  a.bf16 = cfg->dtype == KDA_BF16;
  a.q = static_cast<const float*>(q); a.k = static_cast<const float*>(k);
  a.v = static_cast<const float*>(v);
  a.loga = log_a; a.beta = beta; a.g = g; a.norm_w = norm_w;
  a.state_in = state_in; a.state_out = state_out; a.tape = tape; a.tape_kua = tape_kua;
  a.slots = slots; a.pool_size = pool_size; a.y = y;
  a.norm_eps = cfg->norm_eps; a.q_scale = cfg->q_scale;
  a.early_state = (cfg->launch_flags & KDA_LAUNCH_EARLY_STATE) != 0;
  return cuda_status(kda::launch_step(a, reinterpret_cast<cudaStream_t>(stream)));
}

static int layer_step_common(const kda_config* cfg, int32_t batch, int32_t T, const void* x,
                             const void* f, const void* beta_logit, const void* g,
                             const float* conv_w, const float* A_log, const float* dt_bias,
                             const float* norm_w, void* conv_state, const float* state_in,
                             float* state_out, float* tape, float* tape_kua, void* window,
                             const int32_t* slots, int32_t pool_size, void* y,
                             kda_stream_t stream) {
  int st = check_cfg(cfg);
  if (st) return st;
  if (batch < 0) return KDA_ERR_INVALID_ARG;
  if (batch == 0) return KDA_OK;
  if ((st = check_ptrs({x, f, beta_logit, g, conv_w, A_log, dt_bias, norm_w, state_in, y},
                       {slots, conv_state, window})))
    return st;
  if ((st = check_pool(slots, pool_size, batch))) return st;
  kda::StepArgs a{};
  a.B = batch; a.T = T; a.H = cfg->num_heads; a.D = cfg->head_dim;
  a.bf16 = cfg->dtype == KDA_BF16;
  a.g = g; a.norm_w = norm_w;
  a.state_in = state_in; a.state_out = state_out; a.tape = tape; a.tape_kua = tape_kua;
  a.slots = slots; a.pool_size = pool_size; a.y = y;
  a.norm_eps = cfg->norm_eps; a.q_scale = cfg->q_scale;
  a.x = x; a.f = f; a.beta_logit = beta_logit;
  a.conv_w = conv_w; a.A_log = A_log; a.dt_bias = dt_bias;
  a.conv_state = conv_state; a.window = window; a.K = cfg->conv_size;
  a.lb = cfg->gate_lower_bound; a.l2_eps = cfg->l2_eps;
  a.gate_softplus = cfg->gate_kind == KDA_GATE_SOFTPLUS;
  a.early_state = (cfg->launch_flags & KDA_LAUNCH_EARLY_STATE) != 0;
  return cuda_status(kda::launch_step(a, reinterpret_cast<cudaStream_t>(stream)));
}

int kda_layer_decode(const kda_config* cfg, int32_t batch, const void* x, const void* f,
                     const void* beta_logit, const void* g, const float* conv_w,
                     const float* A_log, const float* dt_bias, const float* norm_w,
                     void* conv_state, float* state, const int32_t* state_slots,
                     int32_t pool_size, void* y, kda_stream_t stream) {
  return layer_step_common(cfg, batch, 1, x, f, beta_logit, g, conv_w, A_log, dt_bias, norm_w,
                           conv_state, state, state, nullptr, nullptr, nullptr, state_slots,
                           pool_size, y, stream);
}

static int layer_verify_common(const kda_config* cfg, int32_t batch, int32_t block_len,
                               const void* x, const void* f, const void* beta_logit,
                               const void* g, const float* conv_w, const float* A_log,
                               const float* dt_bias, const float* norm_w,
                               const void* conv_state, const float* state,
                               const int32_t* state_slots, int32_t pool_size, float* tape,
                               float* tape_kua, void* conv_window, void* y,
                               kda_stream_t stream) {
  if (block_len < 1 || block_len > 16) return KDA_ERR_INVALID_ARG;
  if (batch > 0) {
    int st = check_ptrs({tape ? tape : tape_kua, conv_window}, {});
    if (st) return st;
  }
  return layer_step_common(cfg, batch, block_len, x, f, beta_logit, g, conv_w, A_log, dt_bias,
                           norm_w, const_cast<void*>(conv_state), state, nullptr, tape,
                           tape_kua, conv_window, state_slots, pool_size, y, stream);
}

int kda_layer_verify(const kda_config* cfg, int32_t batch, int32_t block_len, const void* x,
                     const void* f, const void* beta_logit, const void* g,
                     const float* conv_w, const float* A_log, const float* dt_bias,
                     const float* norm_w, const void* conv_state, const float* state,
                     const int32_t* state_slots, int32_t pool_size, float* tape,
                     void* conv_window, void* y, kda_stream_t stream) {
  if (batch > 0 && tape == nullptr) return KDA_ERR_INVALID_ARG;
  return layer_verify_common(cfg, batch, block_len, x, f, beta_logit, g, conv_w, A_log,
                             dt_bias, norm_w, conv_state, state, state_slots, pool_size, tape,
                             nullptr, conv_window, y, stream);
}

int kda_layer_verify_compact(const kda_config* cfg, int32_t batch, int32_t block_len,
                             const void* x, const void* f, const void* beta_logit,
                             const void* g, const float* conv_w, const float* A_log,
                             const float* dt_bias, const float* norm_w,
                             const void* conv_state, const float* state,
                             const int32_t* state_slots, int32_t pool_size, float* tape_kua,
                             void* conv_window, void* y, kda_stream_t stream) {
  if (batch > 0 && tape_kua == nullptr) return KDA_ERR_INVALID_ARG;
  return layer_verify_common(cfg, batch, block_len, x, f, beta_logit, g, conv_w, A_log,
                             dt_bias, norm_w, conv_state, state, state_slots, pool_size,
                             nullptr, tape_kua, conv_window, y, stream);
}

int kda_decode(const kda_config* cfg, int32_t batch, const void* q, const void* k,
               const void* v, const float* log_a, const float* beta, const void* g,
               const float* norm_w, float* state, const int32_t* state_slots,
               int32_t pool_size, void* y, kda_stream_t stream) {
  return step_common(cfg, batch, 1, q, k, v, log_a, beta, g, norm_w, state, state, nullptr,
                     nullptr, state_slots, pool_size, y, stream);
}

int kda_verify(const kda_config* cfg, int32_t batch, int32_t block_len, const void* q,
               const void* k, const void* v, const float* log_a, const float* beta,
               const void* g, const float* norm_w, const float* state,
               const int32_t* state_slots, int32_t pool_size, float* tape, void* y,
               kda_stream_t stream) {
  if (block_len < 1 || block_len > 16) return KDA_ERR_INVALID_ARG;
  if (batch > 0) {
    int st = check_ptrs({tape}, {});
    if (st) return st;
  }
  return step_common(cfg, batch, block_len, q, k, v, log_a, beta, g, norm_w, state, nullptr,
                     tape, nullptr, state_slots, pool_size, y, stream);
}

int kda_verify_compact(const kda_config* cfg, int32_t batch, int32_t block_len, const void* q,
                       const void* k, const void* v, const float* log_a, const float* beta,
                       const void* g, const float* norm_w, const float* state,
                       const int32_t* state_slots, int32_t pool_size, float* tape_kua,
                       void* y, kda_stream_t stream) {
  if (block_len < 1 || block_len > 16) return KDA_ERR_INVALID_ARG;
  if (batch > 0) {
    int st = check_ptrs({tape_kua}, {});
    if (st) return st;
  }
  return step_common(cfg, batch, block_len, q, k, v, log_a, beta, g, norm_w, state, nullptr,
                     nullptr, tape_kua, state_slots, pool_size, y, stream);
}

int kda_rollback(const kda_config* cfg, int32_t batch, int32_t block_len,
                 const int32_t* accepted, const float* tape, const void* conv_window,
                 float* state, void* conv_state, const int32_t* state_slots,
                 int32_t pool_size, kda_stream_t stream) {
  int st = check_cfg(cfg);
  if (st) return st;
  if (batch < 0 || block_len < 1 || block_len > 16) return KDA_ERR_INVALID_ARG;
  if (batch == 0) return KDA_OK;
  if ((conv_window == nullptr) != (conv_state == nullptr)) return KDA_ERR_INVALID_ARG;
  if ((st = check_ptrs({accepted, tape, state}, {conv_window, conv_state, state_slots})))
    return st;
  if ((st = check_pool(state_slots, pool_size, batch))) return st;
  kda::RollbackArgs a{};
  a.B = batch; a.T = block_len; a.H = cfg->num_heads; a.D = cfg->head_dim;
  a.K = cfg->conv_size; a.bf16 = cfg->dtype == KDA_BF16;
  a.accepted = accepted; a.tape = tape; a.window = conv_window; a.state = state;
  a.conv_state = conv_state; a.slots = state_slots; a.pool_size = pool_size;
  return cuda_status(kda::launch_rollback(a, reinterpret_cast<cudaStream_t>(stream)));
}

int kda_rollback_replay(const kda_config* cfg, int32_t batch, int32_t block_len,
                        const int32_t* accepted, const float* tape_kua,
                        const void* conv_window, float* state, void* conv_state,
                        const int32_t* state_slots, int32_t pool_size, kda_stream_t stream) {
  int st = check_cfg(cfg);
  if (st) return st;
  if (batch < 0 || block_len < 1 || block_len > 16) return KDA_ERR_INVALID_ARG;
  if (batch == 0) return KDA_OK;
  if ((conv_window == nullptr) != (conv_state == nullptr)) return KDA_ERR_INVALID_ARG;
  if ((st = check_ptrs({accepted, tape_kua, state}, {conv_window, conv_state, state_slots})))
    return st;
  if ((st = check_pool(state_slots, pool_size, batch))) return st;
  kda::RollbackArgs a{};
  a.B = batch; a.T = block_len; a.H = cfg->num_heads; a.D = cfg->head_dim;
  a.K = cfg->conv_size; a.bf16 = cfg->dtype == KDA_BF16;
  a.accepted = accepted; a.tape_kua = tape_kua; a.window = conv_window; a.state = state;
  a.conv_state = conv_state; a.slots = state_slots; a.pool_size = pool_size;
  a.early_state = (cfg->launch_flags & KDA_LAUNCH_EARLY_STATE) != 0;
  return cuda_status(kda::launch_rollback(a, reinterpret_cast<cudaStream_t>(stream)));
}

int kda_proj_gemm(int32_t M, int32_t N, int32_t K, const void* A, const void* B,
                  const kda_proj_out* outs, int32_t n_outs, void* status,
                  kda_stream_t stream) {
  if (M < 0 || N < 0 || K < 8 || (K % 8) != 0 || (N % 8) != 0) return KDA_ERR_INVALID_ARG;
  if (outs == nullptr || n_outs < 1 || n_outs > kda::proj_gemm_max_outs())
    return KDA_ERR_INVALID_ARG;
  int st;
  if ((st = check_ptrs({A, B}, {})) != KDA_OK) return st;
  if (status != nullptr && (reinterpret_cast<uintptr_t>(status) & 3u) != 0)
    return KDA_ERR_MISALIGNED;
  kda::ProjOut po[4];
  for (int i = 0; i < n_outs; ++i) {
    const kda_proj_out& o = outs[i];
    if ((st = check_ptrs({o.out}, {})) != KDA_OK) return st;
    if (o.col_begin < 0 || o.col_end > N || o.col_begin >= o.col_end ||
        (o.col_begin % 8) != 0 || (o.col_end % 8) != 0 || (o.ld % 8) != 0 ||
        o.ld < (int64_t)(o.col_end - o.col_begin))
      return KDA_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j)
      if (o.col_begin < outs[j].col_end && outs[j].col_begin < o.col_end)
        return KDA_ERR_INVALID_ARG;
    po[i].out = o.out; po[i].ld = o.ld; po[i].col_begin = o.col_begin; po[i].col_end = o.col_end;
  }
  if (M == 0 || N == 0) return KDA_OK;
  return cuda_status(kda::launch_proj_gemm(M, N, K, A, B, po, n_outs, static_cast<int*>(status),
                                           reinterpret_cast<cudaStream_t>(stream)));
}

int kda_selftest_wait_timeout(void* workspace, kda_stream_t stream) {
  if (workspace == nullptr) return KDA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, 256, s) != cudaSuccess) return KDA_ERR_CUDA;
  return cuda_status(kda::launch_wait_timeout_selftest(workspace, s));
}

int kda_workspace_status(const void* workspace, kda_stream_t stream) {
  if (workspace == nullptr) return KDA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return KDA_ERR_CUDA;
  return word == 0 ? KDA_OK : KDA_ERR_TIMEOUT;
}

}  // extern "C"
