// Internal launch interface between the C ABI (kda_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kda {

struct PrepArgs {
  const int32_t* cu;
  int n_seqs, total, H, D, K;
  bool bf16;
  const void* x;
  const void* f;
  const void* beta_logit;
  const float* conv_w;
  const float* A_log;
  const float* dt_bias;
  void* conv_state;
  const int32_t* slots;
  int pool_size;
  int mode;  // 0 commit, 1 tape
  int commit_in_kernel;
  int short_tb;        // > 0: every sequence has at most about this many tokens (1, 8, 16)
  void* window;
  float* q;
  float* k;
  float* v;
  float* loga;
  float* beta;
  float lb, l2_eps;
  int gate_softplus;   // 1: log a = -A softplus(f + dt_bias); 0: lb sigmoid(A (f + dt_bias))
};

struct StepArgs {  // decode (T = 1) and verify (T = block_len)
  int B, T, H, D;
  bool bf16;
  const float* q;
  const float* k;
  const float* v;
  const float* loga;
  const float* beta;
  const void* g;
  const float* norm_w;
  const float* state_in;
  float* state_out;  // decode: == state_in; verify: nullptr
  float* tape;       // verify only: the state after every step
  float* tape_kua;   // verify only: k, u and a of every step (the compact tape)
  const int32_t* slots;
  int pool_size;
  void* y;
  float norm_eps, q_scale;
  // raw inputs of the fused prep (kda_layer_decode / kda_layer_verify); x == nullptr otherwise
  const void* x;            // [B, T, H, 3d] pre-conv q|k|v
  const void* f;            // [B, T, H, d]
  const void* beta_logit;   // [B, T, H]
  const float* conv_w;      // [H, 3d, K]
  const float* A_log;       // [H]
  const float* dt_bias;     // [H, d]
  void* conv_state;         // [pool, K-1, H, 3d]: updated in place (decode) or read (verify)
  void* window;             // verify: [B, K-1+T, H, 3d] = [history; x] for rollback
  int K;
  float lb, l2_eps;
  int gate_softplus;        // as in PrepArgs
  bool early_state;         // stream the state before waiting for the previous kernel
};

struct RollbackArgs {
  int B, T, H, D, K;
  bool bf16;
  const int32_t* accepted;
  const float* tape;       // full-state tape, or
  const float* tape_kua;   // the compact tape, replayed from the live state
  const void* window;
  float* state;
  void* conv_state;
  const int32_t* slots;
  int pool_size;
  bool early_state;        // replay: as in StepArgs
};

// Workspace of the chunked prefill (byte offsets from its base, 256-aligned).
struct PrefillLayout {
  size_t status, flags, zeroed, W, Ut, Qt, Kp, o, M, gC, total;
  int nslots;
  size_t wsize;  // bytes per workspace element (4 fp32 / 2 bf16)
};
PrefillLayout prefill_layout(int n_seqs, int total, int H, int D, int C, bool bf16);

struct PrefillArgs {
  const int32_t* cu;
  int n_seqs, total, H, D, C;
  bool bf16;
  const float* q;
  const float* k;
  const float* v;
  const float* loga;
  const float* beta;
  const void* g;
  const float* norm_w;
  const float* state_in;
  float* state_out;
  const int32_t* slots;
  int pool_size;
  void* y;
  char* ws;
  PrefillLayout L;
  float norm_eps, q_scale, lb, l2_eps;
  // raw inputs of the fused prep path (kda_layer_prefill); x == nullptr otherwise
  const void* x;
  const void* f;
  const void* beta_logit;
  const float* conv_w;
  const float* A_log;
  const float* dt_bias;
  const void* conv_state;   // [pool, K-1, H, 3d] history, or nullptr for zeros
  int K;
  int gate_softplus;        // unbounded decay: the SIMT passes with exact diagonal gram blocks
  bool separate_passes;     // never the co-scheduled single launch
};

// One output range of the projection GEMM: columns [col_begin, col_end) of C = A B^T go
// to out[row * ld + (col - col_begin)] (bf16).
struct ProjOut {
  void* out;
  long long ld;
  int col_begin, col_end;
};
cudaError_t launch_proj_gemm(int M, int N, int K, const void* A, const void* B,
                             const ProjOut* outs, int n_outs, int* status, cudaStream_t st);
int proj_gemm_max_outs();

cudaError_t launch_prep(const PrepArgs& a, cudaStream_t st);
cudaError_t launch_step(const StepArgs& a, cudaStream_t st);
cudaError_t launch_rollback(const RollbackArgs& a, cudaStream_t st);
cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t st);

// Kernels this host thread has launched through the library (cumulative).
inline long long& launch_counter() {
  static thread_local long long n = 0;
  return n;
}

// Caller-owned events recorded on the prefill's stream after the intra-chunk,
// inter-chunk and output-norm passes (null entries are skipped); per host thread.
struct PhaseEvents {
  cudaEvent_t ev[3];
};
PhaseEvents& phase_events();
bool sm100_interchunk_supported(const PrefillArgs& a);
bool sm100_intra_supported(const PrefillArgs& a);
bool sm100_fused_supported(const PrefillArgs& a);
cudaError_t launch_conv_commit(const PrepArgs& a, cudaStream_t st);
cudaError_t launch_intra_sm100(const PrefillArgs& a, cudaStream_t st);
// both tensor-core passes in one cooperative launch; `launched` false = not applicable
cudaError_t launch_cosched_sm100(const PrefillArgs& a, cudaStream_t st, bool* launched);
// fused_norm: set when the pass also applied the gated RMSNorm and wrote y
cudaError_t launch_interchunk_sm100(const PrefillArgs& a, cudaStream_t st, bool* fused_norm);
cudaError_t launch_wait_timeout_selftest(void* workspace, cudaStream_t st);
int prep_tile();
int prep_kmax();

}  // namespace kda
