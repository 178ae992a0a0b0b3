// kda_prefill_noalloc: kda_prefill with its scratch in a fixed device array, for
// callers that cannot allocate device memory.
//
// The scratch is one file-scope __device__ array of KDA_NOALLOC_SCRATCH_BYTES.
// Host code may not pass the array's name to a kernel (on the host it is only a
// stand-in symbol, not a device address), so every call looks up the real address
// with cudaGetSymbolAddress while the caller's device is current.  The lookup is
// not cached: after a cudaDeviceReset the module is loaded again and the array may
// sit at another address, which a cached pointer would not follow.  The first call
// on a device also loads the module there (a set-up step that should not happen
// inside a stream capture).
#include "../../include/kda.h"
#include "kda_launch.h"

namespace {

constexpr size_t kScratchBytes = (size_t)KDA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch on the current device.
int scratch_on_current_device(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return KDA_ERR_CUDA;
  *out = p;
  return KDA_OK;
}

}  // namespace

extern "C" {

int kda_prefill_noalloc(const kda_config* cfg, int32_t n_seqs, int32_t total_tokens,
                        const int32_t* cu_seqlens, const void* q, const void* k, const void* v,
                        const float* log_a, const float* beta, const void* g,
                        const float* norm_w, const float* state_in, float* state_out,
                        const int32_t* state_slots, int32_t pool_size, void* y,
                        kda_stream_t stream) {
  const size_t need = kda_prefill_workspace_size(cfg, n_seqs, total_tokens);
  if (need == 0 || n_seqs == 0) {
    // invalid configuration or nothing to do: kda_prefill reports which, launches nothing
    return kda_prefill(cfg, n_seqs, total_tokens, cu_seqlens, q, k, v, log_a, beta, g, norm_w,
                       state_in, state_out, state_slots, pool_size, y, nullptr, 0, stream);
  }
  if (need > kScratchBytes) return KDA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const int st = scratch_on_current_device(&scratch);
  if (st != KDA_OK) return st;
  // kda_prefill clears the status word itself and overwrites every other byte it
  // reads, so the previous call's contents need no clearing here.
  return kda_prefill(cfg, n_seqs, total_tokens, cu_seqlens, q, k, v, log_a, beta, g, norm_w,
                     state_in, state_out, state_slots, pool_size, y, scratch, kScratchBytes,
                     stream);
}

}  // extern "C"
