// Shared device helpers for the KDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// ---------------------------------------------------------------------------
// programmatic dependent launch (sm_90+): a kernel launched with the programmatic
// stream-serialization attribute may start before the kernel ahead of it on the
// stream has finished; grid_dep_wait() blocks until that kernel has completed and its
// memory is visible (at once when there is none).  grid_dep_trigger() lets the next
// such kernel be scheduled once every CTA of this grid has issued it or exited.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// launch `kernel` on `st` as a programmatic dependent of the previous kernel there
template <typename Args>
inline cudaError_t launch_dependent(void (*kernel)(Args), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t st, const Args& args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args);
}

// ---------------------------------------------------------------------------
// element I/O: activations are fp32 or bf16, arithmetic is fp32
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ld1(const float* p) { return *p; }
__device__ __forceinline__ float ld1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st1(float* p, float x) { *p = x; }
__device__ __forceinline__ void st1(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// two consecutive elements (8-byte / 4-byte aligned)
__device__ __forceinline__ float2 ld2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 ld2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ void st2(float* p, float a, float b) {
  *reinterpret_cast<float2*>(p) = make_float2(a, b);
}
__device__ __forceinline__ void st2(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}

// four consecutive elements (16-byte / 8-byte aligned)
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
  float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void st4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// logistic function; exp overflow to +inf gives exactly 0, never NaN
__device__ __forceinline__ float sigmoid(float x) { return 1.0f / (1.0f + expf(-x)); }

// log(1 + e^z) = max(z, 0) + log(1 + e^{-|z|}), without overflow
__device__ __forceinline__ float softplus(float z) { return fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))); }

// log decay of one key channel with A = exp(A_log[h]) and z = f + dt_bias: the bounded
// sigmoid lb * sigmoid(A z), or -A softplus(z) for the gate without a lower bound
__device__ __forceinline__ float gate_log_decay(float A, float z, float lb, int softplus_gate) {
  return softplus_gate ? -A * softplus(z) : lb * sigmoid(A * z);
}

// ---------------------------------------------------------------------------
// Packed sequences -> fixed-size tiles.
//
// Tile c of sequence s (rows [cu[s] + c*TILE, ...)) gets the slot
//     slot(s, c) = floor(cu[s] / TILE) + s + c.
// slot is strictly increasing over (s, c), so slots never collide, and every
// slot is below total/TILE + n_seqs + 1 (floor(a) + ceil(b) <= floor(a+b) + 1).
// A CTA per slot finds its sequence by binary search; slots in the gaps exit.
// All indices are clamped to [0, total] so a malformed cu_seqlens stays in bounds.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int num_slots(int total, int n_seqs, int tile) {
  return total / tile + n_seqs + 1;
}

__device__ __forceinline__ int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

struct TileRange {
  int seq;    // sequence index
  int start;  // first token row of the sequence
  int end;    // one past its last row
  int t0;     // first row of this tile
  int len;    // rows in this tile (0 = empty slot)
  int chunk;  // tile index within the sequence
};

__device__ __forceinline__ TileRange slot_to_tile(const int32_t* __restrict__ cu, int n_seqs,
                                                  int total, int tile, int slot) {
  int lo = 0, hi = n_seqs - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    int base = clampi(__ldg(cu + mid), 0, total) / tile + mid;
    if (base <= slot) lo = mid; else hi = mid - 1;
  }
  TileRange r;
  r.seq = lo;
  r.start = clampi(__ldg(cu + lo), 0, total);
  r.end = clampi(__ldg(cu + lo + 1), r.start, total);
  r.chunk = slot - (r.start / tile + lo);
  r.t0 = r.start + r.chunk * tile;
  r.len = (r.chunk < 0 || r.t0 >= r.end) ? 0 : min(tile, r.end - r.t0);
  return r;
}

__device__ __forceinline__ void seq_range(const int32_t* __restrict__ cu, int total, int s,
                                          int& start, int& end) {
  start = clampi(__ldg(cu + s), 0, total);
  end = clampi(__ldg(cu + s + 1), start, total);
}

// state row of sequence s in a pool; -1 = skip
__device__ __forceinline__ int pool_row(const int32_t* __restrict__ slots, int s, int pool_size) {
  int r = slots ? __ldg(slots + s) : s;
  return (r >= 0 && r < pool_size) ? r : -1;
}

}  // namespace kda
