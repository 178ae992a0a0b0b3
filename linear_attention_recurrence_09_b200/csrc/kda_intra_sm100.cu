// Intra-chunk pass of kda_prefill on the 5th-generation tensor cores (sm_100a).
// Used for d = 128, chunk 64, bf16 activations; writes the same per-slot
// workspace tiles as the SIMT intra_chunk_kernel (W, U~, Q~, K'^T, M, e^{G_C}).
//
// One CTA per (chunk slot, head).  With G the cumulative log decay of the chunk:
//   * Gram: A'[r,i] = sum_c k_r k_i e^{G_r - G_i} and M[r,i] = q_scale sum_c q_r k_i e^{G_r - G_i}.
//     The exponent is split at a reference row, row 15 for rows 0-31 and row 47
//     for rows 32-63: with the gate bounded below by -5, every factor is at most
//     e^80 (within fp32) and the products with i <= r are at most 1.  Both halves
//     run as ONE tf32 tcgen05 MMA, M = N = K = 128: A rows are the column-scaled
//     keys of both halves (32 + 64 rows), B rows the row-scaled keys and queries
//     (4 x 32 rows); only the two diagonal blocks of the product are read.  tf32
//     (not bf16) because the gram's rounding dominates the parity error budget.
//   * T = (I + A)^{-1} diag(b) by forward substitution in fp32 (4 threads per column).
//   * W^T = (K e^G)^T T^T and U~^T = V^T T^T as bf16 MMAs, M = 128 (key / value
//     channels), N = 64, K = 64 tokens, with K e^G and V read MN-major (stored
//     token-major by the threads that compute them).  T and K e^G are each split
//     into a bf16 high part and the bf16 rounding of the remainder (hi + lo), and
//     W accumulates hi.hi + hi.lo + lo.hi, U~ accumulates V.hi + V.lo: the
//     rounding of T and K e^G was the largest term left in the error budget.
// Q~ = q_scale Q e^G, K'^T = (K e^{G_C - G})^T and e^{G_C} are elementwise.
#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_sm100.cuh"

namespace kda {
namespace {

constexpr int D = 128, C = 64;
constexpr int THREADS = 256;
constexpr uint32_t TMEM_COLS = 128;
constexpr int KP_LD = 66;     // K'^T staging row stride (elements): odd word stride

// shared memory carve-up (offsets from a 1024-byte aligned base)
constexpr uint32_t OFF_GA = 0;          // gram A: tf32, 4 K-blocks x 128 rows x 128 B (64 KB)
constexpr uint32_t OFF_GB = 65536;      // gram B: same shape (64 KB)
constexpr uint32_t OFF_KT = 131072;     // K e^G, high bf16 part: MN-major [64 t][128 c] (16 KB)
constexpr uint32_t OFF_KL = 147456;     // K e^G, low bf16 part (the rounding remainder)
constexpr uint32_t OFF_VT = 163840;     // V:     bf16 MN-major [64 t][128 c] (16 KB)
constexpr uint32_t OFF_G = 180224;      // G fp32 [64][128] (32 KB); later A fp32 [64][65]
constexpr uint32_t OFF_KP = 212992;     // K'^T staging bf16 [128][KP_LD]
constexpr uint32_t OFF_T = OFF_GA;      // T high part, bf16 K-major [64 r][64 i] (8 KB), after the gram
constexpr uint32_t OFF_TL = OFF_GA + 8192;  // T low part
constexpr uint32_t SMEM_BYTES = OFF_KP + 128 * KP_LD * 2 + 1024;

__device__ __forceinline__ uint32_t gram_off(int n, int c) {   // tf32 K-major, K = 128
  return (uint32_t)((c >> 5) * 16384) + sw128_off32(n, c & 31);
}
__device__ __forceinline__ uint32_t mn_off(int t, int c) {     // bf16 MN-major [t][c]
  const int row = t & 7;
  return (uint32_t)((c >> 6) * 8192 + (t >> 3) * 1024 + row * 128 +
                    (((((c & 63) >> 3) ^ row) & 7) << 4) + (c & 7) * 2);
}

__device__ __forceinline__ void st_tf32x4(unsigned char* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}
__device__ __forceinline__ void st_bf16x4(unsigned char* p, float a, float b, float c, float d) {
  st4(reinterpret_cast<__nv_bfloat16*>(p), make_float4(a, b, c, d));
}

__global__ void __launch_bounds__(THREADS, 1) intra_chunk_sm100_kernel(const PrefillArgs a) {
  extern __shared__ __align__(1024) unsigned char smraw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sb = smem_u32(sm);
  __shared__ float bs[C];
  __shared__ uint32_t tmem_holder;
  __shared__ __align__(8) uint64_t bar_mma;
  __shared__ volatile int abort_flag;

  const int h = blockIdx.y, H = a.H, slot = blockIdx.x;
  const TileRange tr = slot_to_tile(a.cu, a.n_seqs, a.total, C, slot);
  if (tr.len == 0) return;
  if (pool_row(a.slots, tr.seq, a.pool_size) < 0) return;
  const int L = tr.len, t0 = tr.t0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t tile = (size_t)slot * H + h;
  __nv_bfloat16* Wo = reinterpret_cast<__nv_bfloat16*>(a.ws + a.L.W) + tile * C * D;
  __nv_bfloat16* Uo = reinterpret_cast<__nv_bfloat16*>(a.ws + a.L.Ut) + tile * C * D;
  __nv_bfloat16* Qo = reinterpret_cast<__nv_bfloat16*>(a.ws + a.L.Qt) + tile * C * D;
  __nv_bfloat16* KTo = reinterpret_cast<__nv_bfloat16*>(a.ws + a.L.Kp) + tile * D * C;
  __nv_bfloat16* Mo = reinterpret_cast<__nv_bfloat16*>(a.ws + a.L.M) + tile * C * C;
  float* gCo = reinterpret_cast<float*>(a.ws + a.L.gC) + tile * D;
  int* status = reinterpret_cast<int*>(a.ws + a.L.status);
  float* G = reinterpret_cast<float*>(sm + OFF_G);
  float* Af = G;                                  // [64][65], after the gram
  __nv_bfloat16* KP = reinterpret_cast<__nv_bfloat16*>(sm + OFF_KP);

  // ---- log decay -> G (rows past the sequence end add 0), beta ----
  {
    float4 lv[8];   // 8 float4 per thread, all in flight before the first store
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int e4 = tid + m * THREADS;         // float4 index in the [64][128] tile
      const int r = e4 >> 5, c4 = (e4 & 31) * 4;
      lv[m] = (r < L) ? ld4(a.loga + ((size_t)(t0 + r) * H + h) * D + c4)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) reinterpret_cast<float4*>(G)[tid + m * THREADS] = lv[m];
  }
  if (tid < C) bs[tid] = (tid < L) ? __ldg(a.beta + (size_t)(t0 + tid) * H + h) : 0.f;
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_mma), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  if (tid < D) {
    float acc = 0.f;
    for (int r = 0; r < C; ++r) {
      acc += G[r * D + tid];
      G[r * D + tid] = acc;
    }
    gCo[tid] = __expf(acc);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  // ---- elementwise operands: 4 consecutive channels of one token row per item ----
  const float qsc = a.q_scale;
  constexpr int BATCH = 4;   // items whose loads are in flight together
#pragma unroll 1
  for (int b0 = 0; b0 < (C * (D / 4)) / THREADS; b0 += BATCH) {
  float4 qa[BATCH], ka[BATCH], va[BATCH];
#pragma unroll
  for (int u = 0; u < BATCH; ++u) {
    const int it = tid + (b0 + u) * THREADS;
    const int r = it >> 5, c4 = (it & 31) * 4;
    qa[u] = ka[u] = va[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < L) {
      const size_t idx = ((size_t)(t0 + r) * H + h) * D + c4;
      qa[u] = ld4(a.q + idx);
      ka[u] = ld4(a.k + idx);
      va[u] = ld4(a.v + idx);
    }
  }
#pragma unroll
  for (int u = 0; u < BATCH; ++u) {
    const int it = tid + (b0 + u) * THREADS;
    const int r = it >> 5, c4 = (it & 31) * 4;
    const float4 q4 = qa[u], k4 = ka[u], v4 = va[u];
    const float qv[4] = {q4.x, q4.y, q4.z, q4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
    float kb[4], qb[4], kc0[4], kc1[4], qt[4], kt[4], kp[4];
    const int rref = (r < 32) ? 15 : 47;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c4 + j;
      const float g = G[r * D + c];
      const float er = __expf(g - G[rref * D + c]);
      kb[j] = kv[j] * er;
      qb[j] = qsc * qv[j] * er;
      kc0[j] = (r < 32) ? kv[j] * __expf(G[15 * D + c] - g) : 0.f;
      kc1[j] = kv[j] * __expf(G[47 * D + c] - g);
      const float eg = __expf(g);
      qt[j] = qsc * qv[j] * eg;
      kt[j] = kv[j] * eg;
      kp[j] = kv[j] * __expf(G[63 * D + c] - g);
    }
    const int nk = (r < 32) ? r : 64 + (r - 32);
    st_tf32x4(sm + OFF_GB + gram_off(nk, c4), kb[0], kb[1], kb[2], kb[3]);
    st_tf32x4(sm + OFF_GB + gram_off(nk + 32, c4), qb[0], qb[1], qb[2], qb[3]);
    if (r < 32) st_tf32x4(sm + OFF_GA + gram_off(r, c4), kc0[0], kc0[1], kc0[2], kc0[3]);
    st_tf32x4(sm + OFF_GA + gram_off(32 + r, c4), kc1[0], kc1[1], kc1[2], kc1[3]);
    {
      float hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        hi[j] = __bfloat162float(__float2bfloat16_rn(kt[j]));
        lo[j] = kt[j] - hi[j];
      }
      st_bf16x4(sm + OFF_KT + mn_off(r, c4), hi[0], hi[1], hi[2], hi[3]);
      st_bf16x4(sm + OFF_KL + mn_off(r, c4), lo[0], lo[1], lo[2], lo[3]);
    }
    st_bf16x4(sm + OFF_VT + mn_off(r, c4), v4.x, v4.y, v4.z, v4.w);
    st4(Qo + (size_t)r * D + c4, make_float4(qt[0], qt[1], qt[2], qt[3]));
#pragma unroll
    for (int j = 0; j < 4; ++j) KP[(c4 + j) * KP_LD + r] = __float2bfloat16_rn(kp[j]);
  }
  }
  fence_proxy_async();
  __syncthreads();

  // ---- gram MMA (tf32, 128 x 128 x 128) ----
  int issued = 0;   // MMA batches committed by thread 0
  if (tid == 0) {
    tc_fence_after();
    const uint32_t id = idesc_tf32(128, 128);
#pragma unroll
    for (int s = 0; s < 16; ++s)
      umma_tf32(tmem, sw128_desc(sb + OFF_GA + (s >> 2) * 16384 + (s & 3) * 32),
                sw128_desc(sb + OFF_GB + (s >> 2) * 16384 + (s & 3) * 32), id, s > 0);
    umma_commit(smem_u32(&bar_mma));
    issued = 1;
  }
  bool ok = mbar_wait_warp(smem_u32(&bar_mma), 0, &abort_flag);
  tc_fence_after();
  for (int e = tid; e < C * (C + 1); e += THREADS) Af[e] = 0.f;   // G is dead now
  __syncthreads();
  // D[m][n]: rows 0-31 = keys 0-31 vs cols 0-31 (keys) / 32-63 (queries) of rows 0-31;
  // rows 32-95 = keys 0-63 vs cols 64-95 (keys) / 96-127 (queries) of rows 32-63
  if (ok && (warp == 0 || warp == 5 || warp == 6)) {
    const int q = warp & 3;
    const int i = (warp == 0) ? lane : (warp == 5 ? lane : 32 + lane);
    const int rbase = (warp == 0) ? 0 : 32;
    const uint32_t col = (warp == 0) ? 0u : 64u;
    float av[32], mv[32];
    tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + col, av);
    tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + col + 32, mv);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int r = rbase + j;
      if (i < r) Af[r * (C + 1) + i] = bs[r] * av[j];
      Mo[r * C + i] = __float2bfloat16_rn(i <= r ? mv[j] : 0.f);
    }
  } else if (warp == 7) {
#pragma unroll
    for (int j = 0; j < 32; ++j) Mo[j * C + 32 + lane] = __float2bfloat16_rn(0.f);
  }
  tc_fence_before();
  __syncthreads();

  // ---- T = (I + A)^{-1} diag(b): column j, rows r = 4m + t owned by lane t ----
  {
    const int j = tid >> 2, t = tid & 3;
    float x[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) x[m] = 0.f;
#pragma unroll
    for (int r = 0; r < C; ++r) {
      float p = 0.f;
#pragma unroll
      for (int m = 0; m < 16; ++m)
        if (4 * m + t < r) p = fmaf(Af[r * (C + 1) + 4 * m + t], x[m], p);
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      p += __shfl_xor_sync(0xffffffffu, p, 2);
      if ((r & 3) == t) x[r >> 2] = ((r == j) ? 1.f : 0.f) - p;
    }
    const float bj = bs[j];
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int r = 4 * m + t;
      const float tv = x[m] * bj;
      const __nv_bfloat16 hi = __float2bfloat16_rn(tv);
      *reinterpret_cast<__nv_bfloat16*>(sm + OFF_T + sw128_off(r, j)) = hi;
      *reinterpret_cast<__nv_bfloat16*>(sm + OFF_TL + sw128_off(r, j)) =
          __float2bfloat16_rn(tv - __bfloat162float(hi));
    }
  }
  fence_proxy_async();
  __syncthreads();

  // ---- W^T = K~^T T^T (cols 0-63), U~^T = V^T T^T (cols 64-127) ----
  if (tid == 0 && ok) {
    tc_fence_after();
    const uint32_t id = idesc_bf16_amn(128, 64);
    // W^T: Khi.Thi + Khi.Tlo + Klo.Thi
#pragma unroll
    for (int s = 0; s < 4; ++s)
      umma(tmem, sw128_mn_desc(sb + OFF_KT + s * 2048, 8192),
           sw128_desc(sb + OFF_T + s * 32), id, s > 0);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      umma(tmem, sw128_mn_desc(sb + OFF_KT + s * 2048, 8192),
           sw128_desc(sb + OFF_TL + s * 32), id, 1);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      umma(tmem, sw128_mn_desc(sb + OFF_KL + s * 2048, 8192),
           sw128_desc(sb + OFF_T + s * 32), id, 1);
    // U~^T: V.Thi + V.Tlo
#pragma unroll
    for (int s = 0; s < 4; ++s)
      umma(tmem + 64, sw128_mn_desc(sb + OFF_VT + s * 2048, 8192),
           sw128_desc(sb + OFF_T + s * 32), id, s > 0);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      umma(tmem + 64, sw128_mn_desc(sb + OFF_VT + s * 2048, 8192),
           sw128_desc(sb + OFF_TL + s * 32), id, 1);
    umma_commit(smem_u32(&bar_mma));
    issued = 2;
  }
  // K'^T out while the MMAs run (rows of 64 tokens, 16-byte stores)
  for (int e = tid; e < D * (C / 8); e += THREADS) {
    const int c = e >> 3, part = (e & 7) * 8;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(KP + c * KP_LD + part);
    uint4 v;
    v.x = src[0]; v.y = src[1]; v.z = src[2]; v.w = src[3];
    *reinterpret_cast<uint4*>(KTo + (size_t)c * C + part) = v;
  }
  if (ok) ok = mbar_wait_warp(smem_u32(&bar_mma), 1, &abort_flag);
  tc_fence_after();
  if (ok) {
    const int q = warp & 3;
    const int c = 32 * q + lane;
    __nv_bfloat16* dst = (warp < 4) ? Wo : Uo;
    const uint32_t col = (warp < 4) ? 0u : 64u;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float v[32];
      tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + col + 32 * half, v);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        dst[(size_t)(32 * half + j) * D + c] = __float2bfloat16_rn(v[j]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_flag && tid == 0) {
    // let the last issued MMA batch retire before TMEM is released (bounded), then report
    if (issued > 0) {
      const long long t1 = clock64();
      while (!mbar_try(smem_u32(&bar_mma), (uint32_t)(issued - 1)) &&
             clock64() - t1 < WAIT_LIMIT_CYCLES) {
      }
    }
    atomicExch(status, 5 /* KDA_ERR_TIMEOUT */);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

}  // namespace

bool sm100_intra_supported(const PrefillArgs& a) { return a.bf16 && a.D == D && a.C == C; }

cudaError_t launch_intra_sm100(const PrefillArgs& a, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(intra_chunk_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  intra_chunk_sm100_kernel<<<dim3(a.L.nslots, a.H), THREADS, SMEM_BYTES, st>>>(a);
  return cudaGetLastError();
}

}  // namespace kda
