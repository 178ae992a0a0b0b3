// kda_proj_gemm: the layer's projections as one bf16 GEMM on the 5th-generation tensor
// cores (sm_100a): C = A B^T with A [M, K] (activations, one row per token) and B [N, K]
// (a weight matrix stored output-row-major), fp32 accumulation in TMEM, bf16 results.
//
// glm53-flash-mlx README, quantization recipe: the runtime fuses the six KDA input
// projections into one matmul; llama.cpp PR #27754, KDA commit: the output gate is low
// rank, g_b(g_a(x)).  One launch computes the fused product and its epilogue routes
// column ranges of C to separate tensors (q|k|v, f, beta logit, g_a), so the layer's
// inputs land in their own dense layouts without a copy; the same kernel with K = the
// gate rank computes g_b.
//
// Persistent: one CTA per SM walks 128 x 256 output tiles (M fastest, so a band of B
// rows stays in L2 while the CTAs sweep A).  Warp 0 issues TMA loads of 64-wide K slices
// (A 16 KB + B 32 KB per stage, 128-byte swizzle) into a 4-stage ring; warp 1 allocates
// all 512 TMEM columns and issues the MMAs from one thread (M = 128, N = 256, K = 16 per
// instruction, four per stage); the accumulator is double-buffered in TMEM (2 x 256
// columns), so warps 2-5 read tile i out of TMEM (one row per thread, TMEM lane quarter =
// warp % 4), convert to bf16 and store while the MMAs of tile i + 1 run.
// Every wait is bounded; on expiry the CTA records KDA_ERR_TIMEOUT in the caller's status
// word (when given), lets what it issued retire, frees TMEM and exits.
#include <cuda.h>

#include "../../include/kda.h"
#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_sm100.cuh"

namespace kda {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int STAGES = 4;
constexpr uint32_t A_STAGE = BM * BK * 2;          // 16 KB
constexpr uint32_t B_STAGE = BN * BK * 2;          // 32 KB
constexpr uint32_t STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;                // two 256-column fp32 accumulators
constexpr uint32_t OFF_BAR = STAGES * STAGE_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;   // + barriers, + alignment slack
constexpr int MAX_OUTS = 4;

enum { BAR_FULL = 0, BAR_EMPTY = BAR_FULL + STAGES, BAR_TFULL = BAR_EMPTY + STAGES,
       BAR_TEMPTY = BAR_TFULL + 2, BAR_COUNT = BAR_TEMPTY + 2 };
static_assert(BAR_COUNT * 8 <= 256, "barrier slots");

struct GemmOut {
  __nv_bfloat16* out;
  long long ld;        // elements between rows
  int c0, c1;          // output columns [c0, c1) of C
};

struct GemmArgs {
  int M, N, K;
  int n_outs;
  GemmOut outs[MAX_OUTS];
  int* status;
};

struct GemmMaps {
  CUtensorMap A, B;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int NOUT_DUMMY = 0>
__global__ void __launch_bounds__(THREADS, 1)
proj_gemm_kernel(const GemmArgs g, const __grid_constant__ GemmMaps maps) {
  extern __shared__ __align__(1024) unsigned char smraw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  __shared__ uint32_t tmem_holder;
  __shared__ volatile int abort_flag;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (g.M + BM - 1) / BM, num_n = (g.N + BN - 1) / BN;
  const int ntiles = num_m * num_n;
  const int nk = (g.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(BAR_FULL + s), 1);
      mbar_init(bar(BAR_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(BAR_TFULL + b), 1);
      mbar_init(bar(BAR_TEMPTY + b), 32 * EPI_WARPS);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_holder)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int it = 0, issued = 0;
      for (int t = blockIdx.x; t < ntiles && !abort_flag; t += gridDim.x) {
        const int m0 = (t % num_m) * BM, n0 = (t / num_m) * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          if (it >= STAGES && !mbar_wait(bar(BAR_EMPTY + s), ((it / STAGES) - 1) & 1, &abort_flag))
            break;
          const uint32_t sa = sbase + s * STAGE_BYTES, sb = sa + A_STAGE;
          mbar_expect_tx(bar(BAR_FULL + s), STAGE_BYTES);
          tma_load_2d(sa, &maps.A, kb * BK, m0, bar(BAR_FULL + s));
          tma_load_2d(sb, &maps.B, kb * BK, n0, bar(BAR_FULL + s));
          tma_load_2d(sb + B_STAGE / 2, &maps.B, kb * BK, n0 + BN / 2, bar(BAR_FULL + s));
          issued = it + 1;
        }
      }
      if (abort_flag) {   // let the copies in flight land before the CTA exits
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
          const long long t0 = clock64();
          while (!mbar_try(bar(BAR_FULL + i % STAGES), (i / STAGES) & 1) &&
                 clock64() - t0 < WAIT_LIMIT_CYCLES) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(BM, BN);
      int it = 0, local = 0;
      bool committed = false;
      for (int t = blockIdx.x; t < ntiles && !abort_flag; t += gridDim.x, ++local) {
        const int buf = local & 1;
        // the epilogue has read this accumulator out (tile local - 2)
        if (local >= 2 && !mbar_wait(bar(BAR_TEMPTY + buf), ((local >> 1) - 1) & 1, &abort_flag))
          break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * BN);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(bar(BAR_FULL + s), (it / STAGES) & 1, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = sw128_desc(sbase + s * STAGE_BYTES);
          const uint64_t db = sw128_desc(sbase + s * STAGE_BYTES + A_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)   // 16 bf16 = 32 bytes along K per instruction
            umma(d, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), idesc, (kb | k) ? 1u : 0u);
          umma_commit(bar(BAR_EMPTY + s));
          committed = true;
        }
        if (!ok) break;
        umma_commit(bar(BAR_TFULL + buf));
      }
      if (abort_flag && committed) {   // let the issued MMAs retire before TMEM is freed
        const int s = (it + STAGES - 1) % STAGES;
        const long long t0 = clock64();
        while (!mbar_try(bar(BAR_EMPTY + s), ((it - 1) / STAGES) & 1) &&
               clock64() - t0 < WAIT_LIMIT_CYCLES) {
        }
      }
    }
  } else {
    // ---------------- epilogue warps 2..5 ----------------
    const int q = warp & 3;                         // TMEM lane quarter
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    int local = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
      const int buf = local & 1;
      const int m0 = (t % num_m) * BM, n0 = (t / num_m) * BN;
      if (!mbar_wait_warp(bar(BAR_TFULL + buf), (local >> 1) & 1, &abort_flag)) break;
      tc_fence_after();
      const int row = m0 + 32 * q + lane;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld32(tmem + lane_off + (uint32_t)(buf * BN + c), v);
        if (row < g.M) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            const int col = n0 + c + e;             // 8 columns: one 16-byte store
            if (col >= g.N) break;
#pragma unroll
            for (int o = 0; o < MAX_OUTS; ++o) {
              const GemmOut& go = g.outs[o];
              if (o < g.n_outs && col >= go.c0 && col < go.c1) {
                *reinterpret_cast<uint4*>(go.out + (size_t)row * go.ld + (col - go.c0)) =
                    make_uint4(pack_bf16x2(v[e], v[e + 1]), pack_bf16x2(v[e + 2], v[e + 3]),
                               pack_bf16x2(v[e + 4], v[e + 5]), pack_bf16x2(v[e + 6], v[e + 7]));
                break;
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(BAR_TEMPTY + buf));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_flag && threadIdx.x == 0 && g.status != nullptr)
    atomicExch(g.status, (int)KDA_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn gemm_encode_fn() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<EncodeTiledFn>(fn);
}

// [rows, K] bf16, K contiguous; box [box_rows, 64]; 128-byte swizzle; zero fill past the
// edges (a partial M or N tile and a K tail read zeros)
bool make_kmajor_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, uint64_t rows,
                     uint64_t K, uint32_t box_rows) {
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K * 2};
  const cuuint32_t box[2] = {BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int proj_gemm_max_outs() { return MAX_OUTS; }

cudaError_t launch_proj_gemm(int M, int N, int K, const void* A, const void* B,
                             const ProjOut* outs, int n_outs, int* status, cudaStream_t st) {
  if (n_outs < 1 || n_outs > MAX_OUTS) return cudaErrorInvalidValue;
  EncodeTiledFn enc = gemm_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  GemmMaps maps;
  if (!make_kmajor_map(enc, &maps.A, A, (uint64_t)M, (uint64_t)K, BM) ||
      !make_kmajor_map(enc, &maps.B, B, (uint64_t)N, (uint64_t)K, BN / 2))
    return cudaErrorInvalidValue;
  GemmArgs g{};
  g.M = M; g.N = N; g.K = K; g.n_outs = n_outs; g.status = status;
  for (int i = 0; i < n_outs; ++i) {
    g.outs[i].out = static_cast<__nv_bfloat16*>(outs[i].out);
    g.outs[i].ld = outs[i].ld;
    g.outs[i].c0 = outs[i].col_begin;
    g.outs[i].c1 = outs[i].col_end;
  }
  cudaError_t e = cudaFuncSetAttribute(proj_gemm_kernel<0>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const long long ntiles = (long long)((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const unsigned grid = (unsigned)(ntiles < nsm ? ntiles : nsm);
  if (grid == 0) return cudaSuccess;
  proj_gemm_kernel<0><<<grid, THREADS, SMEM_BYTES, st>>>(g, maps);
  ++launch_counter();
  return cudaGetLastError();
}

}  // namespace kda
