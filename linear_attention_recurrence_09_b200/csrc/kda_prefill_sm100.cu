// Inter-chunk pass of kda_prefill on the 5th-generation tensor cores (sm_100a):
// bf16 tcgen05 MMAs fed by TMA, fp32 accumulators in TMEM, the fp32 state carried
// on chip through the chunks of a sequence.  Used for d = 128, chunk 64, bf16.
//
// One CTA per (32-column value slice, head, sequence): the columns of the state
// evolve independently (each obeys the recurrence with the same k, a, b), so a
// head's 128 value columns are split over 4 CTAs and the serial chain of a
// sequence runs on 4 SMs at once.  Per chunk (C = 64 tokens), with S the bf16
// copy of the state slice (128 x 32):
//   MMA1   D1[128 x 32]  = [W ; Q~] (128 x 128) . S          -> rows 0-63: W S, rows 64-127: Q~ S
//   E1     U = U~ - W S  (fp32, rows past the sequence end forced to 0) -> bf16 U^T in smem
//   MMA2   D2[128 x 32]  = K'^T (128 x 64) . U               (state increment, key rows;
//                                                               K' stored token-major, read MN-major)
//   MMA3   D1[64:128]   += M (64 x 64) . U                   (O = Q~ S + M U; A = [X ; M],
//                                                               X the 8 KB before M: its rows
//                                                               land in D1[0:64], already read)
//   E2     S <- Diag(e^{G_C}) S + D2 in fp32 registers (one key row per thread) -> bf16 S^T
//   E3     O rows of D1 -> y = O / rms(O) * w * sigmoid(g) (FUSE_NORM), else o (fp32,
//          workspace) for the separate gated RMSNorm pass
// With FUSE_NORM the 4 slice CTAs of a head form a thread-block cluster and two extra
// warps per CTA run E3 off the chain: every token's sum of squares over its 128 value
// columns is assembled from the 4 slices' partials, which each CTA sends into every
// peer's shared memory with asynchronous remote stores that complete on the peer's
// mbarrier (a 2-slot ring indexed by chunk parity).
// Warp roles: warp 0 issues TMA (three smem stages, so chunks n+1 and n+2 load while n
// computes: one chunk's tiles take longer than a chunk period to arrive; the U~ slice
// comes with them), warp 1 allocates TMEM and issues the MMAs from one thread, warps
// 2-9 run the epilogues, two warps per TMEM lane quarter (quarter = warp % 4), each
// owning 16 of the 32 value columns.  E1 and E2 are on the serial chain.  With the fused
// norm, MMA3 of chunk n is issued after MMA1 of chunk n+1, off the chain (U is
// double-buffered for it); without it, MMA3 follows MMA2 and the epilogue warps of lane
// quarters 2-3 read O (E3) once it has retired.  Every MMA operand uses the
// 128-byte swizzle: TMA writes the workspace tiles (K-major; K' read MN-major) and the
// epilogue threads write S and U MN-major, 16 bytes at a time.
//
// Every wait is bounded (about a second): on expiry the CTA records
// KDA_ERR_TIMEOUT in the workspace status word, drains what it issued, frees
// its TMEM and exits; the host reads the word with kda_workspace_status.
#include <cuda.h>

#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_sm100.cuh"

namespace kda {
namespace {

constexpr int D = 128, C = 64, J = 32, NSLICE = D / J;
constexpr int NEPI = 8;                          // epilogue warps (2 per TMEM lane quarter)
constexpr int THREADS = 64 + 32 * NEPI;          // TMA, MMA and epilogue warps
constexpr int NOUT = 2;                          // fused norm: O warps (TMEM lanes 64-127)
template <bool FUSE_NORM>
constexpr int threads_of() { return THREADS + (FUSE_NORM ? 32 * NOUT : 0); }
constexpr int JH = J / 2;                        // value columns per epilogue thread
constexpr uint32_t TMEM_COLS = 128;

// shared memory carve-up (offsets from a 1024-byte aligned base)
constexpr uint32_t A1_BYTES = 2 * 128 * 128;     // [W;Q~]: 2 K-blocks x 128 rows x 128 B
constexpr uint32_t A2_BYTES = 128 * 128;         // K'   : 64 tokens x 128 key channels, read MN-major
constexpr uint32_t M_BYTES = 64 * 128;           // M: 64 rows x 64 (the lower half of A3)
constexpr uint32_t UT_BYTES = C * J * 2;         // U~ slice: 64 rows x 32 cols bf16, row-major
constexpr uint32_t STAGE_BYTES = A1_BYTES + A2_BYTES + M_BYTES + UT_BYTES;
constexpr uint32_t NSTAGE = 3;
constexpr uint32_t TX_BYTES = 4 * 8192 + 2 * 8192 + 8192 + UT_BYTES;   // W x2, Q~ x2, K' x2, M, U~
// S (128 key rows) and U (64 token rows) as MN-major B operands: one 128-byte swizzled
// row per key / token with the slice's 32 value columns in its first 64 bytes (the MMAs
// have N = 32 and never read the rest), so a thread writes its 16 columns as 2 x 16 bytes
constexpr uint32_t OFF_S = NSTAGE * STAGE_BYTES;          // S: 128 rows x 128 B
constexpr uint32_t OFF_U = OFF_S + 128 * 128;             // U:  2 buffers of 64 rows x 128 B
constexpr uint32_t U_BYTES = 64 * 128;
constexpr uint32_t OFF_BAR = OFF_U + 2 * U_BYTES;
constexpr uint32_t OFF_SSQ = OFF_BAR + 256;   // fused norm: [2 parities][4 slices][64 tokens] fp32
constexpr uint32_t SMEM_BYTES = OFF_SSQ + 2 * NSLICE * C * 4 + 1024;   // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");

// barrier slots (8 bytes each)
enum { BAR_FULL0 = 0, BAR_FULL1, BAR_FULL2, BAR_EMPTY0, BAR_EMPTY1, BAR_EMPTY2, BAR_MMA1,
       BAR_MMA2, BAR_SREADY,
       BAR_UREADY, BAR_NFULL0, BAR_NFULL1, BAR_OFREE0, BAR_OFREE1, BAR_OFREE2, BAR_ODONE0,
       BAR_ODONE1, BAR_ODONE2, BAR_COUNT };
static_assert(BAR_COUNT * 8 <= 256, "barrier slots");
// norm partial exchange: every token's partial from every slice CTA, 4 bytes each
constexpr uint32_t NORM_TX_BYTES = NSLICE * C * 4;

struct TmaMaps {
  CUtensorMap W, Q, KT, M, Ut;
};

// sigmoid(z) = (1 + tanh(z / 2)) / 2 with one special-function op (tanh.approx, absolute
// error about 2^-11): the outputs are bf16 and the output gate's error stays far inside
// the parity budget; the two inter-chunk kernels share the form, so their outputs agree
__device__ __forceinline__ float fast_sigmoid(float z) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
  return fmaf(0.5f, t, 0.5f);
}

// byte offset of element (row k, column n < 64) of an MN-major, 128B-swizzled bf16 tile
// (rows of 128 bytes, 8-row groups of 1024 bytes, 16-byte chunks XOR-ed with k mod 8)
__device__ __forceinline__ uint32_t mn_row_chunk(int k, int chunk) {
  return (uint32_t)((k >> 3) * 1024 + (k & 7) * 128 + (((chunk ^ k) & 7) << 4));
}
// eight fp32 values -> eight bf16 in one 16-byte chunk
__device__ __forceinline__ uint4 pack8_bf16(const float* v) {
  uint4 r;
  __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
  for (int e = 0; e < 4; ++e) p[e] = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
  return r;
}

// K-major SW128 descriptor advanced by `bytes` (the 14-bit address field never carries)
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

template <bool FUSE_NORM>
__global__ void __launch_bounds__(threads_of<FUSE_NORM>(), 1)
interchunk_sm100_kernel(const PrefillArgs a, const __grid_constant__ TmaMaps maps) {
  extern __shared__ __align__(1024) unsigned char smraw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  __shared__ uint32_t tmem_holder;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * J, h = blockIdx.y, s = blockIdx.z, H = a.H;
  const int row = pool_row(a.slots, s, a.pool_size);
  if (row < 0) return;
  int start, end;
  seq_range(a.cu, a.total, s, start, end);
  const int nch = (end - start + C - 1) / C;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int st = 0; st < (int)NSTAGE; ++st) {
      mbar_init(bar(BAR_FULL0 + st), 1);
      mbar_init(bar(BAR_EMPTY0 + st), 1);
    }
    mbar_init(bar(BAR_MMA1), 1);
    mbar_init(bar(BAR_MMA2), 1);
    mbar_init(bar(BAR_SREADY), 32 * NEPI);
    mbar_init(bar(BAR_UREADY), 32 * NEPI / 2);
    mbar_init(bar(BAR_NFULL0), 1);   // armed by one O thread per phase, filled by st.async
    mbar_init(bar(BAR_NFULL1), 1);
    mbar_init(bar(BAR_OFREE0), NOUT);
    mbar_init(bar(BAR_OFREE1), NOUT);
    mbar_init(bar(BAR_OFREE2), NOUT);
    mbar_init(bar(BAR_ODONE0), 1);
    mbar_init(bar(BAR_ODONE1), 1);
    mbar_init(bar(BAR_ODONE2), 1);
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
  if (FUSE_NORM) cluster_sync_all();   // every peer's barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem = tmem_holder;
  // [W S ; O] of chunk n in D1 buffer n % 3 (three, so the O readers have slack); K'^T U in D2
  auto d1_of = [&](int n) -> uint32_t {
    const int b = n % 3;
    return tmem + (b == 2 ? 96u : 32u * (uint32_t)b);
  };
  const uint32_t d2_tmem = tmem + 64;
  int* status = reinterpret_cast<int*>(a.ws + a.L.status);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = 0;
      for (int n = 0; n < nch && !abort_flag; ++n) {
        const int st = n % NSTAGE;
        if (n >= (int)NSTAGE &&
            !mbar_wait(bar(BAR_EMPTY0 + st), ((n / NSTAGE) - 1) & 1, &abort_flag))
          break;
        const int tile = (start / C + s + n) * H + h;
        const uint32_t A1 = sbase + st * STAGE_BYTES, A2 = A1 + A1_BYTES, Ms = A2 + A2_BYTES;
        const uint32_t UTs = Ms + M_BYTES;
        mbar_expect_tx(bar(BAR_FULL0 + st), TX_BYTES);
        tma_load_2d(A1, &maps.W, 0, tile * C, bar(BAR_FULL0 + st));
        tma_load_2d(A1 + 16384, &maps.W, 64, tile * C, bar(BAR_FULL0 + st));
        tma_load_2d(A1 + 8192, &maps.Q, 0, tile * C, bar(BAR_FULL0 + st));
        tma_load_2d(A1 + 16384 + 8192, &maps.Q, 64, tile * C, bar(BAR_FULL0 + st));
        tma_load_2d(A2, &maps.KT, 0, tile * C, bar(BAR_FULL0 + st));
        tma_load_2d(A2 + 8192, &maps.KT, 64, tile * C, bar(BAR_FULL0 + st));
        tma_load_2d(Ms, &maps.M, 0, tile * C, bar(BAR_FULL0 + st));
        tma_load_2d(UTs, &maps.Ut, j0, tile * C, bar(BAR_FULL0 + st));
        issued = n + 1;
      }
      if (abort_flag) {  // let the copies this thread started land before the CTA exits
        for (int n = (issued >= (int)NSTAGE ? issued - (int)NSTAGE : 0); n < issued; ++n) {
          const long long t0 = clock64();
          while (!mbar_try(bar(BAR_FULL0 + n % NSTAGE), (n / NSTAGE) & 1) &&
                 clock64() - t0 < WAIT_LIMIT_CYCLES) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t id = idesc_bf16(128, J) | (1u << 16);      // B (S or U) MN-major
      const uint32_t id_amn = id | (1u << 15);                   // K' is read MN-major too
      const uint32_t sS = sbase + OFF_S, sU0 = sbase + OFF_U;   // K steps of 16 rows = 2 KB
      // MMA3 of chunk m: O rows (64-127) of D1 buffer m % 3 += M U.  A is the 64 rows before
      // M in shared memory, then M: the upper half of the product lands in the W S rows of
      // that buffer, which E1 has already read and nothing reads again before the buffer's
      // next MMA1 overwrites them.
      auto issue_mma3 = [&](int m) {
        const int stm = m % NSTAGE;
        const uint64_t a3 = sw128_desc(sbase + stm * STAGE_BYTES + A1_BYTES + A2_BYTES - M_BYTES);
        const uint32_t uB = sU0 + (m & 1) * U_BYTES;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma(d1_of(m), desc_add(a3, k * 32), sw128_mn_desc(uB + k * 2048, 8192), id, 1);
        umma_commit(bar(BAR_EMPTY0 + stm));
        // O of chunk m complete in D1 buffer m % 3 (its own barrier: the O warps may lag
        // behind the stage barrier by more than one phase, never behind this one)
        if (FUSE_NORM) umma_commit(bar(BAR_ODONE0 + m % 3));
      };
      int committed = 0;   // commits on BAR_MMA1 so far (one per chunk)
      for (int n = 0; n < nch; ++n) {
        const int st = n % NSTAGE;
        const uint64_t a1 = sw128_desc(sbase + st * STAGE_BYTES);
        const uint32_t a2s = sbase + st * STAGE_BYTES + A1_BYTES;
        const uint32_t d1 = d1_of(n), uB = sU0 + (n & 1) * U_BYTES;
        // the waits that are normally long satisfied first, the chain's own (S ready) last:
        // this chunk's tiles, and (fused norm) the O warps done with chunk n-3's O in this
        // D1 buffer
        if (!mbar_wait(bar(BAR_FULL0 + st), (n / NSTAGE) & 1, &abort_flag)) break;
        if (FUSE_NORM && n >= 3 &&
            !mbar_wait(bar(BAR_OFREE0 + n % 3), ((n / 3) - 1) & 1, &abort_flag))
          break;
        if (!mbar_wait(bar(BAR_SREADY), n & 1, &abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma(d1, desc_add(a1, (k >> 2) * 16384 + (k & 3) * 32),
               sw128_mn_desc(sS + k * 2048, 8192), id, k > 0);
        umma_commit(bar(BAR_MMA1));
        ++committed;
        // fused norm: the previous chunk's output product, off the chain (its U buffer is
        // rewritten only by chunk n+1's E1, which waits for chunk n+1's MMA1, issued after
        // this).  Without it, the epilogue warps read O themselves right after E2, so MMA3
        // follows MMA2 at once (below).
        if (FUSE_NORM && n > 0) issue_mma3(n - 1);
        if (!mbar_wait(bar(BAR_UREADY), n & 1, &abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma(d2_tmem, sw128_mn_desc(a2s + k * 2048, 8192), sw128_mn_desc(uB + k * 2048, 8192),
               id_amn, k > 0);
        umma_commit(bar(BAR_MMA2));
        if (!FUSE_NORM) issue_mma3(n);
      }
      if (FUSE_NORM && !abort_flag && nch > 0) issue_mma3(nch - 1);
      if (abort_flag) {  // let every issued MMA retire before TMEM is freed
        umma_commit(bar(BAR_MMA1));
        const long long t0 = clock64();
        while (!mbar_try(bar(BAR_MMA1), committed & 1) && clock64() - t0 < WAIT_LIMIT_CYCLES) {
        }
      }
    }
  } else if (FUSE_NORM && warp >= 2 + NEPI) {
    // ---------------- O warps (fused norm), off the serial chain ----------------
    // warp 10 / 11: TMEM lanes 64-95 / 96-127 = token rows r of the chunk, all 32 columns.
    // Per chunk: copy O out of D1 and release the buffer to the MMA issuer, then
    // y = O / sqrt(mean over the head's 128 columns of O^2 + eps) * w * sigmoid(g).
    const int q = warp & 3;                 // 2 or 3
    const int r = 32 * (q - 2) + lane;      // token row within the chunk
    const int ow = q - 2;                   // which O warp
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    float* ssq = reinterpret_cast<float*>(sm + OFF_SSQ);
    float nw[J];
#pragma unroll
    for (int c = 0; c < J; ++c) nw[c] = __ldg(a.norm_w + j0 + c);
    // gate row of chunk n (token t0 + r, this slice's 32 columns), zero past the end
    auto load_g = [&](int n, uint4 (&gv)[4]) {
      const int t0 = start + n * C;
#pragma unroll
      for (int k = 0; k < 4; ++k) gv[k] = make_uint4(0, 0, 0, 0);
      if (n < nch && r < min(C, end - t0)) {
        const uint4* gp = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.g) +
                                                         ((size_t)(t0 + r) * H + h) * D + j0);
#pragma unroll
        for (int k = 0; k < 4; ++k) gv[k] = gp[k];
      }
    };
    uint4 graw[4], gnext[4];
    load_g(0, graw);
    for (int n = 0; n < nch; ++n) {
      const int p = n & 1;
      const int t0 = start + n * C;
      const int L = min(C, end - t0);
      const size_t yo = ((size_t)(t0 + r) * H + h) * D + j0;
      load_g(n + 1, gnext);   // one chunk ahead: in flight through this chunk's work
      if (!mbar_wait_warp(bar(BAR_ODONE0 + n % 3), (n / 3) & 1, &abort_flag)) break;
      tc_fence_after();
      float o[J];
      tmem_ld16(d1_of(n) + lane_off, *reinterpret_cast<float(*)[16]>(o));
      tmem_ld16(d1_of(n) + lane_off + 16, *reinterpret_cast<float(*)[16]>(o + 16));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_OFREE0 + n % 3));
      float part = 0.f;
#pragma unroll
      for (int c = 0; c < J; ++c) part = fmaf(o[c], o[c], part);
      // Token r's partial from slice CTA `rank` lands in slot [p][rank][r] of every CTA.  A
      // slot of parity p is rewritten (chunk n) only after this warp's producer passed the
      // full barrier of chunk n-1, which every consumer warp reaches only after reading
      // chunk n-2: two slots need no separate "free" handshake.
      if (ow == 0 && lane == 0) mbar_expect_tx(bar(BAR_NFULL0 + p), NORM_TX_BYTES);
      const uint32_t slot = smem_u32(ssq + (p * NSLICE + blockIdx.x) * C + r);
#pragma unroll
      for (int dst = 0; dst < NSLICE; ++dst)
        st_async_cluster(cluster_map(slot, dst), part, cluster_map(bar(BAR_NFULL0 + p), dst));
      if (!mbar_wait_warp(bar(BAR_NFULL0 + p), (n >> 1) & 1, &abort_flag)) break;
      float tot = 0.f;
#pragma unroll
      for (int k = 0; k < NSLICE; ++k) tot += ssq[(p * NSLICE + k) * C + r];
      if (r < L) {
        const float rstd = rsqrtf(tot * (1.0f / D) + a.norm_eps);
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(graw);
        uint4 out[4];
        __nv_bfloat162* y2 = reinterpret_cast<__nv_bfloat162*>(out);
#pragma unroll
        for (int c = 0; c < J; c += 2) {
          const float2 gv = __bfloat1622float2(g2[c / 2]);
          y2[c / 2] = __floats2bfloat162_rn(o[c] * rstd * nw[c] * fast_sigmoid(gv.x),
                                            o[c + 1] * rstd * nw[c + 1] * fast_sigmoid(gv.y));
        }
        uint4* yp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.y) + yo);
#pragma unroll
        for (int k = 0; k < 4; ++k) yp[k] = out[k];
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) graw[k] = gnext[k];
    }
  } else if (warp < 2 + NEPI) {
    // ---------------- epilogue warps 2..9 ----------------
    const int q = warp & 3;                 // TMEM lane quarter
    const int half = (warp - 2) / 4;        // which 16 of the slice's 32 value columns
    const int i = 32 * q + lane;            // key row of the state slice / TMEM lane
    const int cb = JH * half;               // first column of this thread
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    unsigned char* SB = sm + OFF_S;
    unsigned char* UB0 = sm + OFF_U;
    const float* gCg = reinterpret_cast<const float*>(a.ws + a.L.gC);
    float* og = reinterpret_cast<float*>(a.ws + a.L.o);
    const size_t sg = (((size_t)row * H + h) * D + i) * D + j0 + cb;

    float S[JH];
    if (a.state_in) {
#pragma unroll
      for (int c = 0; c < JH; c += 4) {
        const float4 v = *reinterpret_cast<const float4*>(a.state_in + sg + c);
        S[c] = v.x; S[c + 1] = v.y; S[c + 2] = v.z; S[c + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < JH; ++c) S[c] = 0.f;
    }
    auto write_state = [&]() {   // key row i, columns cb..cb+15: two 16-byte chunks
      *reinterpret_cast<uint4*>(SB + mn_row_chunk(i, cb / 8)) = pack8_bf16(S);
      *reinterpret_cast<uint4*>(SB + mn_row_chunk(i, cb / 8 + 1)) = pack8_bf16(S + 8);
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(BAR_SREADY));
    };
    write_state();

    for (int n = 0; n < nch; ++n) {
      const int st = n % NSTAGE;
      unsigned char* UB = UB0 + (n & 1) * U_BYTES;
      const int tile = (start / C + s + n) * H + h;
      const int t0 = start + n * C;
      const int L = min(C, end - t0);
      const float gc = __ldg(gCg + (size_t)tile * D + i);
      if (q < 2) {
        // E1: U = U~ - W S for token row r = i (0..63), columns cb..cb+15.  The U~ row is
        // read (its stage has landed: this warp waits for it too) before MMA1 is waited for.
        if (!mbar_wait_warp(bar(BAR_FULL0 + st), (n / NSTAGE) & 1, &abort_flag)) break;
        const __nv_bfloat16* ut =
            reinterpret_cast<const __nv_bfloat16*>(sm + st * STAGE_BYTES + A1_BYTES + A2_BYTES +
                                                   M_BYTES) + i * J + cb;
        float uf[JH];
#pragma unroll
        for (int m = 0; m < JH; m += 8) {
          const uint4 raw = *reinterpret_cast<const uint4*>(ut + m);
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p2[e]);
            uf[m + 2 * e] = f.x;
            uf[m + 2 * e + 1] = f.y;
          }
        }
        if (!mbar_wait_warp(bar(BAR_MMA1), n & 1, &abort_flag)) break;
        tc_fence_after();
        float ws[JH];
        tmem_ld16(d1_of(n) + lane_off + cb, ws);
#pragma unroll
        for (int m = 0; m < JH; m += 8) {   // token row i, columns cb+m..cb+m+7
          float u[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) u[e] = (i < L) ? uf[m + e] - ws[m + e] : 0.f;
          *reinterpret_cast<uint4*>(UB + mn_row_chunk(i, (cb + m) / 8)) = pack8_bf16(u);
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(bar(BAR_UREADY));
      }
      // E2: state update for key row i (on the serial chain)
      if (!mbar_wait_warp(bar(BAR_MMA2), n & 1, &abort_flag)) break;
      tc_fence_after();
      {
        float dv[JH];
        tmem_ld16(d2_tmem + lane_off + cb, dv);
#pragma unroll
        for (int m = 0; m < JH; ++m) S[m] = fmaf(gc, S[m], dv[m]);
      }
      write_state();
      if (!FUSE_NORM && q >= 2) {
        // E3 (off the chain): O rows (TMEM lanes 64-127) once MMA3 has retired
        if (!mbar_wait_warp(bar(BAR_EMPTY0 + st), (n / NSTAGE) & 1, &abort_flag)) break;
        tc_fence_after();
        float o[JH];
        tmem_ld16(d1_of(n) + lane_off + cb, o);
        const int r = i - 64;
        if (r < L) {
          float* op = og + ((size_t)(t0 + r) * H + h) * D + j0 + cb;
#pragma unroll
          for (int c = 0; c < JH; c += 4)
            *reinterpret_cast<float4*>(op + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
        }
      }
    }
    if (!abort_flag && a.state_out) {
#pragma unroll
      for (int c = 0; c < JH; c += 4)
        *reinterpret_cast<float4*>(a.state_out + sg + c) =
            make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_flag && threadIdx.x == 0) atomicExch(status, (int)5 /* KDA_ERR_TIMEOUT */);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(TMEM_COLS)
                 : "memory");
  }
  // no CTA leaves while a peer may still write its shared memory or arrive at its barriers
  if (FUSE_NORM) cluster_sync_all();
}

// Self-test of the bounded wait: one warp waits on an mbarrier that nothing
// arrives at, gives up after `limit` cycles and records KDA_ERR_TIMEOUT in the
// status word, exactly as the prefill kernel does on a stalled pipeline.
__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(int* status, long long limit) {
  __shared__ __align__(8) uint64_t never;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&never), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  const long long t0 = clock64();
  bool ok = true;
  while (!mbar_try(smem_u32(&never), 0)) {
    if (clock64() - t0 > limit) { ok = false; break; }
  }
  if (!ok && threadIdx.x == 0) atomicExch(status, 5 /* KDA_ERR_TIMEOUT */);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<EncodeTiledFn>(fn);
}

// 2D bf16 tensor [rows, cols] (cols contiguous), box [box_rows, 64 cols], 128B swizzle
bool make_map(EncodeTiledFn enc, CUtensorMap* m, void* base, uint64_t rows, uint64_t cols,
              uint32_t box_rows, uint32_t box_cols = 64,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_chain_maps(const PrefillArgs& a, ChainMaps* m) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const uint64_t tiles = (uint64_t)a.L.nslots * a.H;
  return make_map(enc, &m->W, a.ws + a.L.W, tiles * C, D, 64) &&
         make_map(enc, &m->Q, a.ws + a.L.Qt, tiles * C, D, 64) &&
         make_map(enc, &m->KT, a.ws + a.L.Kp, tiles * C, D, 64) &&
         make_map(enc, &m->M, a.ws + a.L.M, tiles * C, C, 64) &&
         make_map(enc, &m->Ut, a.ws + a.L.Ut, tiles * C, D, 64);
}

cudaError_t launch_wait_timeout_selftest(void* workspace, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(static_cast<int*>(workspace),
                                                 WAIT_LIMIT_CYCLES / 4);
  return cudaGetLastError();
}

// pairs with the tcgen05 intra-chunk pass (K' token-major), so the same condition
bool sm100_interchunk_supported(const PrefillArgs& a) {
  return a.bf16 && a.D == D && a.C == C && !a.gate_softplus;
}

// the fused norm runs 4-CTA clusters; it is used unless it needs more waves of CTAs than
// the plain launch (the cluster occupancy is queried once per device)
static bool fuse_norm_fits(int clusters) {
  static int max_clusters[64];
  static bool known[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!known[dev]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(NSLICE, 64, 1);
    cfg.blockDim = dim3(threads_of<true>(), 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = NSLICE;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaFuncSetAttribute(interchunk_sm100_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, interchunk_sm100_kernel<true>, &cfg) != cudaSuccess)
      n = 0;
    cudaGetLastError();
    max_clusters[dev] = n;
    known[dev] = true;
  }
  int nsm = 0;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (max_clusters[dev] < 1 || nsm < NSLICE) return false;
  // fuse unless it needs more waves of CTAs than the plain launch (one CTA per SM)
  const long long plain_waves = ((long long)clusters * NSLICE + nsm - 1) / nsm;
  const long long fused_waves = ((long long)clusters + max_clusters[dev] - 1) / max_clusters[dev];
  return fused_waves <= plain_waves;
}

cudaError_t launch_interchunk_sm100(const PrefillArgs& a, cudaStream_t st, bool* fused_norm) {
  static_assert(NSLICE * J == D, "slices must cover the value axis");
  *fused_norm = false;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  TmaMaps maps;
  const uint64_t tiles = (uint64_t)a.L.nslots * a.H;
  if (!make_map(enc, &maps.W, a.ws + a.L.W, tiles * C, D, 64) ||
      !make_map(enc, &maps.Q, a.ws + a.L.Qt, tiles * C, D, 64) ||
      !make_map(enc, &maps.KT, a.ws + a.L.Kp, tiles * C, D, 64) ||
      !make_map(enc, &maps.M, a.ws + a.L.M, tiles * C, C, 64) ||
      !make_map(enc, &maps.Ut, a.ws + a.L.Ut, tiles * C, D, 64, J, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const dim3 grid(NSLICE, a.H, a.n_seqs);
  if (a.y != nullptr && a.total > 0 && fuse_norm_fits(a.H * a.n_seqs)) {
    cudaError_t e = cudaFuncSetAttribute(interchunk_sm100_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads_of<true>(), 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = NSLICE;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, interchunk_sm100_kernel<true>, a, maps);
    if (e == cudaSuccess) {
      *fused_norm = true;
      ++launch_counter();
    }
    return e;
  }
  cudaError_t e = cudaFuncSetAttribute(interchunk_sm100_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  interchunk_sm100_kernel<false><<<grid, threads_of<false>(), SMEM_BYTES, st>>>(a, maps);
  ++launch_counter();
  return cudaGetLastError();
}

}  // namespace kda
