// The inter-chunk chain of the co-scheduled prefill (sm_100a): one CTA carries one head
// through every sequence of the batch, chunk by chunk, with all 128 value columns of the
// state, so H heads need H SMs and the rest of the GPU runs the intra-chunk pass in the
// same launch.  Per chunk (C = 64 tokens), with S the bf16 copy of the state (128 keys x
// 128 values) and the chunk's tiles from the intra-chunk pass:
//   MMA1   D1[128 x 128] = [W ; Q~] (128 x 128) . S      rows 0-63: W S, rows 64-127: Q~ S
//   E1     U = U~ - W S (fp32, rows past the sequence end forced to 0) -> bf16 U in smem
//   MMA2   D2[128 x 128] = K'^T (128 x 64) . U           state increment (key rows)
//   MMA3   D1[64:128]   += M (64 x 64) . U               O = Q~ S + M U (A = [X ; M], X the
//                                                         8 KB before M: its rows land in
//                                                         D1[0:64], already read)
//   E2     S <- Diag(e^{G_C}) S + D2 in fp32 registers -> bf16 S in smem (at a sequence's
//          end the state goes out and the next sequence's comes in instead)
//   E3     y = O / rms(O) * w * sigmoid(g) on TMEM lane quarters 2-3 in four 32-column
//          slices, the sums of squares exchanged through shared memory
// This is the arithmetic of the 4-slice inter-chunk pass with the slices side by side:
// each state element takes the same operations in the same order, and E3 sums a
// token's squares in four 32-column partials, added in slice order, as that pass does.
// Warp roles: warp 0 waits for each tile's ready flag (written by the intra-chunk
// CTAs) and loads the chunk with TMA into two stages; warp 1 allocates all 512 TMEM
// columns (D1 three times, D2) and issues the MMAs from one thread (MMA3 of chunk n
// after MMA1 of chunk n+1, off the chain; U double-buffered for it); warps 4-15 run E1/E2,
// three per TMEM lane quarter (quarter = warp % 4), owning value columns 0-47, 48-95 and
// 96-127; E3 runs on warps 2-3 (slices 0-2) and on the narrowest E2 warps of quarters 2-3
// (slice 3 of the previous chunk, after their E2), so the other E2 warps of those quarters
// carry nothing but the chain.  Every wait is bounded.
#pragma once

#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_sm100.cuh"

namespace kda {
namespace chain {

constexpr int D = 128, C = 64;
constexpr int THREADS = 512;
constexpr uint32_t TMEM_COLS = 512;

// shared memory carve-up (offsets from a 1024-byte aligned base)
constexpr uint32_t A1_BYTES = 2 * 128 * 128;   // [W;Q~]: 2 K-blocks x 128 rows x 128 B
constexpr uint32_t A2_BYTES = 128 * 128;       // K': 64 tokens x 128 keys, read MN-major
constexpr uint32_t M_BYTES = 64 * 128;         // M: 64 rows x 64
constexpr uint32_t UT_HALF = 64 * 128;         // U~: 64 rows x 64 columns, 128B swizzle
constexpr uint32_t STAGE_BYTES = A1_BYTES + A2_BYTES + M_BYTES + 2 * UT_HALF;   // 72 KB
constexpr uint32_t NSTAGE = 2;
constexpr uint32_t TX_BYTES = STAGE_BYTES;
// S (128 key rows) and U (64 token rows) as MN-major B operands: two groups of 64 value
// columns, each a 128-byte swizzled row per key / token
constexpr uint32_t S_GROUP = 128 * 128;
constexpr uint32_t OFF_S = NSTAGE * STAGE_BYTES;
constexpr uint32_t U_GROUP = 64 * 128;
constexpr uint32_t U_BYTES = 2 * U_GROUP;
constexpr uint32_t OFF_U = OFF_S + 2 * S_GROUP;
constexpr uint32_t OFF_NW = OFF_U + 2 * U_BYTES;    // RMSNorm weight, fp32 [128]
constexpr uint32_t OFF_SSQ = OFF_NW + D * 4;        // [2 parities][64 tokens][4 slices] fp32
constexpr uint32_t OFF_BAR = OFF_SSQ + 2 * C * 4 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;   // + alignment slack
static_assert(SMEM_BYTES <= 220 * 1024, "shared memory of one CTA (with the static part)");

enum { BAR_FULL0 = 0, BAR_FULL1, BAR_EMPTY0, BAR_EMPTY1, BAR_MMA1, BAR_MMA2, BAR_SREADY,
       BAR_UREADY, BAR_OFREE0, BAR_OFREE1, BAR_OFREE2, BAR_ODONE0, BAR_ODONE1, BAR_ODONE2,
       BAR_SSQ0, BAR_SSQ1, BAR_SSQ2, BAR_SSQ3, BAR_COUNT };
static_assert(BAR_COUNT * 8 <= 256, "barrier slots");
constexpr int NE = 12;        // E1/E2 warps (4..15)
constexpr int NOUT = 4;       // warps of E3: 2, 3 and the narrowest E2 warps of quarters 2-3

// sigmoid(z) = (1 + tanh(z / 2)) / 2 with one special-function op (tanh.approx, absolute
// error about 2^-11): the outputs are bf16 and the output gate's error stays far inside
// the parity budget; the two inter-chunk kernels share the form, so their outputs agree
__device__ __forceinline__ float sigmoid_fast(float z) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
  return fmaf(0.5f, t, 0.5f);
}

// byte offset of element (row k, 16-byte chunk) of an MN-major, 128B-swizzled tile
__device__ __forceinline__ uint32_t mn_chunk(int k, int chunk) {
  return (uint32_t)((k >> 3) * 1024 + (k & 7) * 128 + (((chunk ^ k) & 7) << 4));
}
__device__ __forceinline__ uint4 pack8(const float* v) {
  uint4 r;
  __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
  for (int e = 0; e < 4; ++e) p[e] = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
  return r;
}
__device__ __forceinline__ uint64_t desc_plus(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// 16 consecutive fp32 columns of this thread's TMEM lane, without the wait
__device__ __forceinline__ void tmem_ld16_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// bounded wait for a tile's ready flag (acquire at GPU scope); false on timeout or abort
__device__ __forceinline__ bool wait_ready(const int* flag, volatile int* abort_flag) {
  const long long t0 = clock64();
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > WAIT_LIMIT_CYCLES) {
      *abort_flag = 1;
      return false;
    }
    __nanosleep(64);
  }
}

// A head's chain walks the batch sequence by sequence, chunk by chunk: the order in which
// the intra-chunk role completes the tiles.  Position: sequence s (pool row `row`, tokens
// [start, end), nch chunks), chunk n.
struct ChainPos {
  int s, row, start, end, nch, n;
};
// the first sequence >= s0 that has a pool row and at least one token; false past the end
__device__ __forceinline__ bool chain_seq_from(const PrefillArgs& a, int s0, ChainPos& k) {
  for (int s = s0; s < a.n_seqs; ++s) {
    const int row = pool_row(a.slots, s, a.pool_size);
    if (row < 0) continue;
    int st, en;
    seq_range(a.cu, a.total, s, st, en);
    if (en > st) {
      k.s = s; k.row = row; k.start = st; k.end = en; k.nch = (en - st + C - 1) / C; k.n = 0;
      return true;
    }
  }
  return false;
}
// the next chunk of the walk; false past the end
__device__ __forceinline__ bool chain_next(const PrefillArgs& a, ChainPos& k) {
  if (++k.n < k.nch) return true;
  return chain_seq_from(a, k.s + 1, k);
}

// The chain of head h over every sequence of the batch.  `flags` holds one word per
// workspace tile, set once the intra-chunk pass has written all of that tile.
__device__ __forceinline__ void chain_body(const PrefillArgs& a, const ChainMaps& maps, int h,
                                           const int* flags) {
  extern __shared__ __align__(1024) unsigned char smraw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  __shared__ uint32_t tmem_holder;
  __shared__ volatile int abort_flag;
  constexpr int MAX_EMPTY = 64;
  __shared__ int walk_chunks, n_empty, empty_seq[MAX_EMPTY];   // set up by all threads at once

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.H;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  if (threadIdx.x == 0) {
    walk_chunks = 0;
    n_empty = 0;
  }
  __syncthreads();
  // the walk's length, and the sequences with a pool row but no tokens (their state passes
  // through): every thread looks at a strided share of the batch
  for (int sq = threadIdx.x; sq < a.n_seqs; sq += blockDim.x) {
    if (pool_row(a.slots, sq, a.pool_size) < 0) continue;
    int st, en;
    seq_range(a.cu, a.total, sq, st, en);
    if (en > st) {
      atomicAdd(&walk_chunks, (en - st + C - 1) / C);
    } else {
      const int e = atomicAdd(&n_empty, 1);
      if (e < MAX_EMPTY) empty_seq[e] = sq;
    }
  }
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int st = 0; st < (int)NSTAGE; ++st) {
      mbar_init(bar(BAR_FULL0 + st), 1);
      mbar_init(bar(BAR_EMPTY0 + st), 1);
    }
    mbar_init(bar(BAR_MMA1), 1);
    mbar_init(bar(BAR_MMA2), 1);
    mbar_init(bar(BAR_SREADY), 32 * NE);
    mbar_init(bar(BAR_UREADY), 32 * NE / 2);
    for (int b = 0; b < 3; ++b) {
      mbar_init(bar(BAR_OFREE0 + b), NOUT);
      mbar_init(bar(BAR_ODONE0 + b), 1);
    }
    for (int b = 0; b < 4; ++b) mbar_init(bar(BAR_SSQ0 + b), 2);   // [quarter 2-3][parity]
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x < D) reinterpret_cast<float*>(sm + OFF_NW)[threadIdx.x] = __ldg(a.norm_w + threadIdx.x);
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
  // [W S ; O] of chunk n in D1 buffer n % 3 (three, so the E3 warps have slack); K'^T U in D2
  auto d1_of = [&](int n) -> uint32_t { return tmem + 128u * (uint32_t)(n % 3); };
  const uint32_t d2_tmem = tmem + 384;
  int* status = reinterpret_cast<int*>(a.ws + a.L.status);
  auto tile_of = [&](const ChainPos& k) { return (k.start / C + k.s + k.n) * H + h; };
  // E3 of chunk m for the 32 tokens of TMEM lane quarter q (2 or 3) and value columns
  // 32 j .. 32 j + 31 (slice j) by one warp: its squares' partial sum goes into the
  // exchange beside the other three slices' (from the quarter's dedicated E3 warp), the four
  // are added in slice order after a bounded mbarrier wait.  `gb` holds the slice's gate row.
  auto o_slice = [&](int m, int t0, int L, int q, int j, const uint4 (&gb)[4]) -> bool {
    if (!mbar_wait_warp(bar(BAR_ODONE0 + m % 3), (m / 3) & 1, &abort_flag)) return false;
    tc_fence_after();
    const int lane = threadIdx.x & 31;
    uint32_t o0[16], o1[16];
    const uint32_t ob = d1_of(m) + ((uint32_t)(32 * q) << 16) + 32 * j;
    tmem_ld16_issue(ob, o0);
    tmem_ld16_issue(ob + 16, o1);
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(BAR_OFREE0 + m % 3));
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) part = fmaf(__uint_as_float(o0[e]), __uint_as_float(o0[e]), part);
#pragma unroll
    for (int e = 0; e < 16; ++e) part = fmaf(__uint_as_float(o1[e]), __uint_as_float(o1[e]), part);
    const int r = 32 * (q - 2) + lane;
    float* ssq = reinterpret_cast<float*>(sm + OFF_SSQ) + (m & 1) * (C * 4);
    ssq[r * 4 + j] = part;
    __syncwarp();
    const uint32_t xb = bar(BAR_SSQ0 + 2 * (q - 2) + (m & 1));
    if (lane == 0) mbar_arrive(xb);
    if (!mbar_wait_warp(xb, (m >> 1) & 1, &abort_flag)) return false;
    const float4 pp = *reinterpret_cast<const float4*>(ssq + r * 4);
    float tot = 0.f;
    tot += pp.x;
    tot += pp.y;
    tot += pp.z;
    tot += pp.w;
    const float rstd = rsqrtf(tot * (1.0f / D) + a.norm_eps);
    if (r < L) {
      const float* nw = reinterpret_cast<const float*>(sm + OFF_NW) + 32 * j;
      uint4* yp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.y) +
                                           ((size_t)(t0 + r) * H + h) * D + 32 * j);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const uint32_t* o = hf ? o1 : o0;
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gb[2 * hf]);
        uint4 out[2];
        __nv_bfloat162* y2 = reinterpret_cast<__nv_bfloat162*>(out);
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const int col = 16 * hf + e;
          const float2 gf = __bfloat1622float2(g2[e / 2]);
          y2[e / 2] = __floats2bfloat162_rn(
              __uint_as_float(o[e]) * rstd * nw[col] * sigmoid_fast(gf.x),
              __uint_as_float(o[e + 1]) * rstd * nw[col + 1] * sigmoid_fast(gf.y));
        }
        yp[2 * hf] = out[0];
        yp[2 * hf + 1] = out[1];
      }
    }
    return true;
  };
  // the gate row of token t0 + 32 (q - 2) + lane of a chunk of L tokens, columns 32 j .. +31
  auto load_gate = [&](int t0, int L, int q, int j, uint4 (&gb)[4]) {
    const int r = 32 * (q - 2) + (threadIdx.x & 31);
    const bool live = r < L;
    const uint4* gp = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.g) +
                                                     ((size_t)(t0 + r) * H + h) * D + 32 * j);
#pragma unroll
    for (int k = 0; k < 4; ++k) gb[k] = make_uint4(0, 0, 0, 0);
    if (live) {
#pragma unroll
      for (int k = 0; k < 4; ++k) gb[k] = __ldg(gp + k);
    }
  };

  if (warp == 0) {
    // ---------------- ready flags + TMA producer ----------------
    if (lane == 0) {
      int issued = 0;
      ChainPos k;
      bool more = chain_seq_from(a, 0, k);
      for (int n = 0; more && !abort_flag; ++n, more = chain_next(a, k)) {
        const int st = n % NSTAGE;
        if (n >= (int)NSTAGE &&
            !mbar_wait(bar(BAR_EMPTY0 + st), ((n / NSTAGE) - 1) & 1, &abort_flag))
          break;
        const int tile = tile_of(k);
        if (!wait_ready(flags + tile, &abort_flag)) break;
        // the tile was written through the generic proxy by other SMs; TMA reads it
        // through the async proxy
        asm volatile("fence.proxy.async.global;" ::: "memory");
        const uint32_t A1 = sbase + st * STAGE_BYTES, A2 = A1 + A1_BYTES, Ms = A2 + A2_BYTES;
        const uint32_t UTs = Ms + M_BYTES;
        const uint32_t fb = bar(BAR_FULL0 + st);
        mbar_expect_tx(fb, TX_BYTES);
        tma_load_2d(A1, &maps.W, 0, tile * C, fb);
        tma_load_2d(A1 + 16384, &maps.W, 64, tile * C, fb);
        tma_load_2d(A1 + 8192, &maps.Q, 0, tile * C, fb);
        tma_load_2d(A1 + 16384 + 8192, &maps.Q, 64, tile * C, fb);
        tma_load_2d(A2, &maps.KT, 0, tile * C, fb);
        tma_load_2d(A2 + 8192, &maps.KT, 64, tile * C, fb);
        tma_load_2d(Ms, &maps.M, 0, tile * C, fb);
        tma_load_2d(UTs, &maps.Ut, 0, tile * C, fb);
        tma_load_2d(UTs + UT_HALF, &maps.Ut, 64, tile * C, fb);
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
      const uint32_t id = idesc_bf16(128, 128) | (1u << 16);   // B (S or U) MN-major
      const uint32_t id_amn = id | (1u << 15);                  // K' is read MN-major too
      const uint32_t sS = sbase + OFF_S, sU0 = sbase + OFF_U;  // K steps of 16 rows = 2 KB
      auto issue_mma3 = [&](int m) {
        const int stm = m % NSTAGE;
        const uint64_t a3 = sw128_desc(sbase + stm * STAGE_BYTES + A1_BYTES + A2_BYTES - M_BYTES);
        const uint32_t uB = sU0 + (m & 1) * U_BYTES;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma(d1_of(m), desc_plus(a3, k * 32), sw128_mn_desc(uB + k * 2048, U_GROUP), id, 1);
        umma_commit(bar(BAR_EMPTY0 + stm));
        umma_commit(bar(BAR_ODONE0 + m % 3));
      };
      const int nch = walk_chunks;   // chunks of the whole walk
      int committed = 0;
      for (int n = 0; n < nch; ++n) {
        const int st = n % NSTAGE;
        const uint64_t a1 = sw128_desc(sbase + st * STAGE_BYTES);
        const uint32_t a2s = sbase + st * STAGE_BYTES + A1_BYTES;
        const uint32_t d1 = d1_of(n), uB = sU0 + (n & 1) * U_BYTES;
        if (!mbar_wait(bar(BAR_FULL0 + st), (n / NSTAGE) & 1, &abort_flag)) break;
        if (n >= 3 && !mbar_wait(bar(BAR_OFREE0 + n % 3), ((n / 3) - 1) & 1, &abort_flag))
          break;
        if (!mbar_wait(bar(BAR_SREADY), n & 1, &abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma(d1, desc_plus(a1, (k >> 2) * 16384 + (k & 3) * 32),
               sw128_mn_desc(sS + k * 2048, S_GROUP), id, k > 0);
        umma_commit(bar(BAR_MMA1));
        ++committed;
        // the previous chunk's output product, off the chain (its U buffer is rewritten
        // only by chunk n+1's E1, which waits for chunk n+1's MMA1, issued after this)
        if (n > 0) issue_mma3(n - 1);
        if (!mbar_wait(bar(BAR_UREADY), n & 1, &abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma(d2_tmem, sw128_mn_desc(a2s + k * 2048, 8192), sw128_mn_desc(uB + k * 2048, U_GROUP),
               id_amn, k > 0);
        umma_commit(bar(BAR_MMA2));
      }
      if (!abort_flag && nch > 0) issue_mma3(nch - 1);
      if (abort_flag) {  // let every issued MMA retire before TMEM is freed
        umma_commit(bar(BAR_MMA1));
        const long long t0 = clock64();
        while (!mbar_try(bar(BAR_MMA1), committed & 1) && clock64() - t0 < WAIT_LIMIT_CYCLES) {
        }
      }
    }
  } else if (warp < 4) {
    // ---------------- E3, slices 0-2 (warps 2, 3), off the serial chain ----------------
    // Per chunk: the three slices' sums of squares into the exchange, then, once the fourth
    // (from the narrowest E2 warp of the quarter) is in, y for the three slices.
    const int q = warp & 3;
    const int r = 32 * (q - 2) + lane;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const float* nwb = reinterpret_cast<const float*>(sm + OFF_NW);
    ChainPos k;
    bool more = chain_seq_from(a, 0, k);
    for (int m = 0; more; ++m) {
      const int t0 = k.start + k.n * C, L = min(C, k.end - t0);
      uint4 gcur[4];    // the gate row's slice 0, in flight through the waits below
      load_gate(t0, L, q, 0, gcur);
      if (r < L)        // slices 1-2 (and 3) into L2
        asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const __nv_bfloat16*>(a.g) +
                                                       ((size_t)(t0 + r) * H + h) * D + 64));
      if (!mbar_wait_warp(bar(BAR_ODONE0 + m % 3), (m / 3) & 1, &abort_flag)) break;
      tc_fence_after();
      const uint32_t ob = d1_of(m) + lane_off;
      float* ssq = reinterpret_cast<float*>(sm + OFF_SSQ) + (m & 1) * (C * 4);
#pragma unroll 1
      for (int j = 0; j < 3; ++j) {
        float part = 0.f;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t o[16];
          tmem_ld16_issue(ob + 32 * j + 16 * hf, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) part = fmaf(__uint_as_float(o[e]), __uint_as_float(o[e]), part);
        }
        ssq[r * 4 + j] = part;
      }
      __syncwarp();
      const uint32_t xb = bar(BAR_SSQ0 + 2 * (q - 2) + (m & 1));
      if (lane == 0) mbar_arrive(xb);
      if (!mbar_wait_warp(xb, (m >> 1) & 1, &abort_flag)) break;
      const float4 pp = *reinterpret_cast<const float4*>(ssq + r * 4);
      float tot = 0.f;
      tot += pp.x;
      tot += pp.y;
      tot += pp.z;
      tot += pp.w;
      const float rstd = rsqrtf(tot * (1.0f / D) + a.norm_eps);
      uint4* yp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.y) +
                                           ((size_t)(t0 + r) * H + h) * D);
#pragma unroll 1
      for (int j = 0; j < 3; ++j) {
        uint4 gnext[4];   // the next slice's gate, in flight through this one
        load_gate(t0, j < 2 ? L : 0, q, j < 2 ? j + 1 : 0, gnext);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t o[16];
          tmem_ld16_issue(ob + 32 * j + 16 * hf, o);
          tmem_ld_wait();
          const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gcur[2 * hf]);
          uint4 out[2];
          __nv_bfloat162* y2 = reinterpret_cast<__nv_bfloat162*>(out);
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int col = 32 * j + 16 * hf + e;
            const float2 gf = __bfloat1622float2(g2[e / 2]);
            y2[e / 2] = __floats2bfloat162_rn(
                __uint_as_float(o[e]) * rstd * nwb[col] * sigmoid_fast(gf.x),
                __uint_as_float(o[e + 1]) * rstd * nwb[col + 1] * sigmoid_fast(gf.y));
          }
          if (r < L) {
            yp[4 * j + 2 * hf] = out[0];
            yp[4 * j + 2 * hf + 1] = out[1];
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) gcur[e] = gnext[e];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_OFREE0 + m % 3));
      more = chain_next(a, k);
    }
  } else {
    // ---------------- E1 / E2 warps 4..15 ----------------
    const int q = warp & 3;                  // TMEM lane quarter
    const int part = (warp - 4) >> 2;        // value columns 0-47, 48-95 or 96-127
    const int cb = 48 * part;
    const int ng = part < 2 ? 3 : 2;         // 16-column groups of this thread
    const int i = 32 * q + lane;             // key row of the state / TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    unsigned char* SB = sm + OFF_S;
    unsigned char* UB0 = sm + OFF_U;
    const float* gCg = reinterpret_cast<const float*>(a.ws + a.L.gC);
    // this thread's part of a state: key row i, value columns cb + 16 g .. (ng groups)
    auto state_at = [&](int row) { return (((size_t)row * H + h) * D + i) * D + cb; };
    float S[3][16];
    auto load_state = [&](int row) {
#pragma unroll
      for (int g = 0; g < 3; ++g)
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          if (g < ng && a.state_in)
            v = *reinterpret_cast<const float4*>(a.state_in + state_at(row) + 16 * g + e);
          S[g][e] = v.x; S[g][e + 1] = v.y; S[g][e + 2] = v.z; S[g][e + 3] = v.w;
        }
    };
    auto store_state = [&](int row) {
      if (!a.state_out) return;
#pragma unroll
      for (int g = 0; g < 3; ++g)
        if (g < ng)
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(a.state_out + state_at(row) + 16 * g + e) =
                make_float4(S[g][e], S[g][e + 1], S[g][e + 2], S[g][e + 3]);
    };
    // sequences without tokens keep their state (state_in, or zeros, to state_out); past
    // MAX_EMPTY of them the list is incomplete and the batch is walked instead
    if (a.state_out) {
      if (n_empty <= MAX_EMPTY) {
        for (int e = 0; e < n_empty; ++e) {
          const int row = pool_row(a.slots, empty_seq[e], a.pool_size);
          load_state(row);
          store_state(row);
        }
      } else {
        for (int sq = 0; sq < a.n_seqs; ++sq) {
          const int row = pool_row(a.slots, sq, a.pool_size);
          int st, en;
          seq_range(a.cu, a.total, sq, st, en);
          if (row < 0 || en > st) continue;
          load_state(row);
          store_state(row);
        }
      }
    }
    auto write_state = [&]() {   // key row i, 16 columns per group: two 16-byte chunks each
#pragma unroll
      for (int g = 0; g < 3; ++g)
        if (g < ng) {
          const int c0 = cb + 16 * g;
          unsigned char* base = SB + (c0 >> 6) * S_GROUP;
          const int ch = (c0 & 63) >> 3;
          *reinterpret_cast<uint4*>(base + mn_chunk(i, ch)) = pack8(S[g]);
          *reinterpret_cast<uint4*>(base + mn_chunk(i, ch + 1)) = pack8(S[g] + 8);
        }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(BAR_SREADY));
    };
    ChainPos k;
    bool more = chain_seq_from(a, 0, k);
    if (more) load_state(k.row);
    write_state();
    uint4 gb[4];   // quarters 2-3: the gate row of the output slice of the previous chunk
    int pt0 = 0, pL = 0, n = 0;   // the previous chunk's first token and length

    for (; more; ++n) {
      const int st = n % NSTAGE;
      unsigned char* UB = UB0 + (n & 1) * U_BYTES;
      const int t0 = k.start + k.n * C;
      const int L = min(C, k.end - t0);
      // the stage has landed, so the producer saw the tile's ready flag: e^{G_C} is readable
      if (!mbar_wait_warp(bar(BAR_FULL0 + st), (n / NSTAGE) & 1, &abort_flag)) break;
      const float gc = __ldcg(gCg + (size_t)tile_of(k) * D + i);
      if (q >= 2 && part == 2 && n > 0) {   // the previous chunk's gate slice 3, into L2
        const int r = 32 * (q - 2) + lane;
        if (r < pL)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const __nv_bfloat16*>(a.g) +
                                                         ((size_t)(pt0 + r) * H + h) * D + 96));
      }
      const bool last = k.n + 1 == k.nch;
      if (last && a.state_in) {   // the next sequence's initial state, into L2
        ChainPos kn;
        if (chain_seq_from(a, k.s + 1, kn)) {
          const char* sp = reinterpret_cast<const char*>(a.state_in + state_at(kn.row));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(sp));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(sp + 128));
        }
      }
      if (q < 2) {
        // E1: U = U~ - W S for token row i (0..63), this thread's columns: groups 0-1, then 2
        const unsigned char* ut = sm + st * STAGE_BYTES + A1_BYTES + A2_BYTES + M_BYTES;
        auto e1_group = [&](int g, const uint32_t (&ws)[16]) {
          const int c0 = cb + 16 * g;
          const unsigned char* hb = ut + (c0 >> 6) * UT_HALF + i * 128;
          float u[16];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int ch = ((c0 & 63) >> 3) + e;
            const uint4 raw = *reinterpret_cast<const uint4*>(hb + (((ch ^ i) & 7) << 4));
            const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const float2 f = __bfloat1622float2(p2[m]);
              u[8 * e + 2 * m] = (i < L) ? f.x - __uint_as_float(ws[8 * e + 2 * m]) : 0.f;
              u[8 * e + 2 * m + 1] = (i < L) ? f.y - __uint_as_float(ws[8 * e + 2 * m + 1]) : 0.f;
            }
          }
          unsigned char* base = UB + (c0 >> 6) * U_GROUP;
          const int ch = (c0 & 63) >> 3;
          *reinterpret_cast<uint4*>(base + mn_chunk(i, ch)) = pack8(u);
          *reinterpret_cast<uint4*>(base + mn_chunk(i, ch + 1)) = pack8(u + 8);
        };
        if (!mbar_wait_warp(bar(BAR_MMA1), n & 1, &abort_flag)) break;
        tc_fence_after();
        {
          uint32_t w0[16], w1[16];
          tmem_ld16_issue(d1_of(n) + lane_off + cb, w0);
          tmem_ld16_issue(d1_of(n) + lane_off + cb + 16, w1);
          tmem_ld_wait();
          e1_group(0, w0);
          e1_group(1, w1);
        }
        if (ng == 3) {
          uint32_t w2[16];
          tmem_ld16_issue(d1_of(n) + lane_off + cb + 32, w2);
          tmem_ld_wait();
          e1_group(2, w2);
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(bar(BAR_UREADY));
      }
      // E2: state update for key row i (on the serial chain)
      if (!mbar_wait_warp(bar(BAR_MMA2), n & 1, &abort_flag)) break;
      tc_fence_after();
      {
        uint32_t d0[16], d1v[16];
        tmem_ld16_issue(d2_tmem + lane_off + cb, d0);
        tmem_ld16_issue(d2_tmem + lane_off + cb + 16, d1v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) S[0][e] = fmaf(gc, S[0][e], __uint_as_float(d0[e]));
#pragma unroll
        for (int e = 0; e < 16; ++e) S[1][e] = fmaf(gc, S[1][e], __uint_as_float(d1v[e]));
      }
      if (ng == 3) {
        uint32_t d2v[16];
        tmem_ld16_issue(d2_tmem + lane_off + cb + 32, d2v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) S[2][e] = fmaf(gc, S[2][e], __uint_as_float(d2v[e]));
      }
      if (last) {   // the sequence's final state out, the next one's initial state in
        store_state(k.row);
        more = chain_seq_from(a, k.s + 1, k);
        if (more) load_state(k.row);
      } else {
        ++k.n;
      }
      write_state();
      // E3 slice 3 of the previous chunk (its output product retired before this chunk's
      // MMA2), on the narrowest E2 warp of the quarter
      if (q >= 2 && part == 2 && n > 0) {
        load_gate(pt0, pL, q, 3, gb);
        if (!o_slice(n - 1, pt0, pL, q, 3, gb)) break;
      }
      pt0 = t0;
      pL = L;
    }
    if (q >= 2 && part == 2 && n > 0 && !abort_flag) {
      load_gate(pt0, pL, q, 3, gb);
      o_slice(n - 1, pt0, pL, q, 3, gb);
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
}

}  // namespace chain
}  // namespace kda
