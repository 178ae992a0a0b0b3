// Intra-chunk pass of the prefill on the 5th-generation tensor cores (sm_100a).
// Used for d = 128, chunk 64, bf16 activations; writes the per-slot workspace
// tiles W, U~, Q~ (token rows), K' (token rows), M and e^{G_C}.
//
// Two input modes share one kernel:
//   * kda_prefill: the prep outputs q, k, v, log a, beta (fp32) are read;
//   * kda_layer_prefill (FUSED): the raw pre-conv x, f and beta logit are read
//     and the prep of llama.cpp PR #27754's KDA commit (one depthwise causal
//     conv over q|k|v, SiLU, q/k L2 norm with max(||x||, eps), bounded-sigmoid
//     decay, sigmoid beta) runs here in fp32, so q/k/v never round-trip HBM.
//
// Persistent: one CTA per SM walks the (chunk slot, head) tiles.  With G the cumulative
// log decay of the chunk:
//   * Gram: A'[r,i] = sum_c k_r k_i e^{G_r - G_i} and M[r,i] = q_scale sum_c q_r k_i e^{G_r - G_i}.
//     The exponent is split at a reference row, row 15 for rows 0-31 and row 47
//     for rows 32-63: with the gate bounded below by -5, every factor is at most
//     e^80 (within fp32) and the products with i <= r are at most 1.  Both halves
//     run as ONE tf32 tcgen05 MMA, M = N = K = 128: A rows are the column-scaled
//     keys of both halves (32 + 64 rows), B rows the row-scaled keys and queries
//     (4 x 32 rows); only the two diagonal blocks of the product are read.  tf32
//     (not bf16) because the gram's rounding dominates the parity error budget.
//   * T = (I + A)^{-1} diag(b): forward substitution on the four 16 x 16 diagonal blocks,
//     then two levels of 32 x 32 doubling on mma.sync tf32 products split three ways (~fp32).
//   * W^T = (K e^G)^T T^T and U~^T = V^T T^T as bf16 MMAs, M = 128 (key / value
//     channels), N = 64, K = 64 tokens, with K e^G and V read MN-major (stored
//     token-major by the threads that compute them).  T and K e^G are each split
//     into a bf16 high part and the bf16 rounding of the remainder (hi + lo), and
//     W accumulates hi.hi + hi.lo + lo.hi, U~ accumulates V.hi + V.lo: the
//     rounding of T and K e^G was the largest term left in the error budget.
// Q~ = q_scale Q e^G, K' = K e^{G_C - G} and e^{G_C} are elementwise.  16 warps: warps
// w and w + 8 walk token rows 8(w%8)..8(w%8)+7 in pairs, each owning 64 of the 128
// channels of q, k and v (two per lane, one packed f32x2 pair); the per-token L2 norms are
// a shuffle reduce-scatter plus one exchange with the partner warp per row pair, and the
// conv keeps its window of K-1 previous rows in registers.  Per row and channel the row
// pass takes three exponentials: e^{G_r - G_ref} and its reciprocal give the gram scalings,
// e^{G_r} is e^{G_15} times the first (rows 0-31) and e^{G_C - G_r} is e^{G_C - G_47} times
// e^{G_47 - G_r} (both factors stay above 2^-116 with the gate bounded below by -5).
// After a tile's row pass, warps 0-7 run its serial tail (key gram readout, solve, W/U~) while
// warps 8-15 compute the next tile's gates (G, beta, e^{G_C}), so the next row pass starts at
// once; warps 12-15 then read the query gram M out of TMEM, off the tail's critical path.
#include <type_traits>

#include "kda_chain_sm100.cuh"
#include "kda_common.cuh"
#include "kda_launch.h"
#include "kda_sm100.cuh"

namespace kda {
namespace {

constexpr int D = 128, C = 64;
constexpr int THREADS = 512;   // 16 warps: two per group of 8 token rows (one per channel half)
constexpr int KC = 4;         // conv taps of the fused path
constexpr uint32_t TMEM_COLS = 128;

// shared memory carve-up (offsets from a 1024-byte aligned base)
constexpr uint32_t OFF_GA = 0;          // gram A: tf32, 4 K-blocks x 128 rows x 128 B (64 KB)
constexpr uint32_t OFF_GB = 65536;      // gram B: same shape (64 KB)
constexpr uint32_t OFF_KT = 131072;     // K e^G, high bf16 part: MN-major [64 t][128 c] (16 KB)
constexpr uint32_t OFF_KL = 147456;     // K e^G, low bf16 part (the rounding remainder)
constexpr uint32_t OFF_VT = 163840;     // V:     bf16 MN-major [64 t][128 c] (16 KB)
constexpr uint32_t OFF_G = 180224;      // G fp32 [64][128] (32 KB), written a tile ahead
constexpr uint32_t OFF_T = OFF_GA;      // T high part, bf16 K-major [64 r][64 i] (8 KB), after the gram
constexpr uint32_t OFF_TL = OFF_GA + 8192;  // T low part
constexpr int AF_LD = 68;                   // row stride (floats) of the fp32 tiles of the solve
constexpr uint32_t TILE32 = 64 * AF_LD * 4;
constexpr uint32_t OFF_XS = OFF_GA + 16384;  // X = (I + A)^{-1}, fp32 [64][68], after the gram
constexpr uint32_t OFF_ZS = OFF_XS + TILE32; // per-warp block products of the solve
constexpr int ZW_LD = 72;                    // their row stride (floats): fragment reads spread banks
constexpr int Z32_LD = 40;                   // the 32 x 32 block product, same bank spread
constexpr uint32_t SMEM_BYTES = OFF_G + 32768 + 1024;
static_assert(OFF_ZS + (4 * 16 * ZW_LD + 32 * Z32_LD) * 4 <= OFF_GB,
              "solve tiles must fit in the gram A area");
static_assert(TILE32 <= 65536, "A (fp32, after the gram) must fit in the gram B area");


// fp32 -> nearest tf32 (10 mantissa bits, ties away from zero: the rounding of
// cvt.rna.tf32.f32) with two integer operations on the bit pattern; finite inputs only
__device__ __forceinline__ float tf32_rna(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xffffe000u);
}
__device__ __forceinline__ void st_bf16x2(void* p, float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ void st_bf16x4(unsigned char* p, float a, float b, float c, float d) {
  st4(reinterpret_cast<__nv_bfloat16*>(p), make_float4(a, b, c, d));
}
// Special-function-unit approximations (flush-to-zero: the values they would keep as
// subnormals, below 2^-126, are negligible next to the bf16 tiles the pass writes).
// Exponents are carried in log2 units, so an exponential is one ex2.
constexpr float LOG2E = 1.4426950408889634f, LN2 = 0.6931471805599453f;
__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcpa(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rsqrta(float x) {
  float y;
  asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float tanha(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// sigmoid of z given z2 = z log2(e); 1 / (1 + inf) = 0 keeps the saturated end exact
__device__ __forceinline__ float sigmoid2(float z2) { return rcpa(1.f + ex2a(-z2)); }

// x = hi + lo with hi, lo tf32 (round to nearest)
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(x - __uint_as_float(hi)));
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// d (16 x 8, fragment layout) += A (16 x 8, row-major, stride lda) . B (8 x 8 [k][n], stride
// ldb), fp32 smem operands, as three tf32 products (the lo.lo term, ~2^-22, dropped), each
// into its own accumulator so consecutive calls form three short dependency chains
__device__ __forceinline__ void mma3_tf32(float (&d)[3][4], const float* A, int lda,
                                          const float* B, int ldb, int g, int t) {
  const float av[4] = {A[g * lda + t], A[(g + 8) * lda + t], A[g * lda + t + 4],
                       A[(g + 8) * lda + t + 4]};
  const float bv[2] = {B[t * ldb + g], B[(t + 4) * ldb + g]};
  uint32_t ah[4], al[4], bh[2], bl[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) split_tf32(av[i], ah[i], al[i]);
#pragma unroll
  for (int i = 0; i < 2; ++i) split_tf32(bv[i], bh[i], bl[i]);
  mma_tf32(d[0], ah, bh);
  mma_tf32(d[1], al, bh);
  mma_tf32(d[2], ah, bl);
}
__device__ __forceinline__ float sum3(const float (&d)[3][4], int i) {
  return d[0][i] + (d[1][i] + d[2][i]);
}

// two channels as loaded -> fp32 (bf16 widens by a 16-bit shift)
__device__ __forceinline__ float2 to_f2(float2 v) { return v; }
__device__ __forceinline__ float2 to_f2(uint32_t v) {
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

// Two fp32 values in one 64-bit register pair, for the packed f32x2 arithmetic of sm_100
// (both halves rounded as the scalar instruction would round them)
typedef unsigned long long f2x;
__device__ __forceinline__ f2x pk2(float lo, float hi) {
  f2x r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 up2(f2x v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ f2x fma2(f2x a, f2x b, f2x c) {
  f2x d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f2x mul2(f2x a, f2x b) {
  f2x d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2x sub2(f2x a, f2x b) {
  f2x d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// a pair rounded to tf32 / bf16 and stored (shared memory by 32-bit address, or global)
__device__ __forceinline__ void st_tf32p(uint32_t saddr, f2x v) {
  const float2 t = up2(v);
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(saddr), "f"(tf32_rna(t.x)),
               "f"(tf32_rna(t.y))
               : "memory");
}
__device__ __forceinline__ void st_bf16p(uint32_t saddr, f2x v) {
  const float2 t = up2(v);
  const __nv_bfloat162 b = __floats2bfloat162_rn(t.x, t.y);
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(saddr), "r"(*reinterpret_cast<const uint32_t*>(&b))
               : "memory");
}
__device__ __forceinline__ void st_shared_b32(uint32_t saddr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(saddr), "r"(v) : "memory");
}
__device__ __forceinline__ f2x ld_shared_f2x(uint32_t saddr) {
  f2x v;
  asm volatile("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(saddr) : "memory");
  return v;
}


// The pass on CTA `cta` of `ncta` working CTAs.  Tile n is (slot n / H, head n % H): the
// tiles in flight at once cover the same tokens of all heads (neighbouring rows of x in
// HBM), and every head's chunks complete in order.  When the pass shares the launch with
// the inter-chunk chains (COSCHED), each tile's word in `flags` is set once all of it has
// been written.
template <bool FUSED, bool COSCHED>
__device__ __forceinline__ void intra_body(const PrefillArgs& a, const int cta, const int ncta,
                                           int* flags) {
  extern __shared__ __align__(1024) unsigned char smraw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sb = smem_u32(sm);
  __shared__ float bs[2][C];       // beta of the tile in flight and of the next one
  __shared__ float qsum[4][D];     // gate pass: per-16-row-group totals of the log decay
  __shared__ float4 pnorm[8][2][2];   // q/k sums of squares of a row pair: [group][parity][half]
  __shared__ uint32_t tmem_holder;
  __shared__ __align__(8) uint64_t bar_mma;
  __shared__ volatile int abort_flag;

  const int H = a.H, nslots = a.L.nslots;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto head_of = [&](int n) { return n % H; };
  auto slot_of = [&](int n) { return n / H; };
  int* status = reinterpret_cast<int*>(a.ws + a.L.status);

  // once per CTA: the MMA barrier and 128 TMEM columns, kept across tiles
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;
  int issued = 0;   // MMA batches committed by thread 0 (two per tile)

  // Persistent: tiles strided over the working CTAs.  Each iteration
  // runs the row pass of the tile in flight on all 16 warps; then warps 0-7 take its serial
  // tail (key gram readout, solve, W/U~) while warps 8-15 look up this CTA's next tile and run
  // its gate pass, whose G and beta the next row pass and tail read, and warps 12-15 read M.
  const int ntiles = nslots * H;
  __shared__ int next_meta[8];   // the next tile: index (-1: none), seq, start, end, t0, len, chunk, state row
  const int pr = warp & 7, hh = warp >> 3;
  const int c2 = 64 * hh + 2 * lane;   // row pass: warps w and w + 8 share rows 8(w%8)..+7
  // ---- the log decay of tile n, its running sum G over the chunk (log2 units: G log2 e)
  // and beta, by warps 8-15 (256 threads: channels gp, gp+1 of rows 16 gq .. 16 gq + 15) ----
  auto gate_pass = [&](int n, const TileRange& nt, int nbuf) {
    const int gt = tid - 256, gp = 2 * (gt & 63), gq = gt >> 6;
    const int nh = head_of(n), ns = slot_of(n);
    using GRawT = typename std::conditional<FUSED, uint32_t, float2>::type;   // 2 channels as loaded
    GRawT graw[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      graw[i] = GRawT{};
      if (16 * gq + i < nt.len) {
        const size_t idx = ((size_t)(nt.t0 + 16 * gq + i) * H + nh) * D + gp;
        graw[i] = FUSED ? *reinterpret_cast<const GRawT*>(static_cast<const __nv_bfloat16*>(a.f) + idx)
                        : *reinterpret_cast<const GRawT*>(a.loga + idx);
      }
    }
    float A_log_h = 0.f;
    float2 dtb = make_float2(0.f, 0.f);
    if (FUSED) {
      A_log_h = __ldg(a.A_log + nh);
      dtb = *reinterpret_cast<const float2*>(a.dt_bias + (size_t)nh * D + gp);
    }
    // while the loads are in flight: pull into L2 the inputs of the tile after this one,
    // 128-byte lines spread over the threads
    {
      const int nid = n + ncta;
      if (nid < ntiles) {
        const int nnh = head_of(nid), nns = slot_of(nid);
        // same sequence (slots of a sequence are consecutive): no search
        const int nc = nt.chunk + (nns - ns);
        TileRange ft;
        if (nc >= 0 && (long long)nc * C < nt.end - nt.start) {
          ft = nt;
          ft.chunk = nc;
          ft.t0 = nt.start + nc * C;
          ft.len = min(C, nt.end - ft.t0);
        } else {
          ft = slot_to_tile(a.cu, a.n_seqs, a.total, C, nns);
        }
        const int w0 = max(ft.start, ft.t0 - (KC - 1));      // window rows inside the sequence
        const int nrow = ft.t0 + ft.len - w0;
        // per row: x (FUSED: 6 lines) or q, k, v (12 lines), then f or log a (2 or 4 lines)
        const int lx = FUSED ? 6 : 12, lg = FUSED ? 2 : 4, per = lx + lg;
        for (int e = gt; e < nrow * per; e += 256) {
          const int tok = w0 + e / per, l = e % per;
          const size_t row = (size_t)tok * H + nnh;
          const char* p;
          if (l < lx) {
            if (FUSED) p = reinterpret_cast<const char*>(static_cast<const __nv_bfloat16*>(a.x) + row * 3 * D) + 128 * l;
            else p = reinterpret_cast<const char*>((l < 4 ? a.q : l < 8 ? a.k : a.v) + row * D) + 128 * (l & 3);
          } else {
            if (tok < ft.t0) continue;                         // no gates for window rows
            p = FUSED ? reinterpret_cast<const char*>(static_cast<const __nv_bfloat16*>(a.f) + row * D) + 128 * (l - lx)
                      : reinterpret_cast<const char*>(a.loga + row * D) + 128 * (l - lx);
          }
          asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
        }
      }
    }
    float g0[16], g1[16];
    if (FUSED) {
      // log2 a = lb log2(e) sigmoid(exp(A_log) (f + dt_bias))
      const float Ah2 = expf(A_log_h) * LOG2E, lb2 = a.lb * LOG2E;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const bool live = 16 * gq + i < nt.len;
        const float2 v = to_f2(graw[i]);
        g0[i] = live ? lb2 * sigmoid2(Ah2 * (v.x + dtb.x)) : 0.f;
        g1[i] = live ? lb2 * sigmoid2(Ah2 * (v.y + dtb.y)) : 0.f;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 v = to_f2(graw[i]);
        g0[i] = v.x * LOG2E;
        g1[i] = v.y * LOG2E;
      }
    }
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      g0[i] += g0[i - 1];
      g1[i] += g1[i - 1];
    }
    qsum[gq][gp] = g0[15];
    qsum[gq][gp + 1] = g1[15];
    if (gt < C) {
      float bv = 0.f;
      if (gt < nt.len) {
        const size_t bi = (size_t)(nt.t0 + gt) * H + nh;
        bv = FUSED ? sigmoid2(LOG2E * ld1(static_cast<const __nv_bfloat16*>(a.beta_logit) + bi))
                   : __ldg(a.beta + bi);
      }
      bs[nbuf][gt] = bv;
    }
    asm volatile("bar.sync 10, 256;" ::: "memory");   // warps 8-15
    float o0 = 0.f, o1 = 0.f;
#pragma unroll
    for (int q = 0; q < 3; ++q)
      if (q < gq) {
        o0 += qsum[q][gp];
        o1 += qsum[q][gp + 1];
      }
    float* G = reinterpret_cast<float*>(sm + OFF_G);
#pragma unroll
    for (int i = 0; i < 16; ++i)
      *reinterpret_cast<float2*>(G + (16 * gq + i) * D + gp) = make_float2(g0[i] + o0, g1[i] + o1);
    if (gq == 3) {
      float* gCo = reinterpret_cast<float*>(a.ws + a.L.gC) + ((size_t)ns * H + nh) * D;
      *reinterpret_cast<float2*>(gCo + gp) = make_float2(ex2a(g0[15] + o0), ex2a(g1[15] + o1));
    }
  };

  int tl = -1, buf = 0;   // tile in flight (-1: none yet) and its beta buffer
  TileRange tr{};
  int prow = -1;
#pragma unroll 1
  while (true) {
  const int h = tl >= 0 ? head_of(tl) : 0, slot = tl >= 0 ? slot_of(tl) : 0;
  const size_t tile = (size_t)slot * H + h;
  __nv_bfloat16* Wo = reinterpret_cast<__nv_bfloat16*>(a.ws + a.L.W) + tile * C * D;
  __nv_bfloat16* Uo = reinterpret_cast<__nv_bfloat16*>(a.ws + a.L.Ut) + tile * C * D;
  __nv_bfloat16* Qo = reinterpret_cast<__nv_bfloat16*>(a.ws + a.L.Qt) + tile * C * D;
  __nv_bfloat16* Ko = reinterpret_cast<__nv_bfloat16*>(a.ws + a.L.Kp) + tile * C * D;
  __nv_bfloat16* Mo = reinterpret_cast<__nv_bfloat16*>(a.ws + a.L.M) + tile * C * C;
  float* G = reinterpret_cast<float*>(sm + OFF_G);
  float* Af = reinterpret_cast<float*>(sm + OFF_GB);   // [64][AF_LD], once the gram is done
  float* Xs = reinterpret_cast<float*>(sm + OFF_XS);
  const float* bsb = bs[buf];
  const int L = tr.len, t0 = tr.t0;

  if (tl >= 0) {
  // ---- inputs of the token-row pass (kept as loaded, converted after).  Warp w < 8 holds
  // channels 0-63 and w >= 8 channels 64-127 of q, k and v, two per lane.
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.x);
  const __nv_bfloat16* cs = static_cast<const __nv_bfloat16*>(a.conv_state);
  using RawT = typename std::conditional<FUSED, uint32_t, float2>::type;   // 2 channels as loaded
  // fused prep state: conv taps (one float4 per channel) and the K-1 previous pre-conv rows
  float4 cw[3][2];
  RawT winr[KC - 1][3];
  if (FUSED) {
#pragma unroll
    for (int sgm = 0; sgm < 3; ++sgm)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        cw[sgm][j] = __ldg(reinterpret_cast<const float4*>(
            a.conv_w + ((size_t)h * 3 * D + sgm * D + c2 + j) * KC));
#pragma unroll
    for (int m = 0; m < KC - 1; ++m) {
      const int tok = t0 + 8 * pr - (KC - 1) + m;
      const __nv_bfloat16* src = nullptr;
      if (tok >= tr.start && tok < tr.end)   // rows past the end only feed padded rows
        src = x + ((size_t)tok * H + h) * 3 * D;
      else if (tok < tr.start && cs != nullptr)
        src = cs + (((size_t)prow * (KC - 1) + (KC - 1 + tok - tr.start)) * H + h) * 3 * D;
#pragma unroll
      for (int sgm = 0; sgm < 3; ++sgm)
        winr[m][sgm] = src ? *reinterpret_cast<const RawT*>(src + sgm * D + c2) : RawT{};
    }
  }
  // row r's q, k, v channels c2, c2+1 (pre-conv x when fused); zero past the sequence end
  auto load_row = [&](int r, RawT& iq, RawT& ik, RawT& iv) {
    iq = ik = iv = RawT{};
    if (r < L) {
      if (FUSED) {
        const __nv_bfloat16* xp = x + ((size_t)(t0 + r) * H + h) * 3 * D;
        iq = *reinterpret_cast<const RawT*>(xp + c2);
        ik = *reinterpret_cast<const RawT*>(xp + D + c2);
        iv = *reinterpret_cast<const RawT*>(xp + 2 * D + c2);
      } else {
        const size_t idx = ((size_t)(t0 + r) * H + h) * D + c2;
        iq = *reinterpret_cast<const RawT*>(a.q + idx);
        ik = *reinterpret_cast<const RawT*>(a.k + idx);
        iv = *reinterpret_cast<const RawT*>(a.v + idx);
      }
    }
  };
  // the first row pair in flight too (rows are processed in pairs, one pair ahead)
  RawT aq, ak, av, bq, bk, bv;
  load_row(8 * pr, aq, ak, av);
  load_row(8 * pr + 1, bq, bk, bv);

  // ---- token rows, in pairs: (prep), operands for the MMAs, Q~ and K' ----
  // A lane's two channels travel as one packed pair through the f32x2 arithmetic.
  {
    // q, k and v leave the conv scaled by log2 e (taps pre-scaled): the L2 norm of q and k
    // cancels the factor (with eps scaled alike) and v takes ln 2 back
    const float qsc = a.q_scale, inv_eps = 1.0f / (a.l2_eps * LOG2E);
    f2x cwp[3][KC];       // conv taps of channels c2, c2+1 per segment (q, k, v), oldest tap first
    f2x win[KC - 1][3];   // previous pre-conv rows, oldest first, per segment
    if (FUSED) {
#pragma unroll
      for (int sgm = 0; sgm < 3; ++sgm) {
        const float4 w0 = cw[sgm][0], w1 = cw[sgm][1];
        cwp[sgm][0] = pk2(LOG2E * w0.x, LOG2E * w1.x);
        cwp[sgm][1] = pk2(LOG2E * w0.y, LOG2E * w1.y);
        cwp[sgm][2] = pk2(LOG2E * w0.z, LOG2E * w1.z);
        cwp[sgm][3] = pk2(LOG2E * w0.w, LOG2E * w1.w);
      }
#pragma unroll
      for (int m = 0; m < KC - 1; ++m)
#pragma unroll
        for (int sgm = 0; sgm < 3; ++sgm) {
          const float2 t = to_f2(winr[m][sgm]);
          win[m][sgm] = pk2(t.x, t.y);
        }
    }
    // reference rows of the exponent split: row 15 for rows 0-31, row 47 for rows 32-63
    const f2x R15 = *reinterpret_cast<const f2x*>(G + 15 * D + c2);
    const f2x R47 = *reinterpret_cast<const f2x*>(G + 47 * D + c2);
    const float2 r47 = up2(R47), r63 = *reinterpret_cast<const float2*>(G + 63 * D + c2);
    const bool lowhalf = pr < 4;
    const f2x RREF = lowhalf ? R15 : R47;
    // 2^{G_15} and 2^{G_63 - G_47}: each spans at most 16 steps of the decay (lb >= -5), so
    // both are >= 2^-116, normal fp32 numbers
    const float2 r15 = up2(R15);
    const f2x E15 = pk2(ex2a(r15.x), ex2a(r15.y));
    const f2x C6347 = pk2(ex2a(r63.x - r47.x), ex2a(r63.y - r47.y));
    const f2x LN2_2 = pk2(LN2, LN2), HALF2 = pk2(0.5f, 0.5f), HLN2_2 = pk2(0.5f * LN2, 0.5f * LN2);
    // shared-memory addresses: the per-thread part here, a row adds j * 128 and the swizzle
    // of j = row & 7 (row = 8 pr + j).  Gram rows: a key at B row r (rows 0-31) or r + 32,
    // its query 32 rows further; the column-scaled key at A row r (rows 0-31) and r + 32.
    const int gq = (c2 & 31) >> 2, mq = (c2 & 63) >> 3;
    const uint32_t gA = sb + OFF_GA + (c2 >> 5) * 16384 + (c2 & 3) * 4 + pr * 1024;
    const uint32_t gB = sb + OFF_GB + (c2 >> 5) * 16384 + (c2 & 3) * 4 + pr * 1024 +
                        (lowhalf ? 0 : 4096);
    const uint32_t mB = sb + (c2 >> 6) * 8192 + pr * 1024 + (c2 & 7) * 2;
    const uint32_t Grow = sb + OFF_G + (uint32_t)(8 * pr * D + c2) * 4;

    // depthwise conv (taps 0..K-2 on the window, K-1 on the row) and SiLU of one row;
    // the row then enters the window.  Returns the partial sums of squares of q and k.
    auto conv_row = [&](RawT iq, RawT ik, RawT iv, f2x& qv, f2x& kv, f2x& vv) -> float2 {
      if (!FUSED) {
        const float2 fq = to_f2(iq), fk = to_f2(ik), fv = to_f2(iv);
        qv = pk2(qsc * fq.x, qsc * fq.y);
        kv = pk2(fk.x, fk.y);
        vv = pk2(fv.x, fv.y);
        return make_float2(0.f, 0.f);
      }
      const RawT raw[3] = {iq, ik, iv};
      f2x z[3];
#pragma unroll
      for (int sgm = 0; sgm < 3; ++sgm) {
        const float2 xf = to_f2(raw[sgm]);
        const f2x x = pk2(xf.x, xf.y);
        f2x acc = mul2(cwp[sgm][KC - 1], x);
        acc = fma2(cwp[sgm][0], win[0][sgm], acc);
        acc = fma2(cwp[sgm][1], win[1][sgm], acc);
        acc = fma2(cwp[sgm][2], win[2][sgm], acc);
        // SiLU in log2 units: acc sigma(acc ln 2), sigma(x) = (1 + tanh(x / 2)) / 2 (one
        // special-function op; its error, within 2^-11 of tanh, is far inside the bf16
        // tiles' rounding)
        const f2x hacc = mul2(acc, HALF2);
        const float2 sh = up2(mul2(acc, HLN2_2));
        z[sgm] = fma2(hacc, pk2(tanha(sh.x), tanha(sh.y)), hacc);
        win[0][sgm] = win[1][sgm];
        win[1][sgm] = win[2][sgm];
        win[2][sgm] = x;
      }
      qv = z[0];
      kv = z[1];
      vv = mul2(z[2], LN2_2);
      const float2 q2 = up2(z[0]), k2 = up2(z[1]);
      return make_float2(fmaf(q2.x, q2.x, q2.y * q2.y), fmaf(k2.x, k2.x, k2.y * k2.y));
    };
    // every operand of token row 8 pr + j for this lane's two channels
    auto operands = [&](int j, f2x qv, f2x kv, f2x vv) {
      const f2x gr = ld_shared_f2x(Grow + j * D * 4);
      // er = 2^{G_r - G_ref} and its reciprocal: |exponent| <= 80 log2 e, both in range
      const float2 d = up2(sub2(gr, RREF));
      const float er0 = ex2a(d.x), er1 = ex2a(d.y);
      const f2x er = pk2(er0, er1), ei = pk2(rcpa(er0), rcpa(er1));
      const f2x kb = mul2(kv, er), qb = mul2(qv, er);
      f2x kc1, eg;   // k 2^{G_47 - G_r} and 2^{G_r}
      if (lowhalf) {
        const float2 d1 = up2(sub2(R47, gr));
        kc1 = mul2(kv, pk2(ex2a(d1.x), ex2a(d1.y)));
        eg = mul2(E15, er);   // 2^{G_15} 2^{G_r - G_15}; below 2^-126 it flushes to 0
      } else {
        kc1 = mul2(kv, ei);
        const float2 g = up2(gr);
        eg = pk2(ex2a(g.x), ex2a(g.y));
      }
      const f2x qt = mul2(qv, eg), kt = mul2(kv, eg);
      const f2x kp = mul2(kc1, C6347);   // k 2^{G_63 - G_r}
      const int jo = j * 128 + (((gq ^ j) & 7) << 4);
      st_tf32p(gB + jo, kb);
      st_tf32p(gB + jo + 4096, qb);
      if (lowhalf) st_tf32p(gA + jo, mul2(kv, ei));   // k 2^{G_15 - G_r}
      st_tf32p(gA + jo + 4096, kc1);
      const uint32_t mp = mB + j * 128 + (((mq ^ j) & 7) << 4);
      const float2 ktf = up2(kt);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(ktf.x, ktf.y);
      const float2 hf = __bfloat1622float2(hi);
      st_shared_b32(mp + OFF_KT, *reinterpret_cast<const uint32_t*>(&hi));
      st_bf16p(mp + OFF_KL, sub2(kt, pk2(hf.x, hf.y)));
      st_bf16p(mp + OFF_VT, vv);
      const float2 qtf = up2(qt), kpf = up2(kp);
      st_bf16x2(Qo + (size_t)(8 * pr + j) * D + c2, qtf.x, qtf.y);
      st_bf16x2(Ko + (size_t)(8 * pr + j) * D + c2, kpf.x, kpf.y);
    };

#pragma unroll 1
    for (int k = 0; k < 4; ++k) {
      const int ra = 8 * pr + 2 * k, rb = ra + 1;
      RawT nq0, nk0, nv0, nq1, nk1, nv1;   // the next pair, in flight through this one
      load_row(k < 3 ? ra + 2 : C, nq0, nk0, nv0);
      load_row(k < 3 ? ra + 3 : C, nq1, nk1, nv1);
      f2x qa, ka, va, qb2, kb2, vb2;
      const float2 sa = conv_row(aq, ak, av, qa, ka, va);
      const float2 sb = conv_row(bq, bk, bv, qb2, kb2, vb2);
      if (FUSED) {
        // q and k norms over 128 channels: the four sums of this warp's 64 channels by a
        // reduce-scatter over the lanes (lane 8v ends with sum v), then the partner warp's
        const bool b4 = lane & 16, b3 = lane & 8;
        float k0 = b4 ? sb.x : sa.x, k1 = b4 ? sb.y : sa.y;
        k0 += __shfl_xor_sync(0xffffffffu, b4 ? sa.x : sb.x, 16);
        k1 += __shfl_xor_sync(0xffffffffu, b4 ? sa.y : sb.y, 16);
        float m = (b3 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, b3 ? k0 : k1, 8);
        m += __shfl_xor_sync(0xffffffffu, m, 4);
        m += __shfl_xor_sync(0xffffffffu, m, 2);
        m += __shfl_xor_sync(0xffffffffu, m, 1);
        if ((lane & 7) == 0) reinterpret_cast<float*>(&pnorm[pr][k & 1][hh])[lane >> 3] = m;
        asm volatile("bar.sync %0, 64;" ::"r"(1 + pr) : "memory");
        const float4 o0 = pnorm[pr][k & 1][0], o1 = pnorm[pr][k & 1][1];
        const float4 part = make_float4(o0.x + o1.x, o0.y + o1.y, o0.z + o1.z, o0.w + o1.w);
        // 1 / max(||x||, eps) = min(rsqrt(||x||^2), 1 / eps), rsqrt(0) = inf; q_scale folded
        const float iqa = ra < L ? qsc * fminf(rsqrta(part.x), inv_eps) : 0.f;
        const float ika = ra < L ? fminf(rsqrta(part.y), inv_eps) : 0.f;
        const float iqb = rb < L ? qsc * fminf(rsqrta(part.z), inv_eps) : 0.f;
        const float ikb = rb < L ? fminf(rsqrta(part.w), inv_eps) : 0.f;
        qa = mul2(qa, pk2(iqa, iqa));
        ka = mul2(ka, pk2(ika, ika));
        qb2 = mul2(qb2, pk2(iqb, iqb));
        kb2 = mul2(kb2, pk2(ikb, ikb));
        if (ra >= L) va = 0ull;
        if (rb >= L) vb2 = 0ull;
      }
      operands(2 * k, qa, ka, va);
      operands(2 * k + 1, qb2, kb2, vb2);
      aq = nq0; ak = nk0; av = nv0;
      bq = nq1; bk = nk1; bv = nv1;
    }
  }
  fence_proxy_async();
  __syncthreads();

  if (tid == 0) {
    tc_fence_after();
    const uint32_t id = idesc_tf32(128, 128);
#pragma unroll
    for (int s = 0; s < 16; ++s)
      umma_tf32(tmem, sw128_desc(sb + OFF_GA + (s >> 2) * 16384 + (s & 3) * 32),
                sw128_desc(sb + OFF_GB + (s >> 2) * 16384 + (s & 3) * 32), id, s > 0);
    umma_commit(smem_u32(&bar_mma));
    ++issued;
  }

  }   // row pass

  if (warp < 8) {
  if (tl >= 0) {
  bool ok = mbar_wait_warp(smem_u32(&bar_mma), 0, &abort_flag);
  tc_fence_after();
  asm volatile("bar.sync 11, 256;" ::: "memory");   // warps 0-7
  // D[m][n]: rows 0-31 = keys 0-31 vs cols 0-31 (keys) / 32-63 (queries) of rows 0-31;
  // rows 32-95 = keys 0-63 vs cols 64-95 (keys) / 96-127 (queries) of rows 32-63.
  // Warps 0-2 (lane quarters 0-2) read the key columns of their quarter into A; warps
  // 12-14 read the query columns (M) later, and quarter 3 (rows 96-127 of D) holds nothing.
  if (ok && warp < 3) {   // the keys (A); the queries (M) are read by warps 12-15
    const int q = warp;
    const int i = (q == 2) ? 32 + lane : lane;          // key index of this TMEM lane
    const int rbase = (q == 0) ? 0 : 32;                 // first row r of the group
    const uint32_t col = (q == 0) ? 0u : 64u;
    float v[32];
    tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + col, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int r = rbase + j;
      if (i < r) Af[r * AF_LD + i] = bsb[r] * v[j];
    }
  }
  tc_fence_before();
  // the diagonal blocks of A come from warps 0 and 2: the substitution below (warps 0-1)
  // starts once warps 0-2 are done
  if (warp < 3) asm volatile("bar.sync 9, 96;" ::: "memory");

  // ---- T = (I + A)^{-1} diag(b), with A strictly lower triangular, by 16 x 16 blocks ----
  // X = (I + A)^{-1}: the four diagonal blocks by forward substitution (one thread per
  // column), then the blocks below (X_ab = -X_aa sum_{k=b}^{a-1} A_ak X_kb for a > b),
  // organised as two levels of 32 x 32 doubling
  if (tid < 64) {
    // right-looking: once x_i is final it goes into every later row's sum, so the chain
    // from one row to the next is one FMA; each x_r still sums its terms in order of i
    const int b = tid >> 4, jj = tid & 15;
    const float* Ab = Af + (16 * b) * AF_LD + 16 * b;
    float xc[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) xc[r] = (r == jj) ? 1.f : 0.f;
#pragma unroll
    for (int i = 0; i < 15; ++i)
#pragma unroll
      for (int r = i + 1; r < 16; ++r) xc[r] = fmaf(-Ab[r * AF_LD + i], xc[i], xc[r]);
#pragma unroll
    for (int r = 0; r < 16; ++r) Xs[(16 * b + r) * AF_LD + 16 * b + jj] = xc[r];
  }
  asm volatile("bar.sync 11, 256;" ::: "memory");
  {
    // Below the diagonal in two levels (m16n8k8 tf32 tensor-core products split three
    // ways, hi.hi + hi.lo + lo.hi ~ fp32; one warp per 16 x 8 output tile):
    //  1. inside each 32-row half: X_10 = -X_11 (A_10 X_00), X_32 = -X_33 (A_32 X_22)
    //  2. the lower-left 32 x 32 block: X_BA = -X_BB (A_BA X_AA), A = rows/cols 0-31,
    //     B = rows/cols 32-63, through Z = A_BA X_AA
    const int g = lane >> 2, t = lane & 3;
    float* Zw = reinterpret_cast<float*>(sm + OFF_ZS) + warp * 16 * ZW_LD;
    float* Z32 = reinterpret_cast<float*>(sm + OFF_ZS) + 4 * 16 * ZW_LD;   // [32][Z32_LD]
    if (warp < 4) {
      const int ab = 2 * (warp >> 1) + 1, bb = ab - 1, n0 = 16 * bb + 8 * (warp & 1);
      float z[3][4] = {};
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        mma3_tf32(z, Af + (16 * ab) * AF_LD + 16 * bb + 8 * ks, AF_LD,
                  Xs + (16 * bb + 8 * ks) * AF_LD + n0, AF_LD, g, t);
      Zw[g * ZW_LD + 2 * t] = sum3(z, 0);
      Zw[g * ZW_LD + 2 * t + 1] = sum3(z, 1);
      Zw[(g + 8) * ZW_LD + 2 * t] = sum3(z, 2);
      Zw[(g + 8) * ZW_LD + 2 * t + 1] = sum3(z, 3);
      __syncwarp();
      float y[3][4] = {};
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        mma3_tf32(y, Xs + (16 * ab) * AF_LD + 16 * ab + 8 * ks, AF_LD, Zw + (8 * ks) * ZW_LD,
                  ZW_LD, g, t);
      float* xo = Xs + (16 * ab + g) * AF_LD + n0 + 2 * t;
      xo[0] = -sum3(y, 0);
      xo[1] = -sum3(y, 1);
      xo[8 * AF_LD] = -sum3(y, 2);
      xo[8 * AF_LD + 1] = -sum3(y, 3);
    }
    asm volatile("bar.sync 11, 256;" ::: "memory");
    // warp w < 8: 16-row block i = w / 4 of B, 16-column block j of A, 8-column half
    const int bi = warp >> 2, bj = (warp >> 1) & 1, n0 = 16 * bj + 8 * (warp & 1);
    if (warp < 8) {   // Z_ij = sum_{k >= j} A_{2+i,k} X_kj
      float z[3][4] = {};
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (k >= bj) {
#pragma unroll
          for (int ks = 0; ks < 2; ++ks)
            mma3_tf32(z, Af + (32 + 16 * bi) * AF_LD + 16 * k + 8 * ks, AF_LD,
                      Xs + (16 * k + 8 * ks) * AF_LD + n0, AF_LD, g, t);
        }
      float* zo = Z32 + (16 * bi + g) * Z32_LD + n0 + 2 * t;
      zo[0] = sum3(z, 0);
      zo[1] = sum3(z, 1);
      zo[8 * Z32_LD] = sum3(z, 2);
      zo[8 * Z32_LD + 1] = sum3(z, 3);
    }
    asm volatile("bar.sync 11, 256;" ::: "memory");
    if (warp < 8) {   // X_{2+i,j} = -sum_{k <= i} X_{2+i,2+k} Z_kj
      float y[3][4] = {};
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (k <= bi) {
#pragma unroll
          for (int ks = 0; ks < 2; ++ks)
            mma3_tf32(y, Xs + (32 + 16 * bi) * AF_LD + 32 + 16 * k + 8 * ks, AF_LD,
                      Z32 + (16 * k + 8 * ks) * Z32_LD + n0, Z32_LD, g, t);
        }
      float* xo = Xs + (32 + 16 * bi + g) * AF_LD + n0 + 2 * t;
      xo[0] = -sum3(y, 0);
      xo[1] = -sum3(y, 1);
      xo[8 * AF_LD] = -sum3(y, 2);
      xo[8 * AF_LD + 1] = -sum3(y, 3);
    }
    asm volatile("bar.sync 11, 256;" ::: "memory");
  }
  // T[r][j] = X[r][j] b_j for j <= r (else 0), as bf16 high and low parts, K-major [r][j]
#pragma unroll
  for (int e = tid; e < C * 8; e += 256) {
    const int r = e >> 3, j0 = 8 * (e & 7);
    float hi[8], lo[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u;
      const float tv = (j <= r) ? Xs[r * AF_LD + j] * bsb[j] : 0.f;
      hi[u] = __bfloat162float(__float2bfloat16_rn(tv));
      lo[u] = tv - hi[u];
    }
    st_bf16x4(sm + OFF_T + sw128_off(r, j0), hi[0], hi[1], hi[2], hi[3]);
    st_bf16x4(sm + OFF_T + sw128_off(r, j0) + 8, hi[4], hi[5], hi[6], hi[7]);
    st_bf16x4(sm + OFF_TL + sw128_off(r, j0), lo[0], lo[1], lo[2], lo[3]);
    st_bf16x4(sm + OFF_TL + sw128_off(r, j0) + 8, lo[4], lo[5], lo[6], lo[7]);
  }
  fence_proxy_async();
  asm volatile("bar.sync 13, 384;" ::: "memory");   // warps 0-7 and 12-15 (M read from TMEM)

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
    ++issued;
  }
  if (ok) ok = mbar_wait_warp(smem_u32(&bar_mma), 1, &abort_flag);
  tc_fence_after();
  if (ok) {
    // warp w: TMEM lane quarter w % 4 (channels), W (w < 4) or U~ (w >= 4), all 64 tokens
    const int q = warp & 3;
    const int c = 32 * q + lane;
    const bool isW = warp < 4;
    __nv_bfloat16* dst = isW ? Wo : Uo;
#pragma unroll
    for (int part = 0; part < 4; ++part) {   // 16 token columns at a time
      float v[16];
      tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (isW ? 0u : 64u) + 16u * part, v);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        dst[(size_t)(16 * part + j) * D + c] = __float2bfloat16_rn(v[j]);
    }
  }
  }   // tail
  } else {
    // the next tile with work: one thread walks this CTA's tiles, the group reads the result
    if (warp == THREADS / 32 - 1 && lane == 0) {
      int n = tl < 0 ? cta : tl + ncta;
      TileRange nt{};
      int np = -1;
      for (; n < ntiles; n += ncta) {
        nt = slot_to_tile(a.cu, a.n_seqs, a.total, C, slot_of(n));
        np = nt.len ? pool_row(a.slots, nt.seq, a.pool_size) : -1;
        if (nt.len > 0 && np >= 0) break;
      }
      next_meta[0] = n < ntiles ? n : -1;
      next_meta[1] = nt.seq; next_meta[2] = nt.start; next_meta[3] = nt.end;
      next_meta[4] = nt.t0; next_meta[5] = nt.len; next_meta[6] = nt.chunk; next_meta[7] = np;
    }
    asm volatile("bar.sync 10, 256;" ::: "memory");   // warps 8-15
    const int n = next_meta[0];
    if (n >= 0) {
      TileRange nt;
      nt.seq = next_meta[1]; nt.start = next_meta[2]; nt.end = next_meta[3];
      nt.t0 = next_meta[4]; nt.len = next_meta[5]; nt.chunk = next_meta[6];
      gate_pass(n, nt, buf ^ 1);
    }
    // M of the tile in flight, before the W/U~ MMA reuses its TMEM columns: warps 12-14 read
    // the query columns of lane quarters 0-2; quarter 3 holds nothing and warp 15 writes the
    // zero upper-right block
    if (tl >= 0 && warp >= 12) {
      const bool okm = mbar_wait_warp(smem_u32(&bar_mma), 0, &abort_flag);
      tc_fence_after();
      const int q = warp & 3;
      if (okm && q < 3) {
        const int i = (q == 2) ? 32 + lane : lane;
        const int rbase = (q == 0) ? 0 : 32;
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + ((q == 0) ? 0u : 64u) + 32u, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int r = rbase + j;
          Mo[r * C + i] = __float2bfloat16_rn(i <= r ? v[j] : 0.f);
        }
      } else if (q == 3) {
#pragma unroll
        for (int j = 0; j < 32; ++j) Mo[j * C + 32 + lane] = __float2bfloat16_rn(0.f);
      }
      tc_fence_before();
      asm volatile("bar.sync 13, 384;" ::: "memory");   // with warps 0-7, before the W/U~ MMA
    }
  }

  tc_fence_before();
  __syncthreads();   // the tile's shared memory and TMEM are free; the next tile's G and beta are in place
  if (COSCHED && tid == 0 && tl >= 0 && !abort_flag) {
    // every write of the tile precedes the barrier: release them with its ready word
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(flags + tile), "r"(1) : "memory");
  }
  if (abort_flag) break;
  tl = next_meta[0];
  if (tl < 0) break;
  tr.seq = next_meta[1]; tr.start = next_meta[2]; tr.end = next_meta[3];
  tr.t0 = next_meta[4]; tr.len = next_meta[5]; tr.chunk = next_meta[6];
  prow = next_meta[7];
  buf ^= 1;
  }   // tiles

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


template <bool FUSED>
__global__ void __launch_bounds__(THREADS, 1) intra_chunk_sm100_kernel(const PrefillArgs a) {
  intra_body<FUSED, false>(a, blockIdx.x, gridDim.x, nullptr);
}

// One launch, two roles: CTAs 0 .. H-1 carry the inter-chunk chains (one per head, all
// value columns, walking the sequences of the batch in order), the others run the
// intra-chunk pass tile by tile in the same order and set each tile's ready word, which the
// chains wait for (bounded).  The intra-chunk role never waits for a chain, and the launch
// is cooperative (every CTA resident), so each wait ends.
template <bool FUSED>
__global__ void __launch_bounds__(THREADS, 1)
prefill_cosched_sm100_kernel(const PrefillArgs a, const __grid_constant__ ChainMaps maps,
                             const int nchain) {
  int* flags = reinterpret_cast<int*>(a.ws + a.L.flags);
  if ((int)blockIdx.x < nchain) chain::chain_body(a, maps, blockIdx.x, flags);
  else intra_body<FUSED, true>(a, (int)blockIdx.x - nchain, (int)gridDim.x - nchain, flags);
}

template <bool FUSED>
cudaError_t launch_cosched_t(const PrefillArgs& a, cudaStream_t st, bool* launched) {
  constexpr size_t smem = SMEM_BYTES > chain::SMEM_BYTES ? SMEM_BYTES : chain::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(prefill_cosched_sm100_kernel<FUSED>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  // A chain completes a chunk in about 0.27 of the intra-chunk pass's time per tile, so
  // the chains keep pace with the other SMs' production when H >= about a fifth of the
  // SMs; with fewer heads they would set the pace, with more than a quarter the pass
  // would lose too many SMs: the separate launches are faster in both cases.
  const int nchain = a.H;
  if (4 * nchain > nsm || 5 * nchain < nsm) return cudaSuccess;
  // a chain walks the batch's sequences one after another, paying a state read and write
  // at each boundary: with sequences of fewer than 4 chunks on average the chains would
  // set the pace, and the separate launches run them side by side instead
  if ((long long)a.total < 4LL * C * a.n_seqs) return cudaSuccess;
  ChainMaps maps;
  if (!make_chain_maps(a, &maps)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nsm, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, prefill_cosched_sm100_kernel<FUSED>, a, maps, nchain);
  if (e == cudaErrorCooperativeLaunchTooLarge) {   // not every CTA fits at once: two passes
    cudaGetLastError();
    return cudaSuccess;
  }
  if (e != cudaSuccess) return e;
  *launched = true;
  ++launch_counter();
  return cudaSuccess;
}

template <bool FUSED>
cudaError_t launch_intra_t(const PrefillArgs& a, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(intra_chunk_sm100_kernel<FUSED>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  // persistent: one CTA per SM (shared memory allows one), each looping over tiles
  const long long ntiles = (long long)a.L.nslots * a.H;
  const unsigned grid = (unsigned)(ntiles < nsm ? ntiles : nsm);
  if (grid == 0) return cudaSuccess;
  intra_chunk_sm100_kernel<FUSED><<<grid, THREADS, SMEM_BYTES, st>>>(a);
  ++launch_counter();
  return cudaGetLastError();
}

}  // namespace

// the exponent split of the gram needs the bounded gate (lb >= -5)
bool sm100_intra_supported(const PrefillArgs& a) {
  return a.bf16 && a.D == D && a.C == C && !a.gate_softplus;
}
bool sm100_fused_supported(const PrefillArgs& a) { return sm100_intra_supported(a) && a.K == KC; }

cudaError_t launch_intra_sm100(const PrefillArgs& a, cudaStream_t st) {
  return a.x ? launch_intra_t<true>(a, st) : launch_intra_t<false>(a, st);
}

cudaError_t launch_cosched_sm100(const PrefillArgs& a, cudaStream_t st, bool* launched) {
  *launched = false;
  if (!sm100_intra_supported(a) || a.y == nullptr || a.total == 0) return cudaSuccess;
  return a.x ? launch_cosched_t<true>(a, st, launched) : launch_cosched_t<false>(a, st, launched);
}

}  // namespace kda
