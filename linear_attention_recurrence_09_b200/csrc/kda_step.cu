// kda_decode / kda_verify / kda_rollback (and kda_layer_decode / kda_layer_verify, which
// run the prep of each token in the same kernel): the token-at-a-time path.
//
// The fused delta-net operator of llama.cpp PR #27754 (backends that
// have it skip the chunked graph for generation): per (sequence, head) the
// d x d fp32 state is read once, decayed along the key axis, reduced twice in
// the same pass (S^T k and S^T q), updated by a rank-1 write and stored once.
// Verify runs that step block_len times from one load of the state and writes
// the state after every step to a tape (speculative verify of a DFlash2 block,
// dflash-mlx issue #63); rollback is a copy out of that tape.  Or, in the manner
// of the tape-replay path that issue names for the GatedDeltaNet rollback, verify
// writes only what each step adds to the state: S_j = Diag(a_j) S_{j-1} + k_j u_j^T,
// so (k_j, u_j, a_j) is 3d floats per step instead of a d x d state, and rollback
// replays the L accepted steps from the live state with the very operations of the
// step (a multiply, then one fused multiply-add per element), which makes the
// replayed state bit-identical to the full tape's.
//
// HBM-bound: the state is 64 KB per head at d = 128, so one CTA per
// (head, sequence) keeps its whole state in registers (16 float4 per thread
// at 256 threads) with 16-byte coalesced loads and stores, and the two column
// reductions go through shared memory across the 8 row groups.
#include <type_traits>

#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {

template <int D>
struct StepShape {
  static constexpr int CG = D / 4;                                // column groups of 4
  static constexpr int RG = (256 / CG < D / 2) ? 256 / CG : D / 2;  // row groups
  static constexpr int ROWS = D / RG;                             // rows per thread (even)
  static constexpr int PAIRS = ROWS / 2;                          // row pairs per thread
  static constexpr int RV = ROWS % 4 == 0 ? 4 : 2;                // rows per staged load
  static constexpr int THREADS = CG * RG;
  static constexpr int NW = (THREADS + 31) / 32;
  // Row group rg holds the key rows rg, rg + RG, rg + 2 RG, ... (so the CTA's i-th state
  // load covers RG consecutive rows); the staged per-row vectors (q, k, a) are stored
  // permuted so that those ROWS rows sit at consecutive positions rg * ROWS + i.
  static __device__ __forceinline__ int pos(int r) { return (r % RG) * ROWS + r / RG; }
};

// sigmoid on the special-function unit (approximate exp and reciprocal, relative error
// ~1e-7); 1 / (1 + inf) = 0 keeps the saturated end exact
__device__ __forceinline__ float fsig(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }

// The state arrives as plain rows (every load issued before any of them is used)
template <int D, int ROWS>
__device__ __forceinline__ void rows_ld(float4 (&raw)[ROWS], const float* base, int rg, int c0) {
  constexpr int RG = D / ROWS;
#pragma unroll
  for (int i = 0; i < ROWS; ++i) raw[i] = ld4(base + (size_t)(rg + i * RG) * D + c0);
}

// RV consecutive entries of a staged d-vector in shared memory as RV / 2 row pairs
template <int RV>
__device__ __forceinline__ void pairs_ld(const float* p, float2 (&v)[RV / 2]) {
  if constexpr (RV == 4) {
    const float4 w = *reinterpret_cast<const float4*>(p);
    v[0] = make_float2(w.x, w.y);
    v[1] = make_float2(w.z, w.w);
  } else {
    v[0] = *reinterpret_cast<const float2*>(p);
  }
}

__device__ __forceinline__ float4 f4_scale(float4 a, float s) {
  return make_float4(a.x * s, a.y * s, a.z * s, a.w * s);
}
__device__ __forceinline__ float4 f4_fma(float s, float4 a, float4 acc) {
  return make_float4(fmaf(s, a.x, acc.x), fmaf(s, a.y, acc.y), fmaf(s, a.z, acc.z),
                     fmaf(s, a.w, acc.w));
}

// The two ways a thread holds its state tile, behind one interface.  Both accumulate a
// column's partial sums S^T k and S^T q in two chains (the thread's even-numbered rows,
// then its odd-numbered rows, added at the end) and update each element with the same
// two roundings (S a, then fma(k, u, .)), so the two give the same state and y bit for bit.
//  * PairedTile: pairs of rows, (S[r][c], S[r + RG][c]), for sm_100's paired fp32 multiply
//    and fused multiply-add (two lanes per instruction, each rounded to nearest like the
//    scalar instruction); the per-row factors of a pair come straight from one vector load
//    of the permuted staged vectors.  Fewest instructions: the verify blocks, whose steps
//    run back to back on chip.
//  * RowTile: rows as float4 with scalar arithmetic (fewest registers and moves; decode,
//    where a CTA runs one step and the state stream dominates).
template <int D>
struct PairedTile {
  using SH = StepShape<D>;
  static constexpr int ROWS = SH::ROWS, PAIRS = SH::PAIRS, RV = SH::RV, RG = SH::RG;
  float2 v[PAIRS][4];
  __device__ __forceinline__ void from_rows(const float4 (&raw)[ROWS]) {
#pragma unroll
    for (int p = 0; p < PAIRS; ++p) {
      const float4 x = raw[2 * p], y = raw[2 * p + 1];
      v[p][0] = make_float2(x.x, y.x);
      v[p][1] = make_float2(x.y, y.y);
      v[p][2] = make_float2(x.z, y.z);
      v[p][3] = make_float2(x.w, y.w);
    }
  }
  // S <- Diag(a) S on the thread's rows; returns the partial column sums of k^T S, q^T S
  __device__ __forceinline__ void decay_reduce(const float* k, const float* q, const float* a,
                                               float4& rk, float4& rq) {
    float2 pk[4], pq[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) pk[c] = pq[c] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i0 = 0; i0 < ROWS; i0 += RV) {
      float2 k2[RV / 2], q2[RV / 2], a2[RV / 2];
      pairs_ld<RV>(k + i0, k2);
      pairs_ld<RV>(q + i0, q2);
      pairs_ld<RV>(a + i0, a2);
#pragma unroll
      for (int j = 0; j < RV / 2; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float2& x = v[i0 / 2 + j][c];
          x = __fmul2_rn(x, a2[j]);
          pk[c] = __ffma2_rn(k2[j], x, pk[c]);
          pq[c] = __ffma2_rn(q2[j], x, pq[c]);
        }
    }
    rk = make_float4(pk[0].x + pk[0].y, pk[1].x + pk[1].y, pk[2].x + pk[2].y, pk[3].x + pk[3].y);
    rq = make_float4(pq[0].x + pq[0].y, pq[1].x + pq[1].y, pq[2].x + pq[2].y, pq[3].x + pq[3].y);
  }
  // S <- S + k u^T on the thread's rows and columns
  __device__ __forceinline__ void rank1(const float* k, float4 u) {
    const float2 u2[4] = {make_float2(u.x, u.x), make_float2(u.y, u.y), make_float2(u.z, u.z),
                          make_float2(u.w, u.w)};
#pragma unroll
    for (int i0 = 0; i0 < ROWS; i0 += RV) {
      float2 k2[RV / 2];
      pairs_ld<RV>(k + i0, k2);
#pragma unroll
      for (int j = 0; j < RV / 2; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) v[i0 / 2 + j][c] = __ffma2_rn(k2[j], u2[c], v[i0 / 2 + j][c]);
    }
  }
  __device__ __forceinline__ void store(float* base, int rg, int c0) const {
#pragma unroll
    for (int p = 0; p < PAIRS; ++p) {
      st4(base + (size_t)(rg + 2 * p * RG) * D + c0,
          make_float4(v[p][0].x, v[p][1].x, v[p][2].x, v[p][3].x));
      st4(base + (size_t)(rg + (2 * p + 1) * RG) * D + c0,
          make_float4(v[p][0].y, v[p][1].y, v[p][2].y, v[p][3].y));
    }
  }
};

template <int D>
struct RowTile {
  using SH = StepShape<D>;
  static constexpr int ROWS = SH::ROWS, RV = SH::RV, RG = SH::RG;
  float4 v[ROWS];
  __device__ __forceinline__ void from_rows(const float4 (&raw)[ROWS]) {
#pragma unroll
    for (int i = 0; i < ROWS; ++i) v[i] = raw[i];
  }
  __device__ __forceinline__ void decay_reduce(const float* k, const float* q, const float* a,
                                               float4& rk, float4& rq) {
    float4 pk[2], pq[2];          // [0]: even-numbered rows, [1]: odd-numbered rows
    pk[0] = pk[1] = pq[0] = pq[1] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i0 = 0; i0 < ROWS; i0 += RV) {
      float2 k2[RV / 2], q2[RV / 2], a2[RV / 2];
      pairs_ld<RV>(k + i0, k2);
      pairs_ld<RV>(q + i0, q2);
      pairs_ld<RV>(a + i0, a2);
#pragma unroll
      for (int j = 0; j < RV / 2; ++j) {
        float4& x = v[i0 + 2 * j];
        float4& y = v[i0 + 2 * j + 1];
        x = f4_scale(x, a2[j].x);
        y = f4_scale(y, a2[j].y);
        pk[0] = f4_fma(k2[j].x, x, pk[0]);
        pk[1] = f4_fma(k2[j].y, y, pk[1]);
        pq[0] = f4_fma(q2[j].x, x, pq[0]);
        pq[1] = f4_fma(q2[j].y, y, pq[1]);
      }
    }
    rk = make_float4(pk[0].x + pk[1].x, pk[0].y + pk[1].y, pk[0].z + pk[1].z, pk[0].w + pk[1].w);
    rq = make_float4(pq[0].x + pq[1].x, pq[0].y + pq[1].y, pq[0].z + pq[1].z, pq[0].w + pq[1].w);
  }
  __device__ __forceinline__ void rank1(const float* k, float4 u) {
#pragma unroll
    for (int i0 = 0; i0 < ROWS; i0 += RV) {
      float2 k2[RV / 2];
      pairs_ld<RV>(k + i0, k2);
#pragma unroll
      for (int j = 0; j < RV / 2; ++j) {
        v[i0 + 2 * j] = f4_fma(k2[j].x, u, v[i0 + 2 * j]);
        v[i0 + 2 * j + 1] = f4_fma(k2[j].y, u, v[i0 + 2 * j + 1]);
      }
    }
  }
  __device__ __forceinline__ void store(float* base, int rg, int c0) const {
#pragma unroll
    for (int i = 0; i < ROWS; ++i) st4(base + (size_t)(rg + i * RG) * D + c0, v[i]);
  }
};

// The T tokens' inputs are independent of the state, so they are made ready for every
// step first, in shared memory: loaded (kda_verify / kda_decode), or with the fused prep
// computed (kda_layer_*): the conv over the window [history; block] for every (token,
// channel) at once, SiLU, the gate, then the q / k L2 norms per token.  Also k . q per
// token.  Shared by the step kernels below; ends with a block barrier.
template <typename T, int D, bool PREP, int THREADS>
__device__ __forceinline__ void stage_inputs(const StepArgs& a, int b, int h, int row, float* qs,
                                             float* ks, float* vs, float* as_, float* gs,
                                             float* xwin, float* kq_s, float* beta_s) {
  using SH = StepShape<D>;
  constexpr int NW = THREADS / 32, C3 = 3 * D;
  const int H = a.H, Tn = a.T, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Km1 = PREP ? a.K - 1 : 0;
  T* csg = PREP ? static_cast<T*>(a.conv_state) : nullptr;
  T* wing = PREP ? static_cast<T*>(a.window) : nullptr;
  if (PREP) {
    // the window [history; x of the block] (history zeros without a conv state); verify
    // also writes it out for the rollback
    for (int e = tid; e < (Km1 + Tn) * C3; e += THREADS) {
      const int j = e / C3, c = e - j * C3;
      float v = 0.f;
      if (j < Km1) {
        if (csg) v = ld1(csg + (((size_t)row * Km1 + j) * H + h) * C3 + c);
      } else {
        v = ld1(static_cast<const T*>(a.x) + (((size_t)b * Tn + (j - Km1)) * H + h) * C3 + c);
      }
      xwin[e] = v;
      if (wing) st1(wing + (((size_t)b * (Km1 + Tn) + j) * H + h) * C3 + c, v);
    }
    const float Ah = __expf(__ldg(a.A_log + h));
    for (int e = tid; e < Tn * D; e += THREADS) {
      const int t = e / D, c = e - t * D;
      const size_t idx = (((size_t)b * Tn + t) * H + h) * D + c;
      const float z = ld1(static_cast<const T*>(a.f) + idx) + __ldg(a.dt_bias + (size_t)h * D + c);
      as_[t * D + SH::pos(c)] = __expf(a.gate_softplus ? -Ah * softplus(z) : a.lb * fsig(Ah * z));
      gs[e] = sigmoid(ld1(static_cast<const T*>(a.g) + idx));
    }
    for (int t = tid; t < Tn; t += THREADS)
      beta_s[t] = fsig(ld1(static_cast<const T*>(a.beta_logit) + ((size_t)b * Tn + t) * H + h));
    __syncthreads();
    // depthwise causal conv (tap K-1 = the token itself) + SiLU: each thread owns channels
    // (their taps loaded once, one 16-byte load when K = 4) and walks the block's tokens
    for (int c = tid; c < C3; c += THREADS) {
      const float* wp = a.conv_w + ((size_t)h * C3 + c) * a.K;
      float w[8];
      if (a.K == 4) {
        const float4 w4 = __ldg(reinterpret_cast<const float4*>(wp));
        w[0] = w4.x; w[1] = w4.y; w[2] = w4.z; w[3] = w4.w;
#pragma unroll
        for (int j = 4; j < 8; ++j) w[j] = 0.f;
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = (j < a.K) ? __ldg(wp + j) : 0.f;
      }
      const int part = c / D;
      const int cc = c - part * D;
      float* dst = part == 0 ? qs + SH::pos(cc) : part == 1 ? ks + SH::pos(cc) : vs + cc;
      for (int t = 0; t < Tn; ++t) {
        float acc = 0.f;
#pragma unroll
        for (int j = 7; j >= 0; --j)
          if (j <= Km1) acc = fmaf(w[j], xwin[(t + j) * C3 + c], acc);
        dst[t * D] = acc * fsig(acc);
      }
    }
    __syncthreads();
    // L2 norms of q and k per token: one warp per (token, q | k), scaled in place
    for (int pidx = warp; pidx < 2 * Tn; pidx += NW) {
      float* arr = ((pidx & 1) ? ks : qs) + (pidx >> 1) * D;
      float ss = 0.f;
      for (int c = lane; c < D; c += 32) ss = fmaf(arr[c], arr[c], ss);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      const float inv = 1.0f / fmaxf(sqrtf(ss), a.l2_eps);
      for (int c = lane; c < D; c += 32) arr[c] *= inv;
    }
  } else {
    for (int e = tid; e < Tn * D; e += THREADS) {
      const int t = e / D, c = e - t * D;
      const size_t idx = (((size_t)b * Tn + t) * H + h) * D + c;
      qs[t * D + SH::pos(c)] = __ldg(a.q + idx);
      ks[t * D + SH::pos(c)] = __ldg(a.k + idx);
      vs[e] = __ldg(a.v + idx);
      as_[t * D + SH::pos(c)] = expf(__ldg(a.loga + idx));
      gs[e] = sigmoid(ld1(static_cast<const T*>(a.g) + idx));
    }
    for (int t = tid; t < Tn; t += THREADS)
      beta_s[t] = __ldg(a.beta + ((size_t)b * Tn + t) * H + h);
  }
  __syncthreads();
  // k . q per token (lane-strided, then a butterfly: the decode kernels' order)
  for (int t = warp; t < Tn; t += NW) {
    float p = 0.f;
    for (int c = lane; c < D; c += 32) p = fmaf(ks[t * D + c], qs[t * D + c], p);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
    if (lane == 0) kq_s[t] = p;
  }
  __syncthreads();

}

// The conv-state commit of kda_layer_decode: the history ends with the block's tokens
// (the last K-1 rows of the window in shared memory)
template <typename T, int D, int THREADS>
__device__ __forceinline__ void commit_conv(const StepArgs& a, int h, int row, const float* xwin) {
  constexpr int C3 = 3 * D;
  const int Km1 = a.K - 1, H = a.H;
  T* csg = static_cast<T*>(a.conv_state);
  for (int e = threadIdx.x; e < Km1 * C3; e += THREADS) {
    const int j = e / C3, c = e - j * C3;
    st1(csg + (((size_t)row * Km1 + j) * H + h) * C3 + c, xwin[(a.T + j) * C3 + c]);
  }
}

// One CTA per (head, sequence), any d: the inputs of every step staged first, then the
// recurrence runs T steps on the state in registers with two block barriers per step.
template <typename T, int D, bool PREP, bool PAIRED>
__global__ void __launch_bounds__(StepShape<D>::THREADS, 2)
step_kernel(const StepArgs a) {
  using SH = StepShape<D>;
  using Tile = std::conditional_t<PAIRED, PairedTile<D>, RowTile<D>>;
  constexpr int CG = SH::CG, RG = SH::RG, ROWS = SH::ROWS;
  constexpr int THREADS = SH::THREADS, NW = SH::NW, TMAX = 16;
  extern __shared__ __align__(16) float dsm[];
  const int Tn = a.T;
  float* qs = dsm;                    // [T][D] normalised q
  float* ks = qs + Tn * D;            // [T][D] normalised k
  float* vs = ks + Tn * D;            // [T][D] v
  float* as_ = vs + Tn * D;           // [T][D] a = e^{log a}
  float* gs = as_ + Tn * D;           // [T][D] g
  float* xwin = gs + Tn * D;          // fused prep: [K-1+T][3d] pre-conv window
  __shared__ __align__(16) float us[D];
  __shared__ __align__(16) float redk[RG][D];
  __shared__ __align__(16) float redq[RG][D];
  __shared__ float ssq[NW], kq_s[TMAX], beta_s[TMAX];

  const int h = blockIdx.x, b = blockIdx.y;
  const int H = a.H;
  grid_dep_trigger();
  if (!a.early_state) grid_dep_wait();
  const int row = pool_row(a.slots, b, a.pool_size);
  if (row < 0) return;
  const int tid = threadIdx.x, cg = tid % CG, rg = tid / CG;
  const int lane = tid & 31, warp = tid >> 5;

  // the state streams in first: the inputs below are made ready while it arrives.  Row
  // group rg (a warp at d = 128) owns rows rg + i RG, lane cg the four columns from 4 cg:
  // every state load and store is a whole 512-byte row per warp, and the CTA's i-th load
  // covers RG consecutive rows.  s0: the first of the thread's staged positions.
  const int s0 = rg * ROWS, c0 = 4 * cg;
  const float* Sg = a.state_in + ((size_t)row * H + h) * D * D;
  Tile S;
  {
    float4 raw[ROWS];
    rows_ld<D>(raw, Sg, rg, c0);
    if (a.early_state) grid_dep_wait();    // the other inputs may come from the kernel before
    stage_inputs<T, D, PREP, THREADS>(a, b, h, row, qs, ks, vs, as_, gs, xwin, kq_s, beta_s);
    S.from_rows(raw);
  }
  const float nw = tid < D ? __ldg(a.norm_w + tid) : 0.f;
  for (int t = 0; t < Tn; ++t) {
    const size_t tok = (size_t)b * Tn + t;
    // decay along the key axis, then both column reductions in one pass
    float4 pk, pq;
    S.decay_reduce(ks + t * D + s0, qs + t * D + s0, as_ + t * D + s0, pk, pq);
    *reinterpret_cast<float4*>(&redk[rg][c0]) = pk;
    *reinterpret_cast<float4*>(&redq[rg][c0]) = pq;
    __syncthreads();                                       // (A) partial reductions

    // per value column: u = b (v - S^T k), o = S^T q + u (k.q), RMSNorm partials
    float o = 0.f;
    if (tid < D) {
      float rk = 0.f, rq = 0.f;
#pragma unroll
      for (int j = 0; j < RG; ++j) { rk += redk[j][tid]; rq += redq[j][tid]; }
      const float u = beta_s[t] * (vs[t * D + tid] - rk);
      o = a.q_scale * fmaf(u, kq_s[t], rq);
      us[tid] = u;
      if (a.tape_kua != nullptr) {   // compact tape: this step's k, u and a
        float* tk = a.tape_kua + (tok * H + h) * 3 * D;
        tk[tid] = ks[t * D + SH::pos(tid)];
        tk[D + tid] = u;
        tk[2 * D + tid] = as_[t * D + SH::pos(tid)];
      }
    }
    if (warp < (D + 31) / 32) {
      float p = o * o;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
      if (lane == 0) ssq[warp] = p;
    }
    __syncthreads();                                       // (B) u and the norm partials

    // rank-1 write and the gated RMSNorm epilogue.  The next step rewrites redk/redq, us
    // and ssq only after its barrier (A), which every thread reaches after these reads.
    S.rank1(ks + t * D + s0, *reinterpret_cast<const float4*>(&us[c0]));
    if (tid < D) {
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < (D + 31) / 32; ++w) ss += ssq[w];
      const float rstd = rsqrtf(ss / (float)D + a.norm_eps);
      st1(static_cast<T*>(a.y) + (tok * H + h) * D + tid, o * rstd * nw * gs[t * D + tid]);
    }
    if (a.tape != nullptr) S.store(a.tape + (tok * H + h) * D * D, rg, c0);
  }

  if (PREP && a.conv_state != nullptr && a.window == nullptr)
    commit_conv<T, D, THREADS>(a, h, row, xwin);
  if (a.state_out != nullptr) S.store(a.state_out + ((size_t)row * H + h) * D * D, rg, c0);
}

template <typename T, bool PREP, bool PAIRED>
static cudaError_t launch_step_p(const StepArgs& a, cudaStream_t st) {
  dim3 grid(a.H, a.B);
  const size_t smem =
      sizeof(float) * ((size_t)5 * a.T * a.D + (PREP ? (size_t)(a.K - 1 + a.T) * 3 * a.D : 0));
  cudaError_t e = cudaSuccess;
  switch (a.D) {
#define KDA_STEP_CASE(DD)                                                                     \
  case DD:                                                                                    \
    e = cudaFuncSetAttribute(step_kernel<T, DD, PREP, PAIRED>,                                \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);         \
    if (e != cudaSuccess) return e;                                                           \
    e = launch_dependent(step_kernel<T, DD, PREP, PAIRED>, grid,                              \
                         dim3(StepShape<DD>::THREADS), smem, st, a);                          \
    break;
    KDA_STEP_CASE(16)
    KDA_STEP_CASE(32)
    KDA_STEP_CASE(64)
    KDA_STEP_CASE(128)
#undef KDA_STEP_CASE
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  ++launch_counter();
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_step_t(const StepArgs& a, cudaStream_t st) {
  if (a.x != nullptr && (a.K < 1 || a.K > 8)) return cudaErrorInvalidValue;
  // one token (decode): the state tile in rows; a block (verify): in row pairs
  if (a.T == 1)
    return a.x ? launch_step_p<T, true, false>(a, st) : launch_step_p<T, false, false>(a, st);
  return a.x ? launch_step_p<T, true, true>(a, st) : launch_step_p<T, false, true>(a, st);
}

cudaError_t launch_step(const StepArgs& a, cudaStream_t st) {
  return a.bf16 ? launch_step_t<__nv_bfloat16>(a, st) : launch_step_t<float>(a, st);
}

// ---------------------------------------------------------------------------
// rollback: state <- tape[L-1], conv state <- window rows [L, L+K-1)
// ---------------------------------------------------------------------------
template <typename E>
__global__ void __launch_bounds__(256) rollback_kernel(const RollbackArgs a) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int L = clampi(__ldg(a.accepted + b), 0, a.T);
  if (L == 0) return;
  const int row = pool_row(a.slots, b, a.pool_size);
  if (row < 0) return;
  const int D = a.D, H = a.H;
  const float4* src = reinterpret_cast<const float4*>(a.tape + (((size_t)b * a.T + (L - 1)) * H + h) * D * D);
  float4* dst = reinterpret_cast<float4*>(a.state + ((size_t)row * H + h) * D * D);
  for (int i = threadIdx.x; i < D * D / 4; i += blockDim.x) dst[i] = src[i];
  if (a.conv_state != nullptr && a.window != nullptr) {
    const int Km1 = a.K - 1, C3 = 3 * D;
    const E* win = static_cast<const E*>(a.window);
    E* cs = static_cast<E*>(a.conv_state);
    for (int e = threadIdx.x; e < Km1 * C3; e += blockDim.x) {
      const int j = e / C3, c = e - (e / C3) * C3;
      cs[(((size_t)row * Km1 + j) * H + h) * C3 + c] =
          win[(((size_t)b * (Km1 + a.T) + L + j) * H + h) * C3 + c];
    }
  }
}

// ---------------------------------------------------------------------------
// rollback by replay: state <- the accepted steps of the compact tape applied to the
// live state, S <- Diag(a_j) S, then S <- S + k_j u_j^T, element by element with the
// step kernel's two roundings (S a, then fma(k, u, .)), so the result equals the full
// tape's entry bit for bit; conv state as in rollback_kernel.  Every element replays on
// its own, so a (head, sequence) state is split over CTAs of RPC key rows each, for
// more loads in flight than one CTA per state gives.
// ---------------------------------------------------------------------------
template <int D>
struct ReplayShape {
  static constexpr int RPC = D < 64 ? D : 64;                     // key rows per CTA
  static constexpr int SLICES = D / RPC;
  static constexpr int CG = D / 4;                                // column groups of 4
  static constexpr int RG = (256 / CG < RPC) ? 256 / CG : RPC;    // row groups
  static constexpr int ROWS = RPC / RG;                           // rows per thread
  static constexpr int THREADS = CG * RG;
};

template <typename E, int D>
__global__ void __launch_bounds__(ReplayShape<D>::THREADS) rollback_replay_kernel(const RollbackArgs a) {
  using RS = ReplayShape<D>;
  constexpr int CG = RS::CG, RG = RS::RG, ROWS = RS::ROWS, RPC = RS::RPC;
  constexpr int THREADS = RS::THREADS, TMAX = 16, PER = 2 * RPC + D;
  __shared__ __align__(16) float ks[TMAX][RPC];
  __shared__ __align__(16) float as_[TMAX][RPC];
  __shared__ __align__(16) float us[TMAX][D];
  const int h = blockIdx.x, b = blockIdx.y, r0 = blockIdx.z * RPC;
  grid_dep_trigger();
  if (!a.early_state) grid_dep_wait();
  const int row = pool_row(a.slots, b, a.pool_size);
  if (row < 0) return;
  const int H = a.H, tid = threadIdx.x, cg = tid % CG, rg = tid / CG, c0 = 4 * cg;
  float* Sg = a.state + ((size_t)row * H + h) * D * D;
  float4 S[ROWS];                  // key rows r0 + rg + i RG, columns c0..c0+3
  auto load_state = [&]() {
#pragma unroll
    for (int i = 0; i < ROWS; ++i) S[i] = ld4(Sg + (size_t)(r0 + rg + i * RG) * D + c0);
  };
  int L;
  if (a.early_state) {             // the state streams in while the kernel before finishes
    load_state();
    grid_dep_wait();
    L = clampi(__ldg(a.accepted + b), 0, a.T);
    if (L == 0) return;
  } else {
    L = clampi(__ldg(a.accepted + b), 0, a.T);
    if (L == 0) return;
    load_state();
  }
  // this CTA's k and a rows and every u column of the L accepted steps
  const float* tk = a.tape_kua + ((size_t)b * a.T * H + h) * 3 * D;   // + j H 3d: step j
  for (int e = tid; e < L * PER; e += THREADS) {
    const int j = e / PER, w = e - j * PER;
    const float* src = tk + (size_t)j * H * 3 * D;
    if (w < RPC) ks[j][w] = __ldg(src + r0 + w);
    else if (w < RPC + D) us[j][w - RPC] = __ldg(src + D + (w - RPC));
    else as_[j][w - RPC - D] = __ldg(src + 2 * D + r0 + (w - RPC - D));
  }
  __syncthreads();
  for (int j = 0; j < L; ++j) {
    const float4 u = *reinterpret_cast<const float4*>(&us[j][c0]);
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
      const int r = rg + i * RG;
      S[i] = f4_fma(ks[j][r], u, f4_scale(S[i], as_[j][r]));
    }
  }
#pragma unroll
  for (int i = 0; i < ROWS; ++i) st4(Sg + (size_t)(r0 + rg + i * RG) * D + c0, S[i]);
  if (blockIdx.z == 0 && a.conv_state != nullptr && a.window != nullptr) {
    const int Km1 = a.K - 1, C3 = 3 * D;
    const E* win = static_cast<const E*>(a.window);
    E* cs = static_cast<E*>(a.conv_state);
    for (int e = tid; e < Km1 * C3; e += THREADS) {
      const int j = e / C3, c = e - (e / C3) * C3;
      cs[(((size_t)row * Km1 + j) * H + h) * C3 + c] =
          win[(((size_t)b * (Km1 + a.T) + L + j) * H + h) * C3 + c];
    }
  }
}

template <typename E>
static cudaError_t launch_replay_e(const RollbackArgs& a, cudaStream_t st) {
  switch (a.D) {
#define KDA_REPLAY_CASE(DD)                                                                   \
  case DD:                                                                                    \
    return launch_dependent(rollback_replay_kernel<E, DD>,                                    \
                            dim3(a.H, a.B, ReplayShape<DD>::SLICES),                          \
                            dim3(ReplayShape<DD>::THREADS), 0, st, a);
    KDA_REPLAY_CASE(16)
    KDA_REPLAY_CASE(32)
    KDA_REPLAY_CASE(64)
    KDA_REPLAY_CASE(128)
#undef KDA_REPLAY_CASE
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_rollback(const RollbackArgs& a, cudaStream_t st) {
  dim3 grid(a.H, a.B);
  if (a.tape_kua != nullptr) {
    const cudaError_t e = a.bf16 ? launch_replay_e<uint16_t>(a, st) : launch_replay_e<uint32_t>(a, st);
    if (e != cudaSuccess) return e;
  } else if (a.bf16) {
    rollback_kernel<uint16_t><<<grid, 256, 0, st>>>(a);
  } else {
    rollback_kernel<uint32_t><<<grid, 256, 0, st>>>(a);
  }
  ++launch_counter();
  return cudaGetLastError();
}

}  // namespace kda
