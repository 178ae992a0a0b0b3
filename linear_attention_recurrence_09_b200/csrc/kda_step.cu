// kda_decode / kda_verify / kda_rollback (and kda_layer_decode / kda_layer_verify, which
// run the prep of each token in the same kernel): the token-at-a-time path.
//
// The "fused operator" for the delta net of llama.cpp PR #27754 (backends that
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
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {

template <int D>
struct StepShape {
  static constexpr int CG = D / 4;                                // column groups of 4
  static constexpr int RG = (256 / CG < D) ? 256 / CG : D;        // row groups
  static constexpr int ROWS = D / RG;                             // rows per thread
  static constexpr int THREADS = CG * RG;
  static constexpr int NW = (THREADS + 31) / 32;
};

// sigmoid on the special-function unit (approximate exp and reciprocal, relative error
// ~1e-7); 1 / (1 + inf) = 0 keeps the saturated end exact
__device__ __forceinline__ float fsig(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }

__device__ __forceinline__ uint32_t smem_u32_(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ float4 f4_scale(float4 a, float s) {
  return make_float4(a.x * s, a.y * s, a.z * s, a.w * s);
}
__device__ __forceinline__ float4 f4_fma(float s, float4 a, float4 acc) {
  return make_float4(fmaf(s, a.x, acc.x), fmaf(s, a.y, acc.y), fmaf(s, a.z, acc.z),
                     fmaf(s, a.w, acc.w));
}

// One CTA per (head, sequence): the T tokens' inputs are independent of the state, so they
// are made ready for every step first (loaded, or with the fused prep computed: the conv
// over the window [history; block] for every (token, channel) at once, SiLU, the gate,
// then the q / k L2 norms per token), and the recurrence then runs T steps on the state
// in registers with two block barriers per step.
template <typename T, int D, bool PREP>
__global__ void __launch_bounds__(StepShape<D>::THREADS)
step_kernel(const StepArgs a) {
  using SH = StepShape<D>;
  constexpr int CG = SH::CG, RG = SH::RG, ROWS = SH::ROWS, THREADS = SH::THREADS, NW = SH::NW;
  constexpr int TMAX = 16, C3 = 3 * D;
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
  const int row = pool_row(a.slots, b, a.pool_size);
  if (row < 0) return;
  const int tid = threadIdx.x, cg = tid % CG, rg = tid / CG;
  const int lane = tid & 31, warp = tid >> 5;

  // the state streams in first: the inputs below are made ready while it arrives
  const float* Sg = a.state_in + ((size_t)row * H + h) * D * D;
  float4 S[ROWS];
#pragma unroll
  for (int i = 0; i < ROWS; ++i) S[i] = ld4(Sg + (size_t)(rg + i * RG) * D + 4 * cg);

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
      as_[e] = __expf(a.gate_softplus ? -Ah * softplus(z) : a.lb * fsig(Ah * z));
      gs[e] = ld1(static_cast<const T*>(a.g) + idx);
    }
    for (int t = tid; t < Tn; t += THREADS)
      beta_s[t] = fsig(ld1(static_cast<const T*>(a.beta_logit) + ((size_t)b * Tn + t) * H + h));
    __syncthreads();
    // depthwise causal conv (tap K-1 = the token itself) + SiLU for every (token, channel)
    for (int e = tid; e < Tn * C3; e += THREADS) {
      const int t = e / C3, c = e - t * C3;
      const float* w = a.conv_w + ((size_t)h * C3 + c) * a.K;
      float acc = __ldg(w + Km1) * xwin[(t + Km1) * C3 + c];
      for (int j = Km1 - 1; j >= 0; --j) acc = fmaf(__ldg(w + j), xwin[(t + j) * C3 + c], acc);
      const float z = acc * fsig(acc);
      const int part = c / D;
      (part == 0 ? qs : part == 1 ? ks : vs)[t * D + (c - part * D)] = z;
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
      qs[e] = __ldg(a.q + idx);
      ks[e] = __ldg(a.k + idx);
      vs[e] = __ldg(a.v + idx);
      as_[e] = expf(__ldg(a.loga + idx));
      gs[e] = ld1(static_cast<const T*>(a.g) + idx);
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

  for (int t = 0; t < Tn; ++t) {
    const size_t tok = (size_t)b * Tn + t;
    const float* kt = ks + t * D;
    const float* qt = qs + t * D;
    const float* at = as_ + t * D;
    // decay along the key axis, then both column reductions in one pass
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
      const int r = rg + i * RG;
      S[i] = f4_scale(S[i], at[r]);
      pk = f4_fma(kt[r], S[i], pk);
      pq = f4_fma(qt[r], S[i], pq);
    }
    *reinterpret_cast<float4*>(&redk[rg][4 * cg]) = pk;
    *reinterpret_cast<float4*>(&redq[rg][4 * cg]) = pq;
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
        tk[tid] = kt[tid];
        tk[D + tid] = u;
        tk[2 * D + tid] = at[tid];
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
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
      const int r = rg + i * RG;
      S[i] = f4_fma(kt[r], *reinterpret_cast<const float4*>(&us[4 * cg]), S[i]);
    }
    if (tid < D) {
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < (D + 31) / 32; ++w) ss += ssq[w];
      const float rstd = rsqrtf(ss / (float)D + a.norm_eps);
      st1(static_cast<T*>(a.y) + (tok * H + h) * D + tid,
          o * rstd * __ldg(a.norm_w + tid) * sigmoid(gs[t * D + tid]));
    }
    if (a.tape != nullptr) {
      float* tp = a.tape + (tok * H + h) * D * D;
#pragma unroll
      for (int i = 0; i < ROWS; ++i) st4(tp + (size_t)(rg + i * RG) * D + 4 * cg, S[i]);
    }
  }

  if (PREP && csg != nullptr && wing == nullptr) {
    // decode: the history now ends with this block's tokens (the last K-1 window rows)
    for (int e = tid; e < Km1 * C3; e += THREADS) {
      const int j = e / C3, c = e - j * C3;
      st1(csg + (((size_t)row * Km1 + j) * H + h) * C3 + c, xwin[(Tn + j) * C3 + c]);
    }
  }
  if (a.state_out != nullptr) {
    float* So = a.state_out + ((size_t)row * H + h) * D * D;
#pragma unroll
    for (int i = 0; i < ROWS; ++i) st4(So + (size_t)(rg + i * RG) * D + 4 * cg, S[i]);
  }
}

template <typename T, bool PREP>
static cudaError_t launch_step_p(const StepArgs& a, cudaStream_t st) {
  dim3 grid(a.H, a.B);
  const size_t smem =
      sizeof(float) * ((size_t)5 * a.T * a.D + (PREP ? (size_t)(a.K - 1 + a.T) * 3 * a.D : 0));
  cudaError_t e = cudaSuccess;
  switch (a.D) {
#define KDA_STEP_CASE(DD)                                                                     \
  case DD:                                                                                    \
    e = cudaFuncSetAttribute(step_kernel<T, DD, PREP>,                                        \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);         \
    if (e != cudaSuccess) return e;                                                           \
    step_kernel<T, DD, PREP><<<grid, StepShape<DD>::THREADS, smem, st>>>(a);                  \
    break;
    KDA_STEP_CASE(16)
    KDA_STEP_CASE(32)
    KDA_STEP_CASE(64)
    KDA_STEP_CASE(128)
#undef KDA_STEP_CASE
    default: return cudaErrorInvalidValue;
  }
  ++launch_counter();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Decode at d = 128 as a persistent stream.  Each CTA walks (sequence, head) units; the
// state of the unit after the current one is copied into shared memory with cp.async
// (each thread copies exactly the 16 float4 it will later read, so the buffer needs no
// block barrier) while the current unit is computed from registers, and the small prep
// inputs of the next unit are loaded into a second register set.  Two CTAs per SM
// (64 KB of state in flight each), so the SM never waits for a whole state load.  The
// per-unit arithmetic is step_kernel's with the L2 normalisation of q and k folded into
// the reductions: S^T k = (S^T k~) / max(||k~||, eps) with k~ the un-normalised conv +
// SiLU output, so one barrier fewer per token.  Shared arrays are double-buffered by unit
// parity, which leaves three block barriers per unit.  No spin-waits: the only waits are
// cp.async.wait_all and block barriers.
// ---------------------------------------------------------------------------
namespace {
constexpr int DS_D = 128, DS_THREADS = 256, DS_ROWS = 16;   // rows rg + 8 i per thread

template <bool PREP>
struct DecodeIn {           // one unit's small inputs as loaded (one thread's share)
  float xc[2], hist[2][3];  // PREP: channels tid, tid + 256 (< 3d): x and 3 history rows
  float f, g, beta_l;       // f, g at channel tid (< d); the beta logit (or beta)
  float q, k, v, la;        // !PREP: prep outputs at channel tid (< d); la = log a
};

// the state row of unit u (-1: no unit or skipped)
__device__ __forceinline__ int ds_row(const StepArgs& a, int u) {
  if (u >= a.B * a.H) return -1;
  return pool_row(a.slots, u / a.H, a.pool_size);
}

// asynchronous copy of this thread's 16 float4 of unit u's state into its shared slots
__device__ __forceinline__ void ds_copy_state(const StepArgs& a, int u, int row, float4* sbuf) {
  const int tid = threadIdx.x, cg = tid & 31, rg = tid >> 5, h = u % a.H;
  const float* Sg = a.state_in + ((size_t)row * a.H + h) * DS_D * DS_D;
#pragma unroll
  for (int i = 0; i < DS_ROWS; ++i) {
    const uint32_t dst = smem_u32_(sbuf + i * DS_THREADS + tid);
    const float* src = Sg + (size_t)(rg + 8 * i) * DS_D + 4 * cg;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <typename T, bool PREP>
__device__ __forceinline__ void ds_load_small(const StepArgs& a, int u, int row, DecodeIn<PREP>& in) {
  const int tid = threadIdx.x;
  const int H = a.H, b = u / H, h = u - b * H;
  const size_t base = ((size_t)b * H + h) * DS_D;
  if (PREP) {
    constexpr int C3 = 3 * DS_D;
    const T* xg = static_cast<const T*>(a.x) + ((size_t)b * H + h) * C3;
    const T* cs = static_cast<const T*>(a.conv_state);
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int c = tid + 256 * m;
      in.xc[m] = 0.f;
      in.hist[m][0] = in.hist[m][1] = in.hist[m][2] = 0.f;
      if (c < C3) {
        in.xc[m] = ld1(xg + c);
        if (cs != nullptr) {
#pragma unroll
          for (int j = 0; j < 3; ++j) in.hist[m][j] = ld1(cs + (((size_t)row * 3 + j) * H + h) * C3 + c);
        }
      }
    }
    if (tid < DS_D) {
      in.f = ld1(static_cast<const T*>(a.f) + base + tid);
      in.g = ld1(static_cast<const T*>(a.g) + base + tid);
    }
    in.beta_l = ld1(static_cast<const T*>(a.beta_logit) + (size_t)b * H + h);
  } else {
    if (tid < DS_D) {
      in.q = __ldg(a.q + base + tid);
      in.k = __ldg(a.k + base + tid);
      in.v = __ldg(a.v + base + tid);
      in.la = __ldg(a.loga + base + tid);
      in.g = ld1(static_cast<const T*>(a.g) + base + tid);
    }
    in.beta_l = __ldg(a.beta + (size_t)b * H + h);
  }
}
}  // namespace

template <typename T, bool PREP>
__global__ void __launch_bounds__(DS_THREADS, 2) decode_stream_kernel(const StepArgs a) {
  constexpr int D = DS_D;
  extern __shared__ float4 sbuf[];                      // [DS_ROWS][DS_THREADS]: 64 KB
  __shared__ __align__(16) float zq[2][D], zk[2][D], as_[2][D], us[2][D];
  __shared__ __align__(16) float redk[8][D], redq[8][D];
  __shared__ float nrm[2][8], kq_s[2], ssq[2][4];
  const int tid = threadIdx.x, cg = tid & 31, rg = tid >> 5, lane = tid & 31, warp = tid >> 5;
  const int H = a.H, n_units = a.B * H, G = gridDim.x;
  // this CTA's units with a state row, in order: u, then the next one after it
  auto next_unit = [&](int v) {
    for (; v < n_units; v += G)
      if (ds_row(a, v) >= 0) return v;
    return n_units;
  };
  int u = next_unit(blockIdx.x);
  DecodeIn<PREP> cur, nxt;
  if (u < n_units) {
    ds_copy_state(a, u, ds_row(a, u), sbuf);
    ds_load_small<T, PREP>(a, u, ds_row(a, u), nxt);
  }
  for (int done = 0; u < n_units; ++done) {
    const int un = next_unit(u + G);
    const int row = ds_row(a, u), p = done & 1, b = u / H, h = u - b * H;
    const size_t base = ((size_t)b * H + h) * D;
    // this unit's state: its copy has landed (each thread waits for its own)
    asm volatile("cp.async.wait_all;" ::: "memory");
    float4 S[DS_ROWS];
#pragma unroll
    for (int i = 0; i < DS_ROWS; ++i) S[i] = sbuf[i * DS_THREADS + tid];
    cur = nxt;
    if (un < n_units) ds_load_small<T, PREP>(a, un, ds_row(a, un), nxt);
    float vv = 0.f, beta;
    if (PREP) {
      // depthwise causal conv (K = 4: three history rows and this token) + SiLU; thread tid
      // owns channels tid (q or k) and tid + 256 (v, when < 3d)
      constexpr int C3 = 3 * D;
      T* cs = static_cast<T*>(a.conv_state);
      float z[2];
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int c = tid + 256 * m;
        z[m] = 0.f;
        if (c < C3) {
          const float4 w = __ldg(reinterpret_cast<const float4*>(a.conv_w + ((size_t)h * C3 + c) * 4));
          const float acc = fmaf(w.x, cur.hist[m][0], fmaf(w.y, cur.hist[m][1],
                                 fmaf(w.z, cur.hist[m][2], w.w * cur.xc[m])));
          z[m] = acc * fsig(acc);
          if (cs != nullptr) {
            st1(cs + (((size_t)row * 3 + 0) * H + h) * C3 + c, cur.hist[m][1]);
            st1(cs + (((size_t)row * 3 + 1) * H + h) * C3 + c, cur.hist[m][2]);
            st1(cs + (((size_t)row * 3 + 2) * H + h) * C3 + c, cur.xc[m]);
          }
        }
      }
      // warps 0-3 hold q (channel tid) and v (tid + 256), warps 4-7 hold k
      float sq = z[0] * z[0];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
      if (lane == 0) nrm[p][warp] = sq;
      if (tid < D) {
        zq[p][tid] = z[0];
        vv = z[1];
        const float Ah = __expf(__ldg(a.A_log + h));
        const float zf = cur.f + __ldg(a.dt_bias + (size_t)h * D + tid);
        as_[p][tid] = __expf(a.gate_softplus ? -Ah * softplus(zf) : a.lb * fsig(Ah * zf));
      } else {
        zk[p][tid - D] = z[0];
      }
      beta = fsig(cur.beta_l);
    } else {
      if (tid < D) {
        zq[p][tid] = cur.q;
        zk[p][tid] = cur.k;
        as_[p][tid] = expf(cur.la);
        vv = cur.v;
      }
      beta = cur.beta_l;
    }
    __syncthreads();                                     // (1) q~, k~, a in shared memory
    float iq = 1.f, ik = 1.f;
    if (PREP) {
      const float nq = nrm[p][0] + nrm[p][1] + nrm[p][2] + nrm[p][3];
      const float nk = nrm[p][4] + nrm[p][5] + nrm[p][6] + nrm[p][7];
      iq = 1.0f / fmaxf(sqrtf(nq), a.l2_eps);
      ik = 1.0f / fmaxf(sqrtf(nk), a.l2_eps);
    }
    // decay along the key axis, then both column reductions (of the un-normalised q~, k~)
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int i = 0; i < DS_ROWS; ++i) {
      const int r = rg + 8 * i;
      S[i] = f4_scale(S[i], as_[p][r]);
      pk = f4_fma(zk[p][r], S[i], pk);
      pq = f4_fma(zq[p][r], S[i], pq);
    }
    // every read of this thread's shared slots has been consumed: refill them with the
    // next unit's state while this one finishes
    if (un < n_units) ds_copy_state(a, un, ds_row(a, un), sbuf);
    *reinterpret_cast<float4*>(&redk[rg][4 * cg]) = pk;
    *reinterpret_cast<float4*>(&redq[rg][4 * cg]) = pq;
    if (warp == 0) {
      float t = 0.f;
#pragma unroll
      for (int c = lane; c < D; c += 32) t = fmaf(zk[p][c], zq[p][c], t);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
      if (lane == 0) kq_s[p] = t;
    }
    __syncthreads();                                     // (2) partial reductions
    float o = 0.f;
    if (tid < D) {
      float rk = 0.f, rq = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) { rk += redk[j][tid]; rq += redq[j][tid]; }
      const float uu = beta * (vv - ik * rk);
      o = a.q_scale * (iq * fmaf(uu * ik, kq_s[p], rq));
      us[p][tid] = uu * ik;                              // k u^T = k~ (ik u)^T
      float t = o * o;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
      if (lane == 0) ssq[p][warp] = t;
    }
    __syncthreads();                                     // (3) u and the norm partials
    // rank-1 write with the un-normalised k~ (its scale moved into u), store the state
    float* Sg = a.state_out + ((size_t)row * H + h) * D * D;
    const float4 u4 = *reinterpret_cast<const float4*>(&us[p][4 * cg]);
#pragma unroll
    for (int i = 0; i < DS_ROWS; ++i) {
      const int r = rg + 8 * i;
      st4(Sg + (size_t)r * D + 4 * cg, f4_fma(zk[p][r], u4, S[i]));
    }
    if (tid < D) {
      const float ss = ssq[p][0] + ssq[p][1] + ssq[p][2] + ssq[p][3];
      const float rstd = rsqrtf(ss / (float)D + a.norm_eps);
      st1(static_cast<T*>(a.y) + base + tid, o * rstd * __ldg(a.norm_w + tid) * sigmoid(cur.g));
    }
    u = un;
  }
}

template <typename T, bool PREP>
static cudaError_t launch_decode_stream(const StepArgs& a, cudaStream_t st) {
  constexpr int SMEM = DS_ROWS * DS_THREADS * 16;      // 64 KB of state per CTA
  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_stream_kernel<T, PREP>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  const int units = a.B * a.H, grid = 2 * nsm;          // two resident CTAs per SM
  decode_stream_kernel<T, PREP><<<units < grid ? units : grid, DS_THREADS, SMEM, st>>>(a);
  ++launch_counter();
  return cudaGetLastError();
}

// the persistent stream serves one-token decode at d = 128 (K = 4 when the prep is fused)
static bool decode_stream_applies(const StepArgs& a) {
  return a.T == 1 && a.D == DS_D && a.tape == nullptr && a.tape_kua == nullptr &&
         a.window == nullptr && a.state_out == a.state_in && (a.x == nullptr || a.K == 4);
}

template <typename T>
static cudaError_t launch_step_t(const StepArgs& a, cudaStream_t st) {
  if (a.x != nullptr && (a.K < 1 || a.K > 8)) return cudaErrorInvalidValue;
  if (decode_stream_applies(a))
    return a.x ? launch_decode_stream<T, true>(a, st) : launch_decode_stream<T, false>(a, st);
  return a.x ? launch_step_p<T, true>(a, st) : launch_step_p<T, false>(a, st);
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
// live state, S <- Diag(a_j) S, then S <- S + k_j u_j^T, element by element exactly as
// step_kernel does it (same layout, same two operations), so the result equals the
// full tape's entry bit for bit; conv state as in rollback_kernel
// ---------------------------------------------------------------------------
template <typename E, int D>
__global__ void __launch_bounds__(StepShape<D>::THREADS) rollback_replay_kernel(const RollbackArgs a) {
  using SH = StepShape<D>;
  constexpr int CG = SH::CG, RG = SH::RG, ROWS = SH::ROWS, THREADS = SH::THREADS;
  constexpr int TMAX = 16;
  __shared__ __align__(16) float kua[TMAX][3][D];
  const int h = blockIdx.x, b = blockIdx.y;
  const int L = clampi(__ldg(a.accepted + b), 0, a.T);
  if (L == 0) return;
  const int row = pool_row(a.slots, b, a.pool_size);
  if (row < 0) return;
  const int H = a.H, tid = threadIdx.x, cg = tid % CG, rg = tid / CG;
  float* Sg = a.state + ((size_t)row * H + h) * D * D;
  float4 S[ROWS];
#pragma unroll
  for (int i = 0; i < ROWS; ++i) S[i] = ld4(Sg + (size_t)(rg + i * RG) * D + 4 * cg);
  for (int e = tid; e < L * 3 * D; e += THREADS) {
    const int j = e / (3 * D), w = e - j * 3 * D;
    (&kua[j][0][0])[w] = __ldg(a.tape_kua + (((size_t)b * a.T + j) * H + h) * 3 * D + w);
  }
  __syncthreads();
  for (int j = 0; j < L; ++j) {
    const float4 u4 = *reinterpret_cast<const float4*>(&kua[j][1][4 * cg]);
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
      const int r = rg + i * RG;
      S[i] = f4_scale(S[i], kua[j][2][r]);
      S[i] = f4_fma(kua[j][0][r], u4, S[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < ROWS; ++i) st4(Sg + (size_t)(rg + i * RG) * D + 4 * cg, S[i]);
  if (a.conv_state != nullptr && a.window != nullptr) {
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
  dim3 grid(a.H, a.B);
  switch (a.D) {
    case 16: rollback_replay_kernel<E, 16><<<grid, StepShape<16>::THREADS, 0, st>>>(a); break;
    case 32: rollback_replay_kernel<E, 32><<<grid, StepShape<32>::THREADS, 0, st>>>(a); break;
    case 64: rollback_replay_kernel<E, 64><<<grid, StepShape<64>::THREADS, 0, st>>>(a); break;
    case 128: rollback_replay_kernel<E, 128><<<grid, StepShape<128>::THREADS, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaSuccess;
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
