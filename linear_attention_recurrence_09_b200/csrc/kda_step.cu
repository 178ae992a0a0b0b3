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

__device__ __forceinline__ float4 f4_scale(float4 a, float s) {
  return make_float4(a.x * s, a.y * s, a.z * s, a.w * s);
}
__device__ __forceinline__ float4 f4_fma(float s, float4 a, float4 acc) {
  return make_float4(fmaf(s, a.x, acc.x), fmaf(s, a.y, acc.y), fmaf(s, a.z, acc.z),
                     fmaf(s, a.w, acc.w));
}

template <typename T, int D, bool PREP>
__global__ void __launch_bounds__(StepShape<D>::THREADS)
step_kernel(const StepArgs a) {
  using SH = StepShape<D>;
  constexpr int CG = SH::CG, RG = SH::RG, ROWS = SH::ROWS, THREADS = SH::THREADS;
  __shared__ __align__(16) float ks[D];
  __shared__ __align__(16) float qs[D];
  __shared__ __align__(16) float as_[D];
  __shared__ __align__(16) float us[D];
  __shared__ __align__(16) float redk[RG][D];
  __shared__ __align__(16) float redq[RG][D];
  __shared__ float ssq[SH::NW];
  __shared__ float kq_s;
  // fused prep: conv history [K-1][3d] (oldest first), conv + SiLU outputs, v, beta, norms
  constexpr int KMAX = 8;
  __shared__ __align__(16) float hist[PREP ? KMAX - 1 : 1][PREP ? 3 * D : 1];
  __shared__ __align__(16) float pre[PREP ? 3 * D : 1];
  __shared__ float beta_s, nrm_w[SH::NW];   // per-warp partial sums of squares (q | k)

  const int h = blockIdx.x, b = blockIdx.y;
  const int H = a.H;
  const int row = pool_row(a.slots, b, a.pool_size);
  if (row < 0) return;
  const int tid = threadIdx.x, cg = tid % CG, rg = tid / CG;
  const int lane = tid & 31, warp = tid >> 5;
  const float* __restrict__ qg = a.q;
  const float* __restrict__ kg = a.k;
  const float* __restrict__ vg = a.v;
  const T* __restrict__ gg = static_cast<const T*>(a.g);
  T* __restrict__ yg = static_cast<T*>(a.y);

  // the state streams in first: everything below (the prep of the first token
  // included) runs while it arrives
  const float* Sg = a.state_in + ((size_t)row * H + h) * D * D;
  float4 S[ROWS];
#pragma unroll
  for (int i = 0; i < ROWS; ++i) S[i] = ld4(Sg + (size_t)(rg + i * RG) * D + 4 * cg);

  constexpr int C3 = 3 * D;
  const int Km1 = PREP ? a.K - 1 : 0;
  T* csg = PREP ? static_cast<T*>(a.conv_state) : nullptr;
  T* wing = PREP ? static_cast<T*>(a.window) : nullptr;
  if (PREP) {
    // the sequence's conv history for this head (zeros without a conv state); verify
    // also starts its rollback window with it
    for (int e = tid; e < Km1 * C3; e += THREADS) {
      const int j = e / C3, c = e - j * C3;
      float hv = 0.f;
      if (csg) hv = ld1(csg + (((size_t)row * Km1 + j) * H + h) * C3 + c);
      hist[j][c] = hv;
      if (wing) st1(wing + (((size_t)b * (Km1 + a.T) + j) * H + h) * C3 + c, hv);
    }
    __syncthreads();   // loaded by (row, channel) pairs, used per channel below
  }

  for (int t = 0; t < a.T; ++t) {
    const size_t tok = (size_t)b * a.T + t;
    const size_t base = (tok * H + h) * D;
    if (PREP) {
      // depthwise causal conv (tap K-1 = this token) + SiLU per channel of q|k|v; each
      // thread owns its channels, so it also shifts their history.  Channel c < 2d (q, k)
      // of thread c also accumulates its warp's sum of squares.
      const T* xg = static_cast<const T*>(a.x) + tok * H * C3 + (size_t)h * C3;
      const T* fg = static_cast<const T*>(a.f) + base;
      float sq = 0.f;
      for (int c = tid; c < C3; c += THREADS) {
        const float xc = ld1(xg + c);
        const float* w = a.conv_w + ((size_t)h * C3 + c) * a.K;
        float acc;
        if (a.K == 4) {   // the common case: one 16-byte load of the taps
          const float4 w4 = __ldg(reinterpret_cast<const float4*>(w));
          acc = fmaf(w4.x, hist[0][c], fmaf(w4.y, hist[1][c], fmaf(w4.z, hist[2][c], w4.w * xc)));
        } else {
          acc = __ldg(w + Km1) * xc;
          for (int j = 0; j < Km1; ++j) acc = fmaf(__ldg(w + j), hist[j][c], acc);
        }
        const float z = acc * fsig(acc);
        pre[c] = z;
        if (c < 2 * D) sq = fmaf(z, z, sq);
        for (int j = 0; j + 1 < Km1; ++j) hist[j][c] = hist[j + 1][c];
        if (Km1 > 0) hist[Km1 - 1][c] = xc;
        if (wing) st1(wing + (((size_t)b * (Km1 + a.T) + Km1 + t) * H + h) * C3 + c, xc);
      }
      // warps whose first channels are q (resp. k) hold q (resp. k) partial norms; with
      // d < 32 a warp spans both, so the d < 32 shapes reduce per half-warp group below
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
      if (lane == 0) nrm_w[warp] = sq;
      // decay a = exp(lb sigmoid(exp(A_log) (f + dt_bias))) (or exp(-exp(A_log) softplus(..))
      // for the gate without a lower bound) and beta = sigmoid(logit)
      const float Ah = __expf(__ldg(a.A_log + h));
      for (int c = tid; c < D; c += THREADS) {
        const float z = ld1(fg + c) + __ldg(a.dt_bias + (size_t)h * D + c);
        as_[c] = __expf(a.gate_softplus ? -Ah * softplus(z) : a.lb * fsig(Ah * z));
      }
      if (tid == 0) beta_s = fsig(ld1(static_cast<const T*>(a.beta_logit) + tok * H + h));
      __syncthreads();
      if (D >= 32) {
        // q channels are those of warps [0, d/32), k channels of warps [d/32, 2d/32)
        float nq = 0.f, nk = 0.f;
#pragma unroll
        for (int w = 0; w < D / 32; ++w) { nq += nrm_w[w]; nk += nrm_w[D / 32 + w]; }
        const float iq = 1.0f / fmaxf(sqrtf(nq), a.l2_eps), ik = 1.0f / fmaxf(sqrtf(nk), a.l2_eps);
        for (int c = tid; c < D; c += THREADS) {
          qs[c] = pre[c] * iq;
          ks[c] = pre[D + c] * ik;
        }
      } else {
        // d = 16: one warp covers q and k; reduce each half directly
        float nq = 0.f, nk = 0.f;
        for (int c = 0; c < D; ++c) {
          nq = fmaf(pre[c], pre[c], nq);
          nk = fmaf(pre[D + c], pre[D + c], nk);
        }
        const float iq = 1.0f / fmaxf(sqrtf(nq), a.l2_eps), ik = 1.0f / fmaxf(sqrtf(nk), a.l2_eps);
        for (int c = tid; c < D; c += THREADS) {
          qs[c] = pre[c] * iq;
          ks[c] = pre[D + c] * ik;
        }
      }
    } else {
      for (int c = tid; c < D; c += THREADS) {
        ks[c] = __ldg(kg + base + c);
        qs[c] = __ldg(qg + base + c);
        as_[c] = expf(__ldg(a.loga + base + c));
      }
    }
    __syncthreads();

    // decay along the key axis, then both column reductions in one pass
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
      const int r = rg + i * RG;
      S[i] = f4_scale(S[i], as_[r]);
      pk = f4_fma(ks[r], S[i], pk);
      pq = f4_fma(qs[r], S[i], pq);
    }
    *reinterpret_cast<float4*>(&redk[rg][4 * cg]) = pk;
    *reinterpret_cast<float4*>(&redq[rg][4 * cg]) = pq;
    if (warp == 0) {
      float p = 0.f;
      for (int c = lane; c < D; c += 32) p = fmaf(ks[c], qs[c], p);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
      if (lane == 0) kq_s = p;
    }
    __syncthreads();

    // per value column: u = b (v - S^T k), o = S^T q + u (k.q), RMSNorm partials
    float o = 0.f;
    if (tid < D) {
      float rk = 0.f, rq = 0.f;
#pragma unroll
      for (int j = 0; j < RG; ++j) { rk += redk[j][tid]; rq += redq[j][tid]; }
      const float bt = PREP ? beta_s : __ldg(a.beta + tok * H + h);
      const float vt = PREP ? pre[2 * D + tid] : __ldg(vg + base + tid);
      const float u = bt * (vt - rk);
      o = a.q_scale * fmaf(u, kq_s, rq);
      us[tid] = u;
      if (a.tape_kua != nullptr) {   // compact tape: this step's k, u and a
        float* tk = a.tape_kua + (tok * H + h) * 3 * D;
        tk[tid] = ks[tid];
        tk[D + tid] = u;
        tk[2 * D + tid] = as_[tid];
      }
    }
    if (warp < (D + 31) / 32) {
      float p = o * o;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
      if (lane == 0) ssq[warp] = p;
    }
    __syncthreads();

    // rank-1 write and the gated RMSNorm epilogue
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
      const int r = rg + i * RG;
      S[i] = f4_fma(ks[r], *reinterpret_cast<const float4*>(&us[4 * cg]), S[i]);
    }
    if (tid < D) {
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < (D + 31) / 32; ++w) ss += ssq[w];
      const float rstd = rsqrtf(ss / (float)D + a.norm_eps);
      const float gt = ld1(gg + base + tid);
      st1(yg + base + tid, o * rstd * __ldg(a.norm_w + tid) * sigmoid(gt));
    }
    if (a.tape != nullptr) {
      float* tp = a.tape + (tok * H + h) * D * D;
#pragma unroll
      for (int i = 0; i < ROWS; ++i) st4(tp + (size_t)(rg + i * RG) * D + 4 * cg, S[i]);
    }
    __syncthreads();
  }

  if (PREP && csg != nullptr && wing == nullptr) {
    // decode: the history now ends with this step's token(s); each thread wrote its own
    // channels of hist, so no barrier is needed before it stores them
    for (int c = tid; c < C3; c += THREADS)
      for (int j = 0; j < Km1; ++j) st1(csg + (((size_t)row * Km1 + j) * H + h) * C3 + c, hist[j][c]);
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
  switch (a.D) {
    case 16: step_kernel<T, 16, PREP><<<grid, StepShape<16>::THREADS, 0, st>>>(a); break;
    case 32: step_kernel<T, 32, PREP><<<grid, StepShape<32>::THREADS, 0, st>>>(a); break;
    case 64: step_kernel<T, 64, PREP><<<grid, StepShape<64>::THREADS, 0, st>>>(a); break;
    case 128: step_kernel<T, 128, PREP><<<grid, StepShape<128>::THREADS, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  ++launch_counter();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Decode at d = 128 as a persistent stream.  One CTA per SM walks the (sequence, head)
// units; while it computes unit u from the state in its registers, the loads of unit
// u + grid (its 64 KB state and, with the fused prep, its x row, conv history, f, beta
// logit and g) are already in flight into a second register set, so every SM keeps a
// state's worth of reads outstanding the whole time instead of alternating load and
// compute phases.  The per-unit arithmetic is step_kernel's with the L2 normalisation of
// q and k folded into the reductions: S^T k = (S^T k~) / max(||k~||, eps) with k~ the
// un-normalised conv + SiLU output, so one barrier fewer per token.  Shared arrays are
// double-buffered by unit parity, which leaves three block barriers per unit.
// ---------------------------------------------------------------------------
namespace {
constexpr int DS_D = 128, DS_THREADS = 256, DS_ROWS = 16;   // rows rg + 8 i per thread

template <typename T, bool PREP>
struct DecodeIn {         // one unit's inputs as loaded (one thread's share)
  float4 S[DS_ROWS];
  float xc[2], hist[2][3];  // PREP: channels tid, tid + 256 (< 3d): x and 3 history rows
  float f, g, beta_l;       // f, g at channel tid (< d); the beta logit
  float q, k, v, la;        // !PREP: prep outputs at channel tid (< d); la = log a
  int row;                  // state row (-1: skip)
};

template <typename T, bool PREP>
__device__ __forceinline__ void ds_load(const StepArgs& a, int u, DecodeIn<T, PREP>& in) {
  const int tid = threadIdx.x, cg = tid & 31, rg = tid >> 5;
  const int H = a.H, b = u / H, h = u - b * H;
  in.row = pool_row(a.slots, b, a.pool_size);
  if (in.row < 0) return;
  const float* Sg = a.state_in + ((size_t)in.row * H + h) * DS_D * DS_D;
#pragma unroll
  for (int i = 0; i < DS_ROWS; ++i) in.S[i] = ld4(Sg + (size_t)(rg + 8 * i) * DS_D + 4 * cg);
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
          for (int j = 0; j < 3; ++j) in.hist[m][j] = ld1(cs + (((size_t)in.row * 3 + j) * H + h) * C3 + c);
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
__global__ void __launch_bounds__(DS_THREADS, 1) decode_stream_kernel(const StepArgs a) {
  constexpr int D = DS_D;
  __shared__ __align__(16) float zq[2][D], zk[2][D], as_[2][D], us[2][D];
  __shared__ __align__(16) float redk[8][D], redq[8][D];
  __shared__ float nrm[2][8], kq_s[2], ssq[2][4];
  const int tid = threadIdx.x, cg = tid & 31, rg = tid >> 5, lane = tid & 31, warp = tid >> 5;
  const int H = a.H, n_units = a.B * H;
  DecodeIn<T, PREP> cur, nxt;
  int u = blockIdx.x, done = 0;
  if (u < n_units) ds_load<T, PREP>(a, u, nxt);
  for (; u < n_units; u += gridDim.x) {
    cur = nxt;
    if (u + (int)gridDim.x < n_units) ds_load<T, PREP>(a, u + gridDim.x, nxt);
    if (cur.row < 0) continue;                           // uniform over the CTA
    // buffer parity of the units this CTA computes (skipped units pass no barrier, so
    // they must not flip it)
    const int p = (done++) & 1, b = u / H, h = u - b * H;
    const size_t base = ((size_t)b * H + h) * D;
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
            st1(cs + (((size_t)cur.row * 3 + 0) * H + h) * C3 + c, cur.hist[m][1]);
            st1(cs + (((size_t)cur.row * 3 + 1) * H + h) * C3 + c, cur.hist[m][2]);
            st1(cs + (((size_t)cur.row * 3 + 2) * H + h) * C3 + c, cur.xc[m]);
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
      cur.S[i] = f4_scale(cur.S[i], as_[p][r]);
      pk = f4_fma(zk[p][r], cur.S[i], pk);
      pq = f4_fma(zq[p][r], cur.S[i], pq);
    }
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
    float* Sg = a.state_out + ((size_t)cur.row * H + h) * D * D;
    const float4 u4 = *reinterpret_cast<const float4*>(&us[p][4 * cg]);
#pragma unroll
    for (int i = 0; i < DS_ROWS; ++i) {
      const int r = rg + 8 * i;
      st4(Sg + (size_t)r * D + 4 * cg, f4_fma(zk[p][r], u4, cur.S[i]));
    }
    if (tid < D) {
      const float ss = ssq[p][0] + ssq[p][1] + ssq[p][2] + ssq[p][3];
      const float rstd = rsqrtf(ss / (float)D + a.norm_eps);
      st1(static_cast<T*>(a.y) + base + tid, o * rstd * __ldg(a.norm_w + tid) * fsig(cur.g));
    }
  }
}

template <typename T, bool PREP>
static cudaError_t launch_decode_stream(const StepArgs& a, cudaStream_t st) {
  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int units = a.B * a.H;
  decode_stream_kernel<T, PREP><<<units < nsm ? units : nsm, DS_THREADS, 0, st>>>(a);
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
