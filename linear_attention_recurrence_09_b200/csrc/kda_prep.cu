// kda_prep: depthwise causal conv over q|k|v + SiLU + q/k L2 norm + decay gate + beta.
//
// llama.cpp PR #27754 "model: add GLM-5-Next", KDA commit: q|k|v are convolved as
// ONE depthwise kernel so the conv state is one contiguous block; SiLU follows
// the conv; q/k use max(sqrt(sum), eps) with the literal eps 1e-6; the decay is
// the bounded sigmoid with dt_bias per channel and per-head A broadcast.
//
// One CTA per (16-token tile, head).  The tile's K-1+16 pre-conv rows are staged
// in shared memory (history rows from the conv state or zeros), each thread owns
// two adjacent channels of the head's 3d, and the per-token L2 sums are reduced
// across the d/2 threads of the q (resp. k) channel group.  HBM-bound: every
// input byte is read once (plus a K-1 row halo per tile) and every output byte
// written once.
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {

constexpr int PREP_TILE = 16;
constexpr int PREP_KMAX = 8;

template <typename T, int D>
__global__ void __launch_bounds__(((3 * D / 2 + 31) / 32) * 32)
prep_kernel(const PrepArgs a) {
  constexpr int C3 = 3 * D;
  constexpr int NT = C3 / 2;                       // threads that own a channel pair
  constexpr int GW = (D / 2 < 32) ? D / 2 : 32;    // shuffle width inside one part
  constexpr int WPP = (D / 2 > 32) ? (D / 2) / 32 : 1;  // warps per part
  constexpr int NWARP = ((NT + 31) / 32);
  __shared__ float xs[PREP_TILE + PREP_KMAX - 1][C3];
  __shared__ float wsm[PREP_KMAX][C3];
  __shared__ float part_ss[PREP_TILE][NWARP];

  const int h = blockIdx.y;
  const TileRange tr = slot_to_tile(a.cu, a.n_seqs, a.total, PREP_TILE, blockIdx.x);
  if (tr.len == 0) return;
  const int row = pool_row(a.slots, tr.seq, a.pool_size);
  if (row < 0) return;
  const int H = a.H, K = a.K, Km1 = a.K - 1;
  const int tid = threadIdx.x;
  const T* __restrict__ x = static_cast<const T*>(a.x);
  const T* __restrict__ cs = static_cast<const T*>(a.conv_state);

  const bool own = tid < NT;
  const int ch = 2 * tid;          // channel pair inside the head's 3d
  const int part = ch / D;         // 0 = q, 1 = k, 2 = v
  const int nrows = tr.len + Km1;  // staged rows: history then this tile

  if (own) {
    for (int j = 0; j < K; ++j) {
      wsm[j][ch] = __ldg(a.conv_w + ((size_t)h * C3 + ch) * K + j);
      wsm[j][ch + 1] = __ldg(a.conv_w + ((size_t)h * C3 + ch + 1) * K + j);
    }
    // all staged rows are loaded before any is stored, so the loads overlap
    float2 stage[PREP_TILE + PREP_KMAX - 1];
#pragma unroll
    for (int r = 0; r < PREP_TILE + PREP_KMAX - 1; ++r) {
      const int tok = tr.t0 - Km1 + r;
      float2 val = make_float2(0.f, 0.f);
      if (r < nrows) {
        if (tok >= tr.start) {
          val = ld2(x + ((size_t)tok * H + h) * C3 + ch);
        } else if (cs != nullptr) {
          const int hr = Km1 + (tok - tr.start);  // history row, 0 = oldest
          val = ld2(cs + (((size_t)row * Km1 + hr) * H + h) * C3 + ch);
        }
      }
      stage[r] = val;
    }
#pragma unroll
    for (int r = 0; r < PREP_TILE + PREP_KMAX - 1; ++r) {
      if (r < nrows) {
        xs[r][ch] = stage[r].x;
        xs[r][ch + 1] = stage[r].y;
      }
    }
  }

  // conv + SiLU for the tile (each thread reads only its own columns of xs)
  float v0[PREP_TILE], v1[PREP_TILE], ss[PREP_TILE];
#pragma unroll
  for (int i = 0; i < PREP_TILE; ++i) {
    v0[i] = 0.f; v1[i] = 0.f;
    if (own && i < tr.len) {
      float acc0 = 0.f, acc1 = 0.f;
      for (int j = 0; j < K; ++j) {
        acc0 = fmaf(wsm[j][ch], xs[i + j][ch], acc0);
        acc1 = fmaf(wsm[j][ch + 1], xs[i + j][ch + 1], acc1);
      }
      v0[i] = acc0 * sigmoid(acc0);
      v1[i] = acc1 * sigmoid(acc1);
    }
    ss[i] = (part < 2) ? fmaf(v0[i], v0[i], v1[i] * v1[i]) : 0.f;
  }

  // L2 sums over the d channels of q and of k
#pragma unroll
  for (int i = 0; i < PREP_TILE; ++i) {
#pragma unroll
    for (int off = GW / 2; off >= 1; off >>= 1) ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], off);
  }
  if (WPP > 1) {
    if ((tid & 31) == 0 && tid / 32 < NWARP) {
#pragma unroll
      for (int i = 0; i < PREP_TILE; ++i) part_ss[i][tid / 32] = ss[i];
    }
    __syncthreads();
    if (own && part < 2) {
#pragma unroll
      for (int i = 0; i < PREP_TILE; ++i) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < WPP; ++w) t += part_ss[i][part * WPP + w];
        ss[i] = t;
      }
    }
  }

  if (own) {
    float* dst = part == 0 ? a.q : (part == 1 ? a.k : a.v);
    const int c = ch - part * D;
#pragma unroll
    for (int i = 0; i < PREP_TILE; ++i) {
      if (i < tr.len) {
        const float sc = (part < 2) ? 1.0f / fmaxf(sqrtf(ss[i]), a.l2_eps) : 1.0f;
        st2(dst + ((size_t)(tr.t0 + i) * H + h) * D + c, v0[i] * sc, v1[i] * sc);
      }
    }
    if (a.mode == 1 && a.window != nullptr) {  // TAPE: [history; x] per sequence
      T* win = static_cast<T*>(a.window);
      const size_t base = (size_t)tr.start + (size_t)tr.seq * Km1;
      const int r0 = (tr.chunk == 0) ? 0 : Km1;
      for (int r = r0; r < nrows; ++r) {
        const size_t wr = base + (size_t)(tr.t0 - tr.start) + r;
        st2(win + (wr * H + h) * C3 + ch, xs[r][ch], xs[r][ch + 1]);
      }
    }
    if (a.mode == 0 && a.commit_in_kernel && cs != nullptr && tr.chunk == 0 &&
        tr.len == tr.end - tr.start) {
      // whole sequence in this tile: the new history is the last K-1 staged rows
      T* csw = static_cast<T*>(a.conv_state);
      for (int j = 0; j < Km1; ++j)
        st2(csw + (((size_t)row * Km1 + j) * H + h) * C3 + ch, xs[tr.len + j][ch],
            xs[tr.len + j][ch + 1]);
    }
  }

  // decay gate and beta (loads first, then the arithmetic)
  const T* __restrict__ f = static_cast<const T*>(a.f);
  const float Ah = expf(__ldg(a.A_log + h));
  constexpr int NTHR = ((3 * D / 2 + 31) / 32) * 32;      // the launch's block size
  constexpr int NB = (PREP_TILE * D + NTHR - 1) / NTHR;  // elements per thread
  const int nthr = NTHR;
  float fv[NB];
#pragma unroll
  for (int m = 0; m < NB; ++m) {
    const int e = tid + m * nthr;
    fv[m] = 0.f;
    if (e < tr.len * D) {
      const int i = e / D, c = e - (e / D) * D;
      fv[m] = ld1(f + ((size_t)(tr.t0 + i) * H + h) * D + c);
    }
  }
#pragma unroll
  for (int m = 0; m < NB; ++m) {
    const int e = tid + m * nthr;
    if (e < tr.len * D) {
      const int i = e / D, c = e - (e / D) * D;
      const size_t idx = ((size_t)(tr.t0 + i) * H + h) * D + c;
      a.loga[idx] = a.lb * sigmoid(Ah * (fv[m] + __ldg(a.dt_bias + (size_t)h * D + c)));
    }
  }
  if (tid < tr.len) {
    const size_t idx = (size_t)(tr.t0 + tid) * H + h;
    a.beta[idx] = sigmoid(ld1(static_cast<const T*>(a.beta_logit) + idx));
  }
}

// Conv-state commit for sequences longer than one tile: the new history is the
// last K-1 rows of [history; x_s].  Runs after prep_kernel (stream order), so the
// old history has been consumed before it is overwritten.
template <typename T>
__global__ void conv_commit_kernel(const PrepArgs a) {
  const int s = blockIdx.x, h = blockIdx.y;
  int start, end;
  seq_range(a.cu, a.total, s, start, end);
  const int len = end - start;
  if (a.commit_in_kernel && len <= PREP_TILE) return;  // done inside prep_kernel
  const int row = pool_row(a.slots, s, a.pool_size);
  if (row < 0) return;
  const int H = a.H, Km1 = a.K - 1, C3 = 3 * a.D;
  const T* x = static_cast<const T*>(a.x);
  T* cs = static_cast<T*>(a.conv_state);
  for (int c = threadIdx.x; c < C3; c += blockDim.x) {
    float nv[PREP_KMAX];
#pragma unroll
    for (int j = 0; j < PREP_KMAX - 1; ++j) {
      nv[j] = 0.f;
      if (j < Km1) {
        const int src = len + j;  // index into [history (K-1 rows); x_s]
        nv[j] = (src >= Km1) ? ld1(x + ((size_t)(start + src - Km1) * H + h) * C3 + c)
                             : ld1(cs + (((size_t)row * Km1 + src) * H + h) * C3 + c);
      }
    }
#pragma unroll
    for (int j = 0; j < PREP_KMAX - 1; ++j)
      if (j < Km1) st1(cs + (((size_t)row * Km1 + j) * H + h) * C3 + c, nv[j]);
  }
}

template <typename T, int D>
static cudaError_t launch_prep_t(const PrepArgs& a, cudaStream_t st) {
  constexpr int threads = ((3 * D / 2 + 31) / 32) * 32;
  dim3 grid(num_slots(a.total, a.n_seqs, PREP_TILE), a.H);
  prep_kernel<T, D><<<grid, threads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.mode == 0 && a.conv_state != nullptr && a.K > 1 && !a.commit_in_kernel) {
    conv_commit_kernel<T><<<dim3(a.n_seqs, a.H), 128, 0, st>>>(a);
    e = cudaGetLastError();
  }
  return e;
}

template <typename T>
static cudaError_t launch_prep_d(const PrepArgs& a, cudaStream_t st) {
  switch (a.D) {
    case 16: return launch_prep_t<T, 16>(a, st);
    case 32: return launch_prep_t<T, 32>(a, st);
    case 64: return launch_prep_t<T, 64>(a, st);
    case 128: return launch_prep_t<T, 128>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_prep(const PrepArgs& a, cudaStream_t st) {
  return a.bf16 ? launch_prep_d<__nv_bfloat16>(a, st) : launch_prep_d<float>(a, st);
}

int prep_tile() { return PREP_TILE; }
int prep_kmax() { return PREP_KMAX; }

}  // namespace kda
