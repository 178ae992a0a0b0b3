// kda_prep: depthwise causal conv over q|k|v + SiLU + q/k L2 norm + decay gate + beta.
//
// llama.cpp PR #27754 "model: add GLM-5-Next", KDA commit: q|k|v are convolved as
// ONE depthwise kernel so the conv state is one contiguous block; SiLU follows
// the conv; q/k use max(sqrt(sum), eps) with eps exactly 1e-6; the decay is
// the bounded sigmoid with dt_bias per channel and per-head A broadcast (or, when the
// gate has no lower bound, the softplus branch of the "Metadata and tensor loading"
// commit).
//
// HBM-bound streaming kernel.  A CTA covers a tile of up to 64 tokens of one
// sequence for HPB consecutive heads; each thread owns 4 adjacent channels of one
// head's 3d (8-byte bf16 / 16-byte fp32 accesses, coalesced across the block),
// walks the tile's tokens in order with 8 rows in flight and keeps the last K-1
// pre-conv rows of its channels in registers, so every input byte is read once
// (plus a K-1 row halo per tile).  The per-token L2 sums of q and k reduce by
// shuffles inside the aligned group of d/4 threads that owns them.  The decay
// gate and beta follow in a second coalesced pass over the tile.
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {

constexpr int PREP_TILE = 64;
constexpr int PREP_KMAX = 8;
constexpr int PREP_THREADS = 192;
constexpr int PREP_UNROLL = 8;     // token rows in flight per thread

__device__ __forceinline__ void unpack4(float4 v, float (&o)[4]) {
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}

template <typename T, int D, int K>
__global__ void __launch_bounds__(PREP_THREADS) prep_kernel(const PrepArgs a) {
  constexpr int C3 = 3 * D;
  constexpr int TPH = C3 / 4;                  // threads per head (4 channels each)
  constexpr int HPB = PREP_THREADS / TPH;      // heads per CTA
  constexpr int G = D / 4;                     // threads per q (or k, v) group
  constexpr int KM1 = K - 1;
  constexpr int KW = KM1 > 0 ? KM1 : 1;

  // a token-step kernel launched next may be scheduled now (it waits for this grid's
  // completion before reading what it writes)
  grid_dep_trigger();
  const TileRange tr = slot_to_tile(a.cu, a.n_seqs, a.total, PREP_TILE, blockIdx.x);
  if (tr.len == 0) return;
  const int row = pool_row(a.slots, tr.seq, a.pool_size);
  if (row < 0) return;
  const int hs = threadIdx.x / TPH, j = threadIdx.x - hs * TPH;
  const int h = blockIdx.y * HPB + hs;
  const bool active = h < a.H;                 // uniform per aligned group of G threads
  const int H = a.H;
  const int ch = 4 * j;                        // first channel of this thread in the head's 3d
  const int part = j / G;                      // 0 = q, 1 = k, 2 = v
  const T* __restrict__ x = static_cast<const T*>(a.x);
  const T* __restrict__ cs = static_cast<const T*>(a.conv_state);

  float w[K][4];
  float win[KW][4];
#pragma unroll
  for (int r = 0; r < KW; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) win[r][c] = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int t = 0; t < K; ++t)
      w[t][c] = active ? __ldg(a.conv_w + ((size_t)h * C3 + ch + c) * K + t) : 0.f;
  if (active) {
    // history: rows t0-K+1 .. t0-1 (from x inside the sequence, else the conv state)
#pragma unroll
    for (int r = 0; r < KM1; ++r) {
      const int tok = tr.t0 - KM1 + r;
      if (tok >= tr.start) {
        unpack4(ld4(x + ((size_t)tok * H + h) * C3 + ch), win[r]);
      } else if (cs != nullptr) {
        unpack4(ld4(cs + (((size_t)row * KM1 + (KM1 + tok - tr.start)) * H + h) * C3 + ch),
                win[r]);
      }
    }
    if (a.mode == 1 && a.window != nullptr && tr.chunk == 0) {
      T* wp = static_cast<T*>(a.window);
      const size_t base = (size_t)tr.start + (size_t)tr.seq * KM1;
#pragma unroll
      for (int r = 0; r < KM1; ++r)
        st4(wp + ((base + r) * H + h) * C3 + ch, make_float4(win[r][0], win[r][1], win[r][2], win[r][3]));
    }
  }
  float* dst = part == 0 ? a.q : (part == 1 ? a.k : a.v);

  for (int i0 = 0; i0 < tr.len; i0 += PREP_UNROLL) {
    float xin[PREP_UNROLL][4];
#pragma unroll
    for (int u = 0; u < PREP_UNROLL; ++u) {
      xin[u][0] = xin[u][1] = xin[u][2] = xin[u][3] = 0.f;
      if (active && i0 + u < tr.len)
        unpack4(ld4(x + ((size_t)(tr.t0 + i0 + u) * H + h) * C3 + ch), xin[u]);
    }
#pragma unroll
    for (int u = 0; u < PREP_UNROLL; ++u) {
      const int i = i0 + u;
      if (i >= tr.len) break;                  // uniform across the CTA
      const int tok = tr.t0 + i;
      float y[4];
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float acc = w[K - 1][c] * xin[u][c];
#pragma unroll
        for (int t = 0; t < KM1; ++t) acc = fmaf(w[t][c], win[t][c], acc);
        y[c] = acc * sigmoid(acc);
        ss = fmaf(y[c], y[c], ss);
      }
      if (KM1 > 0) {
#pragma unroll
        for (int t = 0; t + 1 < KM1; ++t)
#pragma unroll
          for (int c = 0; c < 4; ++c) win[t][c] = win[t + 1][c];
#pragma unroll
        for (int c = 0; c < 4; ++c) win[KW - 1][c] = xin[u][c];
      }
#pragma unroll
      for (int off = G / 2; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (active) {
        const float sc = (part < 2) ? 1.0f / fmaxf(sqrtf(ss), a.l2_eps) : 1.0f;
        st4(dst + ((size_t)tok * H + h) * D + (ch - part * D),
            make_float4(y[0] * sc, y[1] * sc, y[2] * sc, y[3] * sc));
        if (a.mode == 1 && a.window != nullptr) {
          T* wp = static_cast<T*>(a.window);
          const size_t wr = (size_t)tr.start + (size_t)tr.seq * KM1 + KM1 + (tok - tr.start);
          st4(wp + (wr * H + h) * C3 + ch, make_float4(xin[u][0], xin[u][1], xin[u][2], xin[u][3]));
        }
      }
    }
  }
  // whole sequence in this tile: the register window holds its new conv history
  if (KM1 > 0 && active && a.mode == 0 && a.commit_in_kernel && cs != nullptr &&
      tr.chunk == 0 && tr.len == tr.end - tr.start) {
    T* csw = static_cast<T*>(a.conv_state);
#pragma unroll
    for (int r = 0; r < KM1; ++r)
      st4(csw + (((size_t)row * KM1 + r) * H + h) * C3 + ch,
          make_float4(win[r][0], win[r][1], win[r][2], win[r][3]));
  }

  // decay gate (4 channels per item) and beta, coalesced over the tile
  if (active) {
    const T* __restrict__ f = static_cast<const T*>(a.f);
    const float Ah = expf(__ldg(a.A_log + h));
    constexpr int IPR = D / 4;                 // items per token row
    for (int e0 = j; e0 < tr.len * IPR; e0 += 4 * TPH) {
      float4 fv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * TPH;
        if (e < tr.len * IPR)
          fv[u] = ld4(f + ((size_t)(tr.t0 + e / IPR) * H + h) * D + (e % IPR) * 4);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * TPH;
        if (e < tr.len * IPR) {
          const int c = (e % IPR) * 4;
          const float4 db = *reinterpret_cast<const float4*>(a.dt_bias + (size_t)h * D + c);
          const int sp = a.gate_softplus;
          st4(a.loga + ((size_t)(tr.t0 + e / IPR) * H + h) * D + c,
              make_float4(gate_log_decay(Ah, fv[u].x + db.x, a.lb, sp),
                          gate_log_decay(Ah, fv[u].y + db.y, a.lb, sp),
                          gate_log_decay(Ah, fv[u].z + db.z, a.lb, sp),
                          gate_log_decay(Ah, fv[u].w + db.w, a.lb, sp)));
        }
      }
    }
    for (int i = j; i < tr.len; i += TPH)
      a.beta[(size_t)(tr.t0 + i) * H + h] =
          sigmoid(ld1(static_cast<const T*>(a.beta_logit) + (size_t)(tr.t0 + i) * H + h));
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

// kda_prep for short sequences (decode steps, verify blocks): one CTA of d threads per
// (sequence, head).  Thread j < 3d/4 owns channels 4j..4j+3 of the head's q|k|v, thread
// j >= 3d/4 four channels of the decay gate (the first of them also beta).  Every input of
// the CTA (taps, conv history, x rows, f, beta logit) is requested at once, so a launch
// costs about two dependent memory round trips; tokens are taken TB at a time, so a
// sequence longer than the hint is still processed in full.  The conv runs over a register
// window of the last KM >= K rows with the taps placed by distance from the token (zero
// past K), accumulated from the token itself backwards.
template <typename T, int D, int TB, int KM>
__global__ void __launch_bounds__(D) prep_short_kernel(const PrepArgs a) {
  constexpr int C3 = 3 * D, G = D / 4;
  grid_dep_trigger();
  const int s = blockIdx.x, h = blockIdx.y, H = a.H, K = a.K, Km1 = K - 1;
  const int j = threadIdx.x, part = j / G;             // 0 q, 1 k, 2 v, 3 gate
  int start, end;
  seq_range(a.cu, a.total, s, start, end);
  const int row = pool_row(a.slots, s, a.pool_size);
  if (row < 0) return;
  const int len = end - start;
  const T* __restrict__ x = static_cast<const T*>(a.x);
  const T* __restrict__ cs = static_cast<const T*>(a.conv_state);
  T* wp = static_cast<T*>(a.window);
  const size_t wbase = (size_t)start + (size_t)s * Km1;   // window row of this sequence's oldest

  if (part < 3) {
    const int ch = 4 * j;                                  // channel in the head's 3d
    // taps by distance m from the token: wa[m] = w[K-1-m] for m < K, else 0
    float wa[KM][4];
    const float* wr = a.conv_w + ((size_t)h * C3 + ch) * K;
    if (KM == 4 && K == 4) {                               // one 16-byte load per channel
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float4 w4 = __ldg(reinterpret_cast<const float4*>(wr + 4 * c));
        wa[0][c] = w4.w; wa[1][c] = w4.z; wa[2][c] = w4.y; wa[3][c] = w4.x;
      }
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int m = 0; m < KM; ++m) wa[m][c] = m < K ? __ldg(wr + (size_t)c * K + (K - 1 - m)) : 0.f;
    }
    // win[m] = the row m back from the next token (m = 1..KM-1); history rows first
    float win[KM][4];
#pragma unroll
    for (int m = 0; m < KM; ++m) {
      win[m][0] = win[m][1] = win[m][2] = win[m][3] = 0.f;
      if (m >= 1 && m <= Km1 && cs != nullptr)
        unpack4(ld4(cs + (((size_t)row * Km1 + (Km1 - m)) * H + h) * C3 + ch), win[m]);
    }
    if (a.mode == 1 && wp != nullptr) {
#pragma unroll
      for (int m = 1; m < KM; ++m)
        if (m <= Km1)
          st4(wp + ((wbase + (Km1 - m)) * H + h) * C3 + ch,
              make_float4(win[m][0], win[m][1], win[m][2], win[m][3]));
    }
    const unsigned gmask =
        G >= 32 ? 0xffffffffu : (((1u << G) - 1u) << ((j & 31) & ~(G - 1)));
    float* dst = (part == 0 ? a.q : part == 1 ? a.k : a.v) + (ch - part * D);
    for (int t0 = 0; t0 < len; t0 += TB) {
      const int n = min(TB, len - t0);
      float xin[TB][4];
#pragma unroll
      for (int i = 0; i < TB; ++i) {
        xin[i][0] = xin[i][1] = xin[i][2] = xin[i][3] = 0.f;
        if (i < n) unpack4(ld4(x + ((size_t)(start + t0 + i) * H + h) * C3 + ch), xin[i]);
      }
#pragma unroll
      for (int i = 0; i < TB; ++i) {
        if (i >= n) break;                                 // uniform across the CTA
        const int tok = start + t0 + i;
        float y[4], ss = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float acc = fmaf(wa[0][c], xin[i][c], 0.f);
#pragma unroll
          for (int m = 1; m < KM; ++m) acc = fmaf(wa[m][c], win[m][c], acc);
          y[c] = acc * __fdividef(1.f, 1.f + __expf(-acc));   // SiLU, approximate exp / divide
          ss = fmaf(y[c], y[c], ss);
        }
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) ss += __shfl_xor_sync(gmask, ss, off);
        const float sc = (part < 2) ? 1.0f / fmaxf(sqrtf(ss), a.l2_eps) : 1.0f;
        st4(dst + ((size_t)tok * H + h) * D, make_float4(y[0] * sc, y[1] * sc, y[2] * sc, y[3] * sc));
        if (a.mode == 1 && wp != nullptr)
          st4(wp + ((wbase + Km1 + t0 + i) * H + h) * C3 + ch,
              make_float4(xin[i][0], xin[i][1], xin[i][2], xin[i][3]));
#pragma unroll
        for (int m = KM - 1; m >= 2; --m)
#pragma unroll
          for (int c = 0; c < 4; ++c) win[m][c] = win[m - 1][c];
#pragma unroll
        for (int c = 0; c < 4; ++c) win[1][c] = xin[i][c];
      }
    }
    // commit: the new history is the last K-1 rows of [history; x]
    if (a.mode == 0 && a.conv_state != nullptr) {
      T* csw = static_cast<T*>(a.conv_state);
#pragma unroll
      for (int m = 1; m < KM; ++m)
        if (m <= Km1)
          st4(csw + (((size_t)row * Km1 + (Km1 - m)) * H + h) * C3 + ch,
              make_float4(win[m][0], win[m][1], win[m][2], win[m][3]));
    }
  } else {
    // decay gate of four channels, and beta, for every token
    const int c0 = 4 * (j - 3 * G);
    const T* __restrict__ f = static_cast<const T*>(a.f);
    const float Ah = expf(__ldg(a.A_log + h));
    const float4 db = *reinterpret_cast<const float4*>(a.dt_bias + (size_t)h * D + c0);
    const int sp = a.gate_softplus;
    for (int t0 = 0; t0 < len; t0 += TB) {
      const int n = min(TB, len - t0);
      float4 fv[TB];
      float bl[TB];
#pragma unroll
      for (int i = 0; i < TB; ++i) {
        if (i < n) {
          fv[i] = ld4(f + ((size_t)(start + t0 + i) * H + h) * D + c0);
          if (c0 == 0) bl[i] = ld1(static_cast<const T*>(a.beta_logit) + (size_t)(start + t0 + i) * H + h);
        }
      }
#pragma unroll
      for (int i = 0; i < TB; ++i) {
        if (i >= n) break;
        const size_t tok = (size_t)(start + t0 + i);
        st4(a.loga + (tok * H + h) * D + c0,
            make_float4(gate_log_decay(Ah, fv[i].x + db.x, a.lb, sp),
                        gate_log_decay(Ah, fv[i].y + db.y, a.lb, sp),
                        gate_log_decay(Ah, fv[i].z + db.z, a.lb, sp),
                        gate_log_decay(Ah, fv[i].w + db.w, a.lb, sp)));
        if (c0 == 0) a.beta[tok * H + h] = sigmoid(bl[i]);
      }
    }
  }
}

template <typename T, int D, int KM>
static cudaError_t launch_prep_short_k(const PrepArgs& a, cudaStream_t st) {
  const dim3 grid(a.n_seqs, a.H);
  switch (a.short_tb) {
    case 1: prep_short_kernel<T, D, 1, KM><<<grid, D, 0, st>>>(a); break;
    case 8: prep_short_kernel<T, D, 8, KM><<<grid, D, 0, st>>>(a); break;
    default: prep_short_kernel<T, D, 16, KM><<<grid, D, 0, st>>>(a); break;
  }
  ++launch_counter();
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_prep_short(const PrepArgs& a, cudaStream_t st) {
  return a.K <= 4 ? launch_prep_short_k<T, D, 4>(a, st) : launch_prep_short_k<T, D, PREP_KMAX>(a, st);
}

template <typename T, int D, int K>
static cudaError_t launch_prep_k(const PrepArgs& a, cudaStream_t st) {
  constexpr int HPB = PREP_THREADS / (3 * D / 4);
  dim3 grid(num_slots(a.total, a.n_seqs, PREP_TILE), (a.H + HPB - 1) / HPB);
  prep_kernel<T, D, K><<<grid, PREP_THREADS, 0, st>>>(a);
  ++launch_counter();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.mode == 0 && a.conv_state != nullptr && K > 1 && !a.commit_in_kernel) {
    conv_commit_kernel<T><<<dim3(a.n_seqs, a.H), 128, 0, st>>>(a);
    ++launch_counter();
    e = cudaGetLastError();
  }
  return e;
}

template <typename T, int D>
static cudaError_t launch_prep_t(const PrepArgs& a, cudaStream_t st) {
  if (a.short_tb > 0) return launch_prep_short<T, D>(a, st);
  switch (a.K) {
    case 1: return launch_prep_k<T, D, 1>(a, st);
    case 2: return launch_prep_k<T, D, 2>(a, st);
    case 3: return launch_prep_k<T, D, 3>(a, st);
    case 4: return launch_prep_k<T, D, 4>(a, st);
    case 5: return launch_prep_k<T, D, 5>(a, st);
    case 6: return launch_prep_k<T, D, 6>(a, st);
    case 7: return launch_prep_k<T, D, 7>(a, st);
    case 8: return launch_prep_k<T, D, 8>(a, st);
  }
  return cudaErrorInvalidValue;
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

cudaError_t launch_conv_commit(const PrepArgs& a, cudaStream_t st) {
  if (a.conv_state == nullptr || a.K < 2 || a.n_seqs == 0) return cudaSuccess;
  if (a.bf16) conv_commit_kernel<__nv_bfloat16><<<dim3(a.n_seqs, a.H), 128, 0, st>>>(a);
  else conv_commit_kernel<float><<<dim3(a.n_seqs, a.H), 128, 0, st>>>(a);
  ++launch_counter();
  return cudaGetLastError();
}

cudaError_t launch_prep(const PrepArgs& a, cudaStream_t st) {
  return a.bf16 ? launch_prep_d<__nv_bfloat16>(a, st) : launch_prep_d<float>(a, st);
}

int prep_tile() { return PREP_TILE; }
int prep_kmax() { return PREP_KMAX; }

}  // namespace kda
