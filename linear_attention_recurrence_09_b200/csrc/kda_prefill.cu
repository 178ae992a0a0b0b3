// kda_prefill: chunkwise-parallel prefill.
//
// Chunkwise form of the KDA recurrence (the chunked fallback class of
// llama.cpp PR #27754, written here from the delta-rule UT/WY transform of
// DeltaNet's chunkwise algorithm with the per-channel decay of gated linear
// attention).  For a chunk of C tokens starting from state S, with
// G_r = sum_{i<=r} log a_i per key channel:
//   A[r,i] = b_r sum_c k_r k_i e^{G_r - G_i}  (i < r),  M[r,i] = q_scale sum_c q_r k_i e^{G_r - G_i}  (i <= r)
//   W = (I + A)^{-1} diag(b) (K * e^G),  U~ = (I + A)^{-1} diag(b) V
//   U = U~ - W S,   O = (q_scale Q * e^G) S + M U,   S <- Diag(e^{G_C}) S + (K * e^{G_C - G})^T U
//
// Pass 1 (intra_chunk_kernel) is parallel over (chunk, head): it writes, per
// chunk slot, W, U~, Q~ = q_scale Q e^G (rows = tokens), K'^T = (K e^{G_C - G})^T
// (rows = key channels), M and e^{G_C} to the workspace, zero-padded past the end
// of the sequence so every chunk is a full, self-contained tile.
// Pass 2 is serial over the chunks of each sequence and parallel over (value
// slice, head, sequence); it carries its slice of the fp32 state on chip and
// writes o.  It runs as bf16 tcgen05 MMAs for d = 128, chunk 64 (sm100 file) and
// as SIMT fp32 otherwise (inter_chunk_kernel).  Pass 3 applies the gated RMSNorm.
//
// Range of the exponentials.  The gate keeps each log a in [lb, 0] with
// lb >= -5, so over a sub-chunk of 16 tokens a cumulative decay spans at most
// 80 < 88 (the fp32 exp overflow bound).  The gram terms e^{G_r - G_i} are
// therefore split at the start of the row's sub-chunk:
//   e^{G_r - G_i} = e^{G_r - G_ref} * e^{G_ref - G_i},  G_ref = G at the row before it,
// where the first factor is <= 1 and the second is <= e^80.  Every other
// exponential in the chunk form has a non-positive argument and may only
// underflow, which is exact to within fp32.  The softplus gate has no lower bound:
// with it, the pairs inside the row's own sub-chunk take e^{G_r - G_i} directly (one
// exponential per pair and channel, argument <= 0), and only the pairs across a
// sub-chunk boundary use the split, whose two factors are then both <= 1.
#include "kda_common.cuh"
#include "kda_launch.h"

namespace kda {

constexpr int SUB = 16;      // sub-chunk length bounding the exponent span
constexpr int P2_J = 16;     // value columns per SIMT inter-chunk CTA

static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

PrefillLayout prefill_layout(int n_seqs, int total, int H, int D, int C, bool bf16) {
  PrefillLayout L;
  L.wsize = bf16 ? 2 : 4;
  L.nslots = num_slots(total, n_seqs, C);
  const size_t per_slot = (size_t)L.nslots * H * C * D;   // C x D tile per (slot, head)
  size_t off = 0;
  L.status = off; off += 256;
  L.flags = off; off += align256((size_t)L.nslots * H * 4);  // per-tile ready flags
  L.zeroed = off;                                            // status + flags, cleared per call
  L.W = off; off += align256(per_slot * L.wsize);
  L.Ut = off; off += align256(per_slot * L.wsize);
  L.Qt = off; off += align256(per_slot * L.wsize);
  L.Kp = off; off += align256(per_slot * L.wsize);          // K'^T, D x C per (slot, head)
  L.o = off; off += align256((size_t)total * H * D * 4);
  L.M = off; off += align256((size_t)L.nslots * H * C * C * L.wsize);
  L.gC = off; off += align256((size_t)L.nslots * H * D * 4);
  L.total = off;
  return L;
}

// ---------------------------------------------------------------------------
// pass 1: intra-chunk (parallel over chunk x head)
// ---------------------------------------------------------------------------
template <int D, int C>
struct P1Smem {
  static constexpr int LD = D + 1;     // padded row stride: conflict-free column walks
  static constexpr int A_LD = C + 1;
  static constexpr size_t bytes = sizeof(float) * (6 * C * LD + C * A_LD + C);
};

template <typename WT, int D, int C>
__global__ void __launch_bounds__(256) intra_chunk_kernel(const PrefillArgs a) {
  using SM = P1Smem<D, C>;
  constexpr int LD = SM::LD;
  extern __shared__ __align__(16) float smem[];
  float* G = smem;                 // [C][LD] cumulative log decay
  float* Kr = G + C * LD;          // [C][LD] k
  float* Kb = Kr + C * LD;         // [C][LD] k_r e^{G_r - G_ref(r)}
  float* Qb = Kb + C * LD;         // [C][LD] q_scale q_r e^{G_r - G_ref(r)}
  float* Kc = Qb + C * LD;         // [C][LD] k_i e^{G_ref(R) - G_i} for the current R
  float* Qr = Kc + C * LD;         // [C][LD] q_scale q (unscaled by the decay)
  float* A = Qr + C * LD;          // [C][A_LD]
  float* bs = A + C * SM::A_LD;    // [C]

  const int h = blockIdx.y, H = a.H;
  const int slot = blockIdx.x;
  const TileRange tr = slot_to_tile(a.cu, a.n_seqs, a.total, C, slot);
  if (tr.len == 0) return;
  if (pool_row(a.slots, tr.seq, a.pool_size) < 0) return;
  const int L = tr.len, t0 = tr.t0, tid = threadIdx.x;
  const size_t tile = (size_t)slot * H + h;
  WT* Wo = reinterpret_cast<WT*>(a.ws + a.L.W) + tile * C * D;
  WT* Uo = reinterpret_cast<WT*>(a.ws + a.L.Ut) + tile * C * D;
  WT* Qo = reinterpret_cast<WT*>(a.ws + a.L.Qt) + tile * C * D;
  WT* KTo = reinterpret_cast<WT*>(a.ws + a.L.Kp) + tile * D * C;
  WT* Mo = reinterpret_cast<WT*>(a.ws + a.L.M) + tile * C * C;
  float* gCo = reinterpret_cast<float*>(a.ws + a.L.gC) + tile * D;

  for (int e = tid; e < C * D; e += blockDim.x) {
    const int r = e / D, c = e - (e / D) * D;
    float la = 0.f, kk = 0.f, qq = 0.f;
    if (r < L) {
      const size_t idx = ((size_t)(t0 + r) * H + h) * D + c;
      la = __ldg(a.loga + idx);
      kk = __ldg(a.k + idx);
      qq = __ldg(a.q + idx);
    }
    G[r * LD + c] = la; Kr[r * LD + c] = kk; Qb[r * LD + c] = qq;
    Qr[r * LD + c] = a.q_scale * qq;
  }
  for (int r = tid; r < C; r += blockDim.x)
    bs[r] = (r < L) ? __ldg(a.beta + (size_t)(t0 + r) * H + h) : 0.f;
  __syncthreads();

  // cumulative log decay per key channel (padded rows add 0)
  for (int c = tid; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int r = 0; r < C; ++r) { acc += G[r * LD + c]; G[r * LD + c] = acc; }
  }
  __syncthreads();

  // row-scaled gram operands and Q~ (rows past the sequence end are zero)
  for (int e = tid; e < C * D; e += blockDim.x) {
    const int r = e / D, c = e - (e / D) * D;
    const float g = G[r * LD + c];
    const int R = r / SUB;
    const float ref = (R == 0) ? 0.f : G[(R * SUB - 1) * LD + c];
    const float er = __expf(g - ref);
    const float kk = Kr[r * LD + c], qq = Qb[r * LD + c];
    Kb[r * LD + c] = kk * er;
    Qb[r * LD + c] = a.q_scale * qq * er;
    st1(Qo + (size_t)r * D + c, a.q_scale * qq * __expf(g));
  }
  // K'^T[c][r] = k_r[c] e^{G_last[c] - G_r[c]}  (r fastest: coalesced rows of K'^T)
  for (int e = tid; e < C * D; e += blockDim.x) {
    const int c = e / C, r = e - (e / C) * C;
    st1(KTo + (size_t)c * C + r, Kr[r * LD + c] * __expf(G[(C - 1) * LD + c] - G[r * LD + c]));
  }
  for (int c = tid; c < D; c += blockDim.x) gCo[c] = __expf(G[(C - 1) * LD + c]);
  __syncthreads();

  // gram blocks, one row sub-chunk R at a time
  for (int R = 0; R < C / SUB; ++R) {
    const int ncol = (R + 1) * SUB;
    for (int e = tid; e < ncol * D; e += blockDim.x) {
      const int i = e / D, c = e - (e / D) * D;
      const float ref = (R == 0) ? 0.f : G[(R * SUB - 1) * LD + c];
      Kc[i * LD + c] = Kr[i * LD + c] * __expf(ref - G[i * LD + c]);
    }
    __syncthreads();
    for (int p = tid; p < SUB * ncol; p += blockDim.x) {
      const int r = R * SUB + p / ncol, i = p - (p / ncol) * ncol;
      float am = 0.f, mm = 0.f;
      if (i <= r && a.gate_softplus && i >= R * SUB) {
        // same sub-chunk, unbounded decay: e^{G_r - G_i} per channel (argument <= 0)
        const float* kr = Kr + r * LD;
        const float* qr = Qr + r * LD;
        const float* ki = Kr + i * LD;
        const float* gr = G + r * LD;
        const float* gi = G + i * LD;
#pragma unroll 4
        for (int c = 0; c < D; ++c) {
          const float e = __expf(gr[c] - gi[c]);
          am = fmaf(kr[c] * ki[c], e, am);
          mm = fmaf(qr[c] * ki[c], e, mm);
        }
      } else if (i <= r) {
        const float* kb = Kb + r * LD;
        const float* qb = Qb + r * LD;
        const float* kc = Kc + i * LD;
#pragma unroll 8
        for (int c = 0; c < D; ++c) {
          am = fmaf(kb[c], kc[c], am);
          mm = fmaf(qb[c], kc[c], mm);
        }
      }
      A[r * SM::A_LD + i] = (i < r) ? bs[r] * am : 0.f;
      st1(Mo + r * C + i, mm);
    }
    for (int p = tid; p < SUB * (C - ncol); p += blockDim.x) {
      const int r = R * SUB + p / (C - ncol), i = ncol + p % (C - ncol);
      A[r * SM::A_LD + i] = 0.f;
      st1(Mo + r * C + i, 0.f);
    }
    __syncthreads();
  }

  // forward substitution (I + A) X = diag(b) B for B = K e^G (m = 0) and V (m = 1);
  // each thread owns one column of one right-hand side, so no barrier is needed.
  // Padded rows have b = 0 and a zero row of A, so their X rows are zero.
  if (tid < 2 * D) {
    const int m = tid / D, c = tid - (tid / D) * D;
    WT* out = (m == 0) ? Wo : Uo;
    float xcol[C];
#pragma unroll
    for (int r = 0; r < C; ++r) {
      float brc;
      if (m == 0) {
        brc = Kr[r * LD + c] * __expf(G[r * LD + c]);
      } else {
        brc = (r < L) ? __ldg(a.v + ((size_t)(t0 + r) * H + h) * D + c) : 0.f;
      }
      float acc = bs[r] * brc;
#pragma unroll
      for (int i = 0; i < r; ++i) acc = fmaf(-A[r * SM::A_LD + i], xcol[i], acc);
      xcol[r] = acc;
      st1(out + (size_t)r * D + c, acc);
    }
  }
}

// ---------------------------------------------------------------------------
// pass 2, SIMT: inter-chunk (serial over chunks; parallel over slice x head x sequence)
// ---------------------------------------------------------------------------
template <typename WT, int D, int C>
struct P2Smem {
  static constexpr size_t tiles = sizeof(WT) * (3 * C * D + C * C);
  static constexpr size_t floats = sizeof(float) * (2 * C * P2_J + D * P2_J + D);
  static constexpr size_t bytes = ((tiles + 15) / 16) * 16 + floats;
};

template <typename WT>
__device__ __forceinline__ void copy_tile(WT* dst, const WT* src, int n) {
  // n contiguous elements (n * sizeof(WT) a multiple of 16)
  constexpr int V = 16 / sizeof(WT);
  for (int e = threadIdx.x; e < n / V; e += blockDim.x)
    reinterpret_cast<uint4*>(dst)[e] = reinterpret_cast<const uint4*>(src)[e];
}

template <typename WT, int D, int C>
__global__ void __launch_bounds__(256) inter_chunk_kernel(const PrefillArgs a) {
  using SM = P2Smem<WT, D, C>;
  constexpr int J = P2_J;
  constexpr int RPT = C / 16;   // rows of U / O per thread
  constexpr int SPT = D / 16;   // state rows per thread
  extern __shared__ __align__(16) unsigned char smraw[];
  WT* Wt = reinterpret_cast<WT*>(smraw);   // [C][D]
  WT* Qt = Wt + C * D;                     // [C][D]
  WT* KT = Qt + C * D;                     // [D][C]
  WT* Mt = KT + C * D;                     // [C][C]
  float* Ut = reinterpret_cast<float*>(smraw + ((SM::tiles + 15) / 16) * 16);  // [C][J]
  float* U = Ut + C * J;                   // [C][J]
  float* S = U + C * J;                    // [D][J]
  float* gC = S + D * J;                   // [D]

  const int j0 = blockIdx.x * J, h = blockIdx.y, s = blockIdx.z, H = a.H;
  const int row = pool_row(a.slots, s, a.pool_size);
  if (row < 0) return;
  const int tid = threadIdx.x, j = tid % 16, rg = tid / 16;
  int start, end;
  seq_range(a.cu, a.total, s, start, end);

  const WT* Wg = reinterpret_cast<const WT*>(a.ws + a.L.W);
  const WT* Ug = reinterpret_cast<const WT*>(a.ws + a.L.Ut);
  const WT* Qg = reinterpret_cast<const WT*>(a.ws + a.L.Qt);
  const WT* KTg = reinterpret_cast<const WT*>(a.ws + a.L.Kp);
  const WT* Mg = reinterpret_cast<const WT*>(a.ws + a.L.M);
  const float* gCg = reinterpret_cast<const float*>(a.ws + a.L.gC);
  float* og = reinterpret_cast<float*>(a.ws + a.L.o);

  const size_t sbase = ((size_t)row * H + h) * D * D;
  for (int e = tid; e < D * J; e += blockDim.x) {
    const int c = e / J, jj = e - (e / J) * J;
    S[e] = a.state_in ? a.state_in[sbase + (size_t)c * D + j0 + jj] : 0.f;
  }

  const int nch = (end - start + C - 1) / C;
  for (int ci = 0; ci < nch; ++ci) {
    const size_t tile = (size_t)(start / C + s + ci) * H + h;
    const int t0 = start + ci * C;
    const int L = min(C, end - t0);
    copy_tile(Wt, Wg + tile * C * D, C * D);
    copy_tile(Qt, Qg + tile * C * D, C * D);
    copy_tile(KT, KTg + tile * D * C, C * D);
    copy_tile(Mt, Mg + tile * C * C, C * C);
    for (int e = tid; e < C * J; e += blockDim.x) {
      const int r = e / J, jj = e - (e / J) * J;
      Ut[e] = ld1(Ug + (tile * C + r) * D + j0 + jj);
    }
    for (int c = tid; c < D; c += blockDim.x) gC[c] = gCg[tile * D + c];
    __syncthreads();

    // U = U~ - W S
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
      const int r = rg + 16 * m;
      float acc = Ut[r * J + j];
      for (int c = 0; c < D; ++c) acc = fmaf(-ld1(Wt + r * D + c), S[c * J + j], acc);
      U[r * J + j] = acc;
    }
    __syncthreads();

    // O = Q~ S + M U
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
      const int r = rg + 16 * m;
      float acc = 0.f;
      for (int c = 0; c < D; ++c) acc = fmaf(ld1(Qt + r * D + c), S[c * J + j], acc);
      for (int i = 0; i <= r; ++i) acc = fmaf(ld1(Mt + r * C + i), U[i * J + j], acc);
      if (r < L) og[((size_t)(t0 + r) * H + h) * D + j0 + j] = acc;
    }
    // S <- Diag(e^{G_C}) S + K'^T U
    float snew[SPT];
#pragma unroll
    for (int m = 0; m < SPT; ++m) {
      const int c = rg + 16 * m;
      float acc = gC[c] * S[c * J + j];
      for (int r = 0; r < C; ++r) acc = fmaf(ld1(KT + c * C + r), U[r * J + j], acc);
      snew[m] = acc;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < SPT; ++m) S[(rg + 16 * m) * J + j] = snew[m];
    __syncthreads();
  }

  if (a.state_out) {
    for (int e = tid; e < D * J; e += blockDim.x) {
      const int c = e / J, jj = e - (e / J) * J;
      a.state_out[sbase + (size_t)c * D + j0 + jj] = S[e];
    }
  }
}

// ---------------------------------------------------------------------------
// pass 3: y = o / sqrt(mean(o^2) + eps) * w * sigmoid(g) per (token, head) row.
// Streaming: lane owns 4 consecutive channels, D/4 lanes per row, and each warp keeps
// NORM_PASSES groups of rows' loads in flight before reducing any of them.
// ---------------------------------------------------------------------------
constexpr int NORM_PASSES = 4;
template <int D>
constexpr int norm_rows_per_cta() { return 8 * (128 / D) * NORM_PASSES; }

template <typename T, int D>
__global__ void __launch_bounds__(256) gated_norm_kernel(const PrefillArgs a) {
  constexpr int LPR = D / 4, RPW = 32 / LPR;   // lanes per row, rows per warp and pass
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, c = 4 * (lane % LPR);
  const size_t nrows = (size_t)a.total * a.H;
  const size_t base = (size_t)blockIdx.x * norm_rows_per_cta<D>() + (size_t)warp * RPW * NORM_PASSES;
  const float* o = reinterpret_cast<const float*>(a.ws + a.L.o);
  const T* g = static_cast<const T*>(a.g);
  float4 ov[NORM_PASSES], gv[NORM_PASSES];
#pragma unroll
  for (int p = 0; p < NORM_PASSES; ++p) {
    const size_t row = base + (size_t)p * RPW + sub;
    ov[p] = gv[p] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < nrows) {
      ov[p] = ld4(o + row * D + c);
      gv[p] = ld4(g + row * D + c);
    }
  }
  const float4 w = ld4(a.norm_w + c);
#pragma unroll
  for (int p = 0; p < NORM_PASSES; ++p) {
    float ss = ov[p].x * ov[p].x + ov[p].y * ov[p].y + ov[p].z * ov[p].z + ov[p].w * ov[p].w;
#pragma unroll
    for (int off = LPR / 2; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float rstd = rsqrtf(ss / (float)D + a.norm_eps);
    const size_t row = base + (size_t)p * RPW + sub;
    if (row < nrows)
      st4(static_cast<T*>(a.y) + row * D + c,
          make_float4(ov[p].x * rstd * w.x * sigmoid(gv[p].x), ov[p].y * rstd * w.y * sigmoid(gv[p].y),
                      ov[p].z * rstd * w.z * sigmoid(gv[p].z), ov[p].w * rstd * w.w * sigmoid(gv[p].w)));
  }
}

template <typename T, int D, int C>
static cudaError_t launch_prefill_dc(const PrefillArgs& a, cudaStream_t st) {
  cudaError_t e;
  const PhaseEvents& pe = phase_events();
  // the tcgen05 passes exchange K' token-major, the SIMT passes K'^T: they pair only
  // with each other, and raw (pre-conv) inputs are only read by the tcgen05 pass
  if (sm100_intra_supported(a) != sm100_interchunk_supported(a)) return cudaErrorInvalidValue;
  if (a.x != nullptr && !sm100_fused_supported(a)) return cudaErrorInvalidValue;
  if (sm100_intra_supported(a) && !a.separate_passes) {
    bool one = false;
    if ((e = launch_cosched_sm100(a, st, &one)) != cudaSuccess) return e;
    if (one) {   // both passes and the norm in one launch
      for (int i = 0; i < 3; ++i)
        if (pe.ev[i] && (e = cudaEventRecord(pe.ev[i], st)) != cudaSuccess) return e;
      return cudaSuccess;
    }
  }
  if (sm100_intra_supported(a)) {
    e = launch_intra_sm100(a, st);
    if (e != cudaSuccess) return e;
  } else {
    auto k1 = intra_chunk_kernel<T, D, C>;
    const size_t sm = P1Smem<D, C>::bytes;
    e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k1<<<dim3(a.L.nslots, a.H), 256, sm, st>>>(a);
    ++launch_counter();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (pe.ev[0] && (e = cudaEventRecord(pe.ev[0], st)) != cudaSuccess) return e;
  bool fused_norm = false;
  if (sm100_interchunk_supported(a)) {
    e = launch_interchunk_sm100(a, st, &fused_norm);
    if (e != cudaSuccess) return e;
  } else {
    auto k2 = inter_chunk_kernel<T, D, C>;
    const size_t sm = P2Smem<T, D, C>::bytes;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    k2<<<dim3(D / P2_J, a.H, a.n_seqs), 256, sm, st>>>(a);
    ++launch_counter();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (pe.ev[1] && (e = cudaEventRecord(pe.ev[1], st)) != cudaSuccess) return e;
  if (a.total > 0 && !fused_norm) {
    const size_t rows = (size_t)a.total * a.H;
    constexpr int RPC = norm_rows_per_cta<D>();
    gated_norm_kernel<T, D><<<(unsigned)((rows + RPC - 1) / RPC), 256, 0, st>>>(a);
    ++launch_counter();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (pe.ev[2] && (e = cudaEventRecord(pe.ev[2], st)) != cudaSuccess) return e;
  return cudaSuccess;
}

PhaseEvents& phase_events() {
  static thread_local PhaseEvents pe{};
  return pe;
}

template <typename T, int D>
static cudaError_t launch_prefill_d(const PrefillArgs& a, cudaStream_t st) {
  switch (a.C) {
    case 16: return launch_prefill_dc<T, D, 16>(a, st);
    case 32: return launch_prefill_dc<T, D, 32>(a, st);
    case 64: return launch_prefill_dc<T, D, 64>(a, st);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t launch_prefill_t(const PrefillArgs& a, cudaStream_t st) {
  switch (a.D) {
    case 16: return launch_prefill_d<T, 16>(a, st);
    case 32: return launch_prefill_d<T, 32>(a, st);
    case 64: return launch_prefill_d<T, 64>(a, st);
    case 128: return launch_prefill_d<T, 128>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t st) {
  return a.bf16 ? launch_prefill_t<__nv_bfloat16>(a, st) : launch_prefill_t<float>(a, st);
}

}  // namespace kda
