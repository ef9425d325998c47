// Centroid-based top-p block selection (Sparse VideoGen2, section 2(b):
// "Centroid approximation" scores cluster pairs through their centroids;
// "Top-p strategy" sorts clusters by estimated score and takes them until
// the cumulative score reaches p).
//
// The cut turns floating-point weights into an integer set, so it is decided
// in float64: logits (products of fp32 centroid channels are exact in
// float64), weights and prefix masses.  A float64 decision differs from the
// exact one only when a prefix mass lies within about 1e-12 of p.
//
// One block of kSelRows warps per (head, group of kSelRows q-clusters).
// Phase 1: chunks of 32 k-centroids are staged in shared memory with
// coalesced loads; thread (warp r, lane j) forms the float64 logit of row r
// and centroid j of the chunk.  Phase 2: one warp per row forms
// w_j = n_kj * exp(logit_j - max) for live j (n_kj > 0) and finds the cut
// without sorting: with key_j = the bits of w_j whose lowest 10 bits are
// replaced by 1023 - j (descending key = descending weight, ties to the lower
// j), the kept set is {j : key_j >= t*} where t* is the largest key value t
// with sum_{key_j >= t} w_j >= p * sum_j w_j.  t* is built bit by bit from
// the top (63 warp-wide masked sums).  Selected ids are written in ascending
// order.
#pragma once
#include "common.cuh"

namespace svg {

constexpr int kSelRows = 8;     // q-cluster rows per block (one warp each)
constexpr int kSelChunk = 32;   // k-centroids staged in shared memory at a time
constexpr int kMaxCk = 1024;

__device__ __forceinline__ double warp_sum_bcast(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return __shfl_sync(0xffffffffu, v, 0);   // one lane's rounding for the whole warp
}

__device__ __forceinline__ uint64_t select_key(double w, int j) {
  return (static_cast<uint64_t>(__double_as_longlong(w)) & ~1023ull) | static_cast<uint64_t>(1023 - j);
}

// CPL = k-clusters per lane (ceil(Ck / 32) rounded up to 4, 8, 16 or 32).
template <int D, int CPL>
__global__ void __launch_bounds__(kSelRows * 32, CPL <= 16 ? 3 : 2) select_topp_kernel(
    const float *__restrict__ mu_q, const int32_t *__restrict__ n_q, const float *__restrict__ mu_k,
    const int32_t *__restrict__ n_k, int Cq, int Ck, float p, double scale,
    int32_t *__restrict__ sel_count, int32_t *__restrict__ sel_cols) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  constexpr int KROW = D + 4;                             // padded fp32 row: conflict-free reads
  double *sq = reinterpret_cast<double *>(smem_raw);     // [kSelRows][D]
  double *slog = sq + kSelRows * D;                       // [kSelRows][Ck]
  float *sk = reinterpret_cast<float *>(slog + kSelRows * Ck);   // [kSelChunk][KROW]
  const int h = blockIdx.y;
  const int i0 = blockIdx.x * kSelRows;
  const int nrows = min(kSelRows, Cq - i0);
  for (int t = threadIdx.x; t < kSelRows * D; t += blockDim.x) {
    const int r = t / D, d = t % D;
    sq[t] = r < nrows ? static_cast<double>(mu_q[(static_cast<size_t>(h) * Cq + i0 + r) * D + d]) : 0.0;
  }
  // phase 1: float64 logits, 32 k-centroids at a time
  const float *mkh = mu_k + static_cast<size_t>(h) * Ck * D;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j0 = 0; j0 < Ck; j0 += kSelChunk) {
    const int nj = min(kSelChunk, Ck - j0);
    __syncthreads();   // the previous chunk has been read (and sq is written)
    for (int t = threadIdx.x; t < kSelChunk * (D / 4); t += blockDim.x) {
      const int jr = t / (D / 4), d4 = t % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (jr < nj) v = __ldg(reinterpret_cast<const float4 *>(mkh + static_cast<size_t>(j0 + jr) * D) + d4);
      *reinterpret_cast<float4 *>(sk + jr * KROW + 4 * d4) = v;
    }
    __syncthreads();
    if (lane < nj) {
      const double *qr = sq + w * D;
      const float *kr = sk + lane * KROW;
      double acc = 0.0;
#pragma unroll 8
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 kv = *reinterpret_cast<const float4 *>(kr + 4 * d4);
        acc = fma(qr[4 * d4], static_cast<double>(kv.x), acc);
        acc = fma(qr[4 * d4 + 1], static_cast<double>(kv.y), acc);
        acc = fma(qr[4 * d4 + 2], static_cast<double>(kv.z), acc);
        acc = fma(qr[4 * d4 + 3], static_cast<double>(kv.w), acc);
      }
      slog[w * Ck + j0 + lane] = acc * scale;
    }
  }
  __syncthreads();
  // phase 2: one warp per row
  if (w >= nrows) return;
  const size_t row_id = static_cast<size_t>(h) * Cq + i0 + w;
  if (n_q[row_id] <= 0) {
    if (lane == 0) sel_count[row_id] = 0;
    return;
  }
  const int32_t *nkh = n_k + static_cast<size_t>(h) * Ck;
  const double *lg = slog + w * Ck;
  double wt[CPL];
  int nk[CPL];
  double mx = -INFINITY;
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    const int j = c * 32 + lane;
    nk[c] = j < Ck ? nkh[j] : 0;
    wt[c] = j < Ck ? lg[j] : 0.0;
    if (nk[c] > 0) mx = fmax(mx, wt[c]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  double part = 0.0;
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    wt[c] = nk[c] > 0 ? static_cast<double>(nk[c]) * exp(wt[c] - mx) : 0.0;
    part += wt[c];
  }
  uint32_t keep = 0;   // bit c: cluster c * 32 + lane is kept
  if (p >= 1.f) {
#pragma unroll
    for (int c = 0; c < CPL; ++c) keep |= (nk[c] > 0 ? 1u : 0u) << c;
  } else if (mx != -INFINITY) {
    const double target = static_cast<double>(p) * warp_sum_bcast(part);
    uint64_t key[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) key[c] = nk[c] > 0 ? select_key(wt[c], c * 32 + lane) : 0ull;
    uint64_t t = 0;
    for (int b = 62; b >= 0; --b) {   // live keys are positive doubles: bit 63 is clear
      const uint64_t cand = t | (1ull << b);
      double f = 0.0;
#pragma unroll
      for (int c = 0; c < CPL; ++c) f += key[c] >= cand ? wt[c] : 0.0;
      if (warp_sum_bcast(f) >= target) t = cand;
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) keep |= (nk[c] > 0 && key[c] >= t ? 1u : 0u) << c;
  }
  int32_t *out = sel_cols + row_id * Ck;
  int pos = 0;
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    const bool s = (keep >> c) & 1u;
    const unsigned m = __ballot_sync(0xffffffffu, s);
    if (s) out[pos + __popc(m & ((1u << lane) - 1u))] = c * 32 + lane;
    pos += __popc(m);
  }
  if (lane == 0) sel_count[row_id] = pos;
}

inline size_t select_smem_bytes(int D, int Ck) {
  return (static_cast<size_t>(kSelRows) * D + static_cast<size_t>(kSelRows) * Ck) * sizeof(double) +
         static_cast<size_t>(kSelChunk) * (D + 4) * sizeof(float);
}

// k-clusters per lane for a given Ck (the kernel template parameter).
inline int select_cpl(int Ck) {
  const int c = (Ck + 31) / 32;
  return c <= 4 ? 4 : c <= 8 ? 8 : c <= 16 ? 16 : 32;
}

}  // namespace svg
