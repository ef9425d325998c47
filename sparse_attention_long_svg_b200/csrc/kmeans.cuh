// k-means update step (Sparse VideoGen2, section 2(a) "Clustering"; the
// initial centroids of a warm start come from section 2(c) "Centroid cache").
//
// One Lloyd round = assign (kmeans_tc.cuh) + stable counting sort (sort.cuh)
// + update:  mu_c = (sum of the rows assigned to c) / n_c; an empty cluster
// keeps mu_c.  Rows are summed in fp64.  Every input is a bf16 value (8
// significant bits, magnitudes far inside fp64's range), so every partial sum
// is exact in fp64 and the result does not depend on the summation order:
// the two-level reduction below gives the exact mean, rounded once to fp32.
//
// Level 1 (kmeans_accum_kernel): after the sort every cluster is a contiguous
// range of permuted rows; it is cut into chunks of at most kAccumRows rows
// (chunk starts per cluster come from sort_scan_kernel) and one warp sums one
// chunk into its own fp64 partial row.  No atomics.
// Level 2 (kmeans_finalize_kernel): one warp per cluster adds its partials.
#pragma once
#include "common.cuh"
#include "sort.cuh"

namespace svg {

constexpr int kAccumRows = 64;

__host__ __device__ inline int max_accum_chunks(int N, int C) {
  return (N + kAccumRows - 1) / kAccumRows + C;
}

// grid (ceil(max_accum_chunks / 8), BH), 256 threads: warp j of a head sums
// chunk j.  partial [BH, max_accum_chunks, D] fp64.
template <int D>
__global__ void __launch_bounds__(256) kmeans_accum_kernel(const __nv_bfloat16 *__restrict__ x,
                                                           int N, int C,
                                                           const int32_t *__restrict__ perm,
                                                           const int32_t *__restrict__ offsets,
                                                           const int32_t *__restrict__ row_chunks,
                                                           double *__restrict__ partial) {
  constexpr int PER = D / 32;
  __shared__ int s_rc[kMaxClusters + 1];
  const int h = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int32_t *rc = row_chunks + static_cast<size_t>(h) * (C + 1);
  for (int c = threadIdx.x; c <= C; c += blockDim.x) s_rc[c] = rc[c];
  __syncthreads();
  const int j = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (j >= s_rc[C]) return;
  // cluster of chunk j: the last c with s_rc[c] <= j (clusters with no rows own no chunk)
  int lo = 0, hi = C - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_rc[mid] <= j) lo = mid; else hi = mid - 1;
  }
  const int c = lo;
  const int c0 = offsets[static_cast<size_t>(h) * (C + 1) + c];
  const int c1 = offsets[static_cast<size_t>(h) * (C + 1) + c + 1];
  const int r0 = c0 + (j - s_rc[c]) * kAccumRows;
  const int r1 = min(c1, r0 + kAccumRows);
  const int32_t *p = perm + static_cast<size_t>(h) * N;
  const __nv_bfloat16 *xh = x + static_cast<size_t>(h) * N * D;
  double acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.0;
  for (int g = r0; g < r1; g += 32) {
    const int n = g + lane < r1 ? p[g + lane] : 0;
    const int cnt = min(32, r1 - g);
    for (int jj = 0; jj < cnt; jj += 8) {
      float v[8][PER];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int t = __shfl_sync(0xffffffffu, n, (jj + u) & 31);
        const __nv_bfloat16 *row = xh + static_cast<size_t>(t) * D + lane * PER;
        if constexpr (PER == 4) {
          const uint2 raw = *reinterpret_cast<const uint2 *>(row);
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
          v[u][0] = f0.x; v[u][1] = f0.y; v[u][2] = f1.x; v[u][3] = f1.y;
        } else {
          const uint32_t raw = *reinterpret_cast<const uint32_t *>(row);
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw));
          v[u][0] = f0.x; v[u][1] = f0.y;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (jj + u < cnt)                 // warp-uniform
#pragma unroll
          for (int e = 0; e < PER; ++e) acc[e] += static_cast<double>(v[u][e]);
    }
  }
  double *out = partial + (static_cast<size_t>(h) * max_accum_chunks(N, C) + j) * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; ++e) out[e] = acc[e];
}

// One warp per cluster: mu = (sum of its partials) / n (or unchanged when
// n = 0), refreshed bf16 hi/lo split and squared norm for the next assign step
// (rows of a head are Cpad apart there).
// Also clears the near-tie counter for the next assign step.
template <int D>
__global__ void __launch_bounds__(256) kmeans_finalize_kernel(int N, int C, int Cpad,
                                                              const int32_t *__restrict__ offsets,
                                                              const int32_t *__restrict__ row_chunks,
                                                              const double *__restrict__ partial,
                                                              float *__restrict__ mu,
                                                              __nv_bfloat16 *__restrict__ hi,
                                                              __nv_bfloat16 *__restrict__ lo,
                                                              float *__restrict__ norms,
                                                              int32_t *__restrict__ num_ties) {
  constexpr int PER = D / 32;
  const int h = blockIdx.y;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *num_ties = 0;
  const int c = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (c >= C) return;
  const int cnt = offsets[static_cast<size_t>(h) * (C + 1) + c + 1] -
                  offsets[static_cast<size_t>(h) * (C + 1) + c];
  const int j0 = row_chunks[static_cast<size_t>(h) * (C + 1) + c];
  const int j1 = row_chunks[static_cast<size_t>(h) * (C + 1) + c + 1];
  const double *pp = partial + static_cast<size_t>(h) * max_accum_chunks(N, C) * D + lane * PER;
  double acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.0;
  for (int j = j0; j < j1; ++j)
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] += pp[static_cast<size_t>(j) * D + e];
  float *m = mu + (static_cast<size_t>(h) * C + c) * D + lane * PER;
  const size_t srow = (static_cast<size_t>(h) * Cpad + c) * D + lane * PER;
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const float out = cnt > 0 ? static_cast<float>(acc[e] / cnt) : m[e];
    m[e] = out;
    s = fmaf(out, out, s);
    const __nv_bfloat16 vh = __float2bfloat16_rn(out);
    hi[srow + e] = vh;
    lo[srow + e] = __float2bfloat16_rn(out - __bfloat162float(vh));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) norms[static_cast<size_t>(h) * Cpad + c] = s;
}

}  // namespace svg
