// k-means update step (Sparse VideoGen2, section 2(a) "Clustering"; the
// initial centroids of a warm start come from section 2(c) "Centroid cache").
//
// One Lloyd round = assign (kmeans_tc.cuh) + stable counting sort (sort.cuh)
// + update:  mu_c = (sum of the rows assigned to c) / n_c; an empty cluster
// keeps mu_c.  Rows are summed in fp64.  Every input is a bf16 value (8
// significant bits, magnitudes far inside fp64's range), so every partial sum
// is exact in fp64 and the result does not depend on the summation order: the
// parallel atomic accumulation below gives the exact mean, rounded once to
// fp32, on every run.
#pragma once
#include "common.cuh"
#include "sort.cuh"

namespace svg {

constexpr int kAccumRowsPerWarp = 64;

// Per warp: kAccumRowsPerWarp consecutive rows of the permuted order of one
// head; lanes own D/32 channels; runs of equal cluster id are summed in
// registers and flushed with fp64 atomics into sums [BH, C, D].
template <int D>
__global__ void __launch_bounds__(256) kmeans_accum_kernel(const __nv_bfloat16 *__restrict__ x,
                                                           int N, int C,
                                                           const int32_t *__restrict__ perm,
                                                           const int32_t *__restrict__ assign,
                                                           double *__restrict__ sums) {
  constexpr int PER = D / 32;
  const int h = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int seg = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int r0 = seg * kAccumRowsPerWarp;
  if (r0 >= N) return;
  const int r1 = min(N, r0 + kAccumRowsPerWarp);
  const int32_t *p = perm + static_cast<size_t>(h) * N;
  const int32_t *a = assign + static_cast<size_t>(h) * N;
  const __nv_bfloat16 *xh = x + static_cast<size_t>(h) * N * D;
  double *sh = sums + static_cast<size_t>(h) * C * D + lane * PER;
  double acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.0;
  int cur = -1;
  for (int g = r0; g < r1; g += 32) {
    const int n = g + lane < r1 ? p[g + lane] : 0;
    const int cid = g + lane < r1 ? a[n] : -1;
    const int cnt = min(32, r1 - g);
    for (int j = 0; j < cnt; j += 4) {
      float v[4][PER];
      int cj[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = __shfl_sync(0xffffffffu, n, (j + u) & 31);
        cj[u] = __shfl_sync(0xffffffffu, cid, (j + u) & 31);
        if (j + u >= cnt) cj[u] = -1;
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
      for (int u = 0; u < 4; ++u) {
        if (cj[u] < 0) continue;            // warp-uniform
        if (cj[u] != cur) {
          if (cur >= 0)
#pragma unroll
            for (int e = 0; e < PER; ++e) atomicAdd(sh + static_cast<size_t>(cur) * D + e, acc[e]);
#pragma unroll
          for (int e = 0; e < PER; ++e) acc[e] = 0.0;
          cur = cj[u];
        }
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += static_cast<double>(v[u][e]);
      }
    }
  }
  if (cur >= 0)
#pragma unroll
    for (int e = 0; e < PER; ++e) atomicAdd(sh + static_cast<size_t>(cur) * D + e, acc[e]);
}

// One warp per cluster: mu = sums / n (or unchanged when n = 0), refreshed
// bf16 hi/lo split and squared norm for the next assign step (rows of a head
// are Cpad apart there), sums cleared for the next round.
template <int D>
__global__ void __launch_bounds__(256) kmeans_finalize_kernel(int C, int Cpad,
                                                              const int32_t *__restrict__ offsets,
                                                              double *__restrict__ sums,
                                                              float *__restrict__ mu,
                                                              __nv_bfloat16 *__restrict__ hi,
                                                              __nv_bfloat16 *__restrict__ lo,
                                                              float *__restrict__ norms) {
  constexpr int PER = D / 32;
  const int h = blockIdx.y;
  const int c = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (c >= C) return;
  const int cnt = offsets[static_cast<size_t>(h) * (C + 1) + c + 1] -
                  offsets[static_cast<size_t>(h) * (C + 1) + c];
  double *sm = sums + (static_cast<size_t>(h) * C + c) * D + lane * PER;
  float *m = mu + (static_cast<size_t>(h) * C + c) * D + lane * PER;
  const size_t srow = (static_cast<size_t>(h) * Cpad + c) * D + lane * PER;
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const float out = cnt > 0 ? static_cast<float>(sm[e] / cnt) : m[e];
    sm[e] = 0.0;
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
