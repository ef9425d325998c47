// k-means update step (Sparse VideoGen2, section 2(a) "Clustering"; the
// initial centroids of a warm start come from section 2(c) "Centroid cache").
//
// One Lloyd round = assign (kmeans_tc.cuh, which also counts the members of
// every cluster) + update:  mu_c = (sum of the rows assigned to c) / n_c; an
// empty cluster keeps mu_c.  Rows are summed in fp64.  Every input is a bf16
// value (8 significant bits); as long as the magnitudes in one channel of one
// cluster span fewer than about 2^28 (far more than activations do), every
// partial sum is exact in fp64 and the result does not depend on the
// summation order: the reduction below gives the exact mean, rounded once to
// fp32, whatever order the rows arrive in.  That is why no step here needs a
// stable order (the stable permutation is built once, after the last round).
//
// kmeans_bucket_kernel: offsets of the clusters from their sizes, then every
//   token is appended to its cluster's range of a bucket list (warp-aggregated
//   atomic cursors, so the order inside a cluster is arbitrary).  The first
//   block of each head also publishes the offsets, the sizes and a table of
//   accumulation chunks (at most kAccumRows rows of one cluster each).
// kmeans_accum_kernel: one block per chunk sums its rows in fp64; a cluster
//   with one chunk is finalised at once, otherwise the last of its chunks to
//   arrive adds the chunks' partial sums and finalises.  Finalising writes the
//   new fp32 centroid, its bf16 hi/lo split and squared norm for the next
//   assign step, and clears the cluster's counters for the next round.
#pragma once
#include "common.cuh"
#include "sort.cuh"

namespace svg {

constexpr int kAccumRows = 256;

__host__ __device__ inline int max_accum_chunks(int N, int C) {
  return (N + kAccumRows - 1) / kAccumRows + C;
}

// One accumulation chunk: rows [r0, r1) of the bucket list, all in cluster c,
// whose first chunk has index j0.
struct KmChunk {
  int32_t c, r0, r1, j0;
};

// Exclusive prefix sum over the threads of a 1024-thread block (one value per
// thread); *total receives the sum.  warp_tot: 32 ints of shared memory.
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int t = lane < static_cast<int>(blockDim.x >> 5) ? warp_tot[lane] : 0;
    int ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    warp_tot[lane] = ti - t;
    if (lane == 31) *total = ti;
  }
  __syncthreads();
  const int r = warp_tot[w] + incl - v;
  __syncthreads();   // warp_tot may be reused by the caller
  return r;
}

// grid (ceil(N / 1024), BH), 1024 threads.
// counts [BH, C]: sizes of this round's clusters (from the assign step);
// cursor [BH, C]: zero on entry, the sizes on exit.
__global__ void __launch_bounds__(1024) kmeans_bucket_kernel(
    const int32_t *__restrict__ assign, int N, int C, const int32_t *__restrict__ counts,
    int32_t *__restrict__ cursor, int32_t *__restrict__ bucket, int32_t *__restrict__ offsets,
    int32_t *__restrict__ counts_out, KmChunk *__restrict__ chunks,
    int32_t *__restrict__ num_chunks) {
  __shared__ int s_off[kMaxClusters];
  __shared__ int warp_tot[32];
  __shared__ int s_total;
  const int h = blockIdx.y, t = threadIdx.x, lane = t & 31;
  const int cnt = t < C ? counts[static_cast<size_t>(h) * C + t] : 0;
  const int excl = block_exclusive_scan(cnt, warp_tot, &s_total);
  if (t < C) s_off[t] = excl;
  if (blockIdx.x == 0) {
    const int total = s_total;
    if (t < C) {
      offsets[static_cast<size_t>(h) * (C + 1) + t] = excl;
      counts_out[static_cast<size_t>(h) * C + t] = cnt;
    }
    if (t == 0) offsets[static_cast<size_t>(h) * (C + 1) + C] = total;
    const int nck = (cnt + kAccumRows - 1) / kAccumRows;
    const int j0 = block_exclusive_scan(nck, warp_tot, &s_total);
    KmChunk *tab = chunks + static_cast<size_t>(h) * max_accum_chunks(N, C);
    for (int k = 0; k < nck; ++k)
      tab[j0 + k] = KmChunk{t, excl + k * kAccumRows, min(excl + cnt, excl + (k + 1) * kAccumRows), j0};
    if (t == 0) num_chunks[h] = s_total;
  }
  __syncthreads();
  const int n = blockIdx.x * blockDim.x + t;
  const int a = n < N ? assign[static_cast<size_t>(h) * N + n] : -1;
  const bool ok = a >= 0 && a < C;
  if (n < N && !ok) record_error(SVG_ERR_DEVICE_CHECK, SITE_KMEANS_RANGE);
  const unsigned live = __ballot_sync(0xffffffffu, ok);
  if (ok) {
    const unsigned peers = __match_any_sync(live, a);
    const int leader = __ffs(peers) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(cursor + static_cast<size_t>(h) * C + a, __popc(peers));
    base = __shfl_sync(live, base, leader);
    const int pos = s_off[a] + base + __popc(peers & ((1u << lane) - 1u));
    if (pos < N) {
      bucket[static_cast<size_t>(h) * N + pos] = n;
    } else {
      record_error(SVG_ERR_DEVICE_CHECK, SITE_KMEANS_RANGE);   // sizes and assignment disagree
    }
  }
}

// grid (max_accum_chunks(N, C), BH), 256 threads (8 warps).
template <int D>
__global__ void __launch_bounds__(256) kmeans_accum_kernel(
    const __nv_bfloat16 *__restrict__ x, int N, int C, int Cpad, const int32_t *__restrict__ bucket,
    const int32_t *__restrict__ offsets, const KmChunk *__restrict__ chunks,
    const int32_t *__restrict__ num_chunks, double *__restrict__ partial,
    int32_t *__restrict__ arrive, int32_t *__restrict__ counts_ws, int32_t *__restrict__ cursor,
    float *__restrict__ mu, __nv_bfloat16 *__restrict__ hi, __nv_bfloat16 *__restrict__ lo,
    float *__restrict__ norms, int32_t *__restrict__ num_ties) {
  constexpr int PER = D / 32;
  constexpr int WARPS = 8, UNROLL = 8;
  __shared__ double s_red[WARPS][D];
  __shared__ float s_sq[D / 32];
  __shared__ int s_last;
  const int h = blockIdx.y, j = blockIdx.x;
  if (j == 0 && h == 0 && threadIdx.x == 0) *num_ties = 0;   // the refine step of this round is done
  if (j >= num_chunks[h]) return;
  const int maxch = max_accum_chunks(N, C);
  const KmChunk ch = chunks[static_cast<size_t>(h) * maxch + j];
  const int c = ch.c;
  const int n_c = offsets[static_cast<size_t>(h) * (C + 1) + c + 1] -
                  offsets[static_cast<size_t>(h) * (C + 1) + c];
  const int nch = (n_c + kAccumRows - 1) / kAccumRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t *b = bucket + static_cast<size_t>(h) * N + ch.r0;
  const __nv_bfloat16 *xh = x + static_cast<size_t>(h) * N * D + lane * PER;
  const int len = ch.r1 - ch.r0;
  double acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.0;
  // warp w takes rows w, w + 8, w + 16, ...; UNROLL rows in flight per warp
  for (int base = warp; base < len; base += WARPS * UNROLL) {
    int id = -1;
    if (lane < UNROLL && base + WARPS * lane < len) id = b[base + WARPS * lane];
    int ids[UNROLL];
    float v[UNROLL][PER];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      ids[u] = __shfl_sync(0xffffffffu, id, u);
      if (ids[u] >= 0) {                       // warp-uniform
        const __nv_bfloat16 *row = xh + static_cast<size_t>(ids[u]) * D;
        if constexpr (PER == 4) {
          const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(row));
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
          v[u][0] = f0.x; v[u][1] = f0.y; v[u][2] = f1.x; v[u][3] = f1.y;
        } else {
          const uint32_t raw = __ldg(reinterpret_cast<const uint32_t *>(row));
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw));
          v[u][0] = f0.x; v[u][1] = f0.y;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u)
      if (ids[u] >= 0)
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += static_cast<double>(v[u][e]);
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) s_red[warp][lane * PER + e] = acc[e];
  __syncthreads();
  const int d = threadIdx.x;
  double sum = 0.0;
  if (d < D)
#pragma unroll
    for (int w = 0; w < WARPS; ++w) sum += s_red[w][d];
  if (nch > 1) {
    double *part = partial + static_cast<size_t>(h) * maxch * D;
    if (d < D) part[static_cast<size_t>(j) * D + d] = sum;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
      s_last = atomicAdd(arrive + static_cast<size_t>(h) * C + c, 1) == nch - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (d < D) {
      sum = 0.0;
      for (int k = 0; k < nch; ++k) sum += __ldcg(part + static_cast<size_t>(ch.j0 + k) * D + d);
    }
    if (threadIdx.x == 0) arrive[static_cast<size_t>(h) * C + c] = 0;
  }
  // finalise cluster c (n_c >= 1 here)
  float out = 0.f;
  if (d < D) {
    out = static_cast<float>(sum / n_c);
    mu[(static_cast<size_t>(h) * C + c) * D + d] = out;
    const __nv_bfloat16 vh = __float2bfloat16_rn(out);
    const size_t srow = (static_cast<size_t>(h) * Cpad + c) * D + d;
    hi[srow] = vh;
    lo[srow] = __float2bfloat16_rn(out - __bfloat162float(vh));
  }
  float sq = out * out;
#pragma unroll
  for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if (lane == 0 && warp < D / 32) s_sq[warp] = sq;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) s += s_sq[w];
    norms[static_cast<size_t>(h) * Cpad + c] = s;
    counts_ws[static_cast<size_t>(h) * C + c] = 0;    // counters of the next round
    cursor[static_cast<size_t>(h) * C + c] = 0;
  }
}

}  // namespace svg
