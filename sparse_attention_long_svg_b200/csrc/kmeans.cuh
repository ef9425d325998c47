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
// kmeans_accum_kernel: one warp per chunk sums its rows in fp64; a cluster
//   with one chunk is finalised at once, otherwise the last of its chunks to
//   arrive adds the chunks' partial sums and finalises.  Finalising writes the
//   new fp32 centroid, its bf16 hi/lo split and squared norm for the next
//   assign step, and clears the cluster's counters for the next round.
#pragma once
#include "common.cuh"
#include "sort.cuh"

namespace svg {

constexpr int kAccumRows = 128;
constexpr int kBucketTokens = 4;   // tokens per thread of the bucket kernel

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

// grid (ceil(N / (1024 * kBucketTokens)), BH), 1024 threads; thread t of a
// block takes tokens base + t + 1024 k, k < kBucketTokens.
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
  const int32_t *ah = assign + static_cast<size_t>(h) * N;
  const int n_base = blockIdx.x * blockDim.x * kBucketTokens + t;
  int a[kBucketTokens];
#pragma unroll
  for (int k = 0; k < kBucketTokens; ++k) {   // issued before the scan so they overlap it
    const int n = n_base + k * static_cast<int>(blockDim.x);
    a[k] = n < N ? ah[n] : -1;
  }
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
  int base[kBucketTokens];
  unsigned peers[kBucketTokens];
#pragma unroll
  for (int k = 0; k < kBucketTokens; ++k) {    // reserve: one atomic per cluster of a warp
    const int n = n_base + k * static_cast<int>(blockDim.x);
    const bool ok = a[k] >= 0 && a[k] < C;
    if (n < N && !ok) record_error(SVG_ERR_DEVICE_CHECK, SITE_KMEANS_RANGE);
    const unsigned live = __ballot_sync(0xffffffffu, ok);
    peers[k] = 0;
    base[k] = 0;
    if (ok) {
      peers[k] = __match_any_sync(live, a[k]);
      if (lane == __ffs(peers[k]) - 1)
        base[k] = atomicAdd(cursor + static_cast<size_t>(h) * C + a[k], __popc(peers[k]));
    }
  }
#pragma unroll
  for (int k = 0; k < kBucketTokens; ++k) {    // place
    const bool ok = peers[k] != 0;
    const unsigned live = __ballot_sync(0xffffffffu, ok);
    if (ok) {
      const int b0 = __shfl_sync(live, base[k], __ffs(peers[k]) - 1);
      const int pos = s_off[a[k]] + b0 + __popc(peers[k] & ((1u << lane) - 1u));
      if (pos < N) {
        bucket[static_cast<size_t>(h) * N + pos] = n_base + k * static_cast<int>(blockDim.x);
      } else {
        record_error(SVG_ERR_DEVICE_CHECK, SITE_KMEANS_RANGE);   // sizes and assignment disagree
      }
    }
  }
}

// Writes cluster c's new centroid from its fp64 row sum: lanes l < D/8 hold
// channels 8l .. 8l+7 of the sum.  Also clears the cluster's counters.
template <int D>
__device__ __forceinline__ void kmeans_finalize_cluster(const double (&sum)[8], int lane, int h,
                                                        int c, int C, int Cpad, int n_c,
                                                        float *__restrict__ mu,
                                                        __nv_bfloat16 *__restrict__ hi,
                                                        __nv_bfloat16 *__restrict__ lo,
                                                        float *__restrict__ norms,
                                                        int32_t *__restrict__ counts_ws,
                                                        int32_t *__restrict__ cursor) {
  constexpr int LPR = D / 8;
  float sq = 0.f;
  if (lane < LPR) {
    float out[8];
    uint32_t hp[4], lp[4];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      out[e] = static_cast<float>(sum[e] / n_c);
      sq = fmaf(out[e], out[e], sq);
    }
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(out[e]), h1 = __float2bfloat16_rn(out[e + 1]);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(out[e] - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(out[e + 1] - __bfloat162float(h1));
      hp[e / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
      lp[e / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
    }
    float4 *m = reinterpret_cast<float4 *>(mu + (static_cast<size_t>(h) * C + c) * D + lane * 8);
    m[0] = make_float4(out[0], out[1], out[2], out[3]);
    m[1] = make_float4(out[4], out[5], out[6], out[7]);
    const size_t srow = (static_cast<size_t>(h) * Cpad + c) * D + lane * 8;
    *reinterpret_cast<uint4 *>(hi + srow) = make_uint4(hp[0], hp[1], hp[2], hp[3]);
    *reinterpret_cast<uint4 *>(lo + srow) = make_uint4(lp[0], lp[1], lp[2], lp[3]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if (lane == 0) {
    norms[static_cast<size_t>(h) * Cpad + c] = sq;
    counts_ws[static_cast<size_t>(h) * C + c] = 0;    // counters of the next round
    cursor[static_cast<size_t>(h) * C + c] = 0;
  }
}

// grid (ceil(max_accum_chunks(N, C) / kAccumWarps), BH), 32 kAccumWarps
// threads: warp w of block b sums chunk j = kAccumWarps b + w.  One-warp blocks:
// chunk lengths vary and a block holds its SM slot until its longest warp
// ends.  A row is D/8 lanes x 16 bytes; a warp load covers
// 32 / (D/8) rows, UNROLL loads are in flight.  Lane l keeps channels
// 8 (l % (D/8)) .. +7 in fp64.
constexpr int kAccumWarps = 1;

template <int D>
__global__ void __launch_bounds__(32 * kAccumWarps) kmeans_accum_kernel(
    const __nv_bfloat16 *__restrict__ x, int N, int C, int Cpad, const int32_t *__restrict__ bucket,
    const int32_t *__restrict__ offsets, const KmChunk *__restrict__ chunks,
    const int32_t *__restrict__ num_chunks, double *__restrict__ partial,
    int32_t *__restrict__ arrive, int32_t *__restrict__ counts_ws, int32_t *__restrict__ cursor,
    float *__restrict__ mu, __nv_bfloat16 *__restrict__ hi, __nv_bfloat16 *__restrict__ lo,
    float *__restrict__ norms, int32_t *__restrict__ num_ties) {
  constexpr int LPR = D / 8;           // lanes per row
  constexpr int RPL = 32 / LPR;        // rows per warp load
  constexpr int UNROLL = 8;
  constexpr int STEP = RPL * UNROLL;   // rows per iteration
  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * kAccumWarps + warp;
  if (j == 0 && h == 0 && lane == 0) *num_ties = 0;   // the refine step of this round is done
  if (j >= num_chunks[h]) return;
  const int maxch = max_accum_chunks(N, C);
  const KmChunk ch = chunks[static_cast<size_t>(h) * maxch + j];
  const int c = ch.c;
  const int32_t *b = bucket + static_cast<size_t>(h) * N + ch.r0;
  const int len = ch.r1 - ch.r0;
  const int sub = lane / LPR, q = lane % LPR;
  const uint4 *xh = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(h) * N * D) + q;
  double sum[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) sum[e] = 0.0;
  for (int r = 0; r < len; r += STEP) {
    const int id = r + lane < len ? b[r + lane] : -1;   // STEP <= 32 row ids, one per lane
    uint4 v[UNROLL];
    bool ok[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int t = __shfl_sync(0xffffffffu, id, u * RPL + sub);
      ok[u] = t >= 0;
      v[u] = ok[u] ? __ldg(xh + static_cast<size_t>(t) * LPR) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      if (!ok[u]) continue;
      const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&v[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p2[e]);
        sum[2 * e] += static_cast<double>(f.x);
        sum[2 * e + 1] += static_cast<double>(f.y);
      }
    }
  }
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) sum[e] += __shfl_xor_sync(0xffffffffu, sum[e], o);
  const int n_c = offsets[static_cast<size_t>(h) * (C + 1) + c + 1] -
                  offsets[static_cast<size_t>(h) * (C + 1) + c];
  const int nch = (n_c + kAccumRows - 1) / kAccumRows;
  if (nch > 1) {
    double *part = partial + static_cast<size_t>(h) * maxch * D;
    if (lane < LPR) {
      double2 *dst = reinterpret_cast<double2 *>(part + static_cast<size_t>(j) * D + lane * 8);
#pragma unroll
      for (int e = 0; e < 4; ++e) dst[e] = make_double2(sum[2 * e], sum[2 * e + 1]);
    }
    __threadfence();
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atomicAdd(arrive + static_cast<size_t>(h) * C + c, 1) == nch - 1;
    if (!__shfl_sync(0xffffffffu, last, 0)) return;
    __threadfence();
    if (lane < LPR) {
#pragma unroll
      for (int e = 0; e < 8; ++e) sum[e] = 0.0;
      for (int k = 0; k < nch; ++k) {
        const double2 *src =
            reinterpret_cast<const double2 *>(part + static_cast<size_t>(ch.j0 + k) * D + lane * 8);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double2 d2 = __ldcg(src + e);
          sum[2 * e] += d2.x;
          sum[2 * e + 1] += d2.y;
        }
      }
    }
    if (lane == 0) arrive[static_cast<size_t>(h) * C + c] = 0;
  }
  kmeans_finalize_cluster<D>(sum, lane, h, c, C, Cpad, n_c, mu, hi, lo, norms, counts_ws, cursor);
}

}  // namespace svg
