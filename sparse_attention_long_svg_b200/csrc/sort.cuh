// Stable counting sort of the tokens of every head by cluster id
// (Sparse VideoGen2, section 2(a) "Permutation": clusters become contiguous,
// tokens keep ascending order inside a cluster).
//
// Three passes over the int32 assignment [BH, N]:
//   1. sort_hist:    per chunk of kChunk tokens, a histogram of cluster ids
//   2. sort_scan:    per head, exclusive scan over chunks (per cluster) and
//                    over clusters -> cluster offsets and per-chunk bases
//   3. sort_scatter: one warp per chunk walks its tokens in order, ranks
//                    equal ids inside each 32-token group with a warp match
//                    and writes perm[offset + base + rank] = token
// Scratch (caller workspace): chunk counts/bases [BH, nchunks, C] int32.
#pragma once
#include "common.cuh"

namespace svg {

constexpr int kChunk = 1024;   // tokens per histogram chunk
constexpr int kMaxClusters = 1024;

__host__ __device__ inline int num_chunks(int N) { return (N + kChunk - 1) / kChunk; }

__global__ void __launch_bounds__(256) sort_hist_kernel(const int32_t *__restrict__ assign, int N,
                                                        int C, int32_t *__restrict__ chunk_cnt) {
  __shared__ int hist[kMaxClusters];
  const int h = blockIdx.y, chunk = blockIdx.x, nch = gridDim.x;
  for (int c = threadIdx.x; c < C; c += blockDim.x) hist[c] = 0;
  __syncthreads();
  const int n0 = chunk * kChunk, n1 = min(N, n0 + kChunk);
  const int32_t *a = assign + static_cast<size_t>(h) * N;
  for (int n = n0 + threadIdx.x; n < n1; n += blockDim.x) {
    int c = a[n];
    if (c < 0 || c >= C) {
      record_error(SVG_ERR_DEVICE_CHECK, SITE_PERMUTE_RANGE);
      continue;
    }
    atomicAdd(&hist[c], 1);
  }
  __syncthreads();
  int32_t *out = chunk_cnt + (static_cast<size_t>(h) * nch + chunk) * C;
  for (int c = threadIdx.x; c < C; c += blockDim.x) out[c] = hist[c];
}

// One block of 1024 threads per head; thread c owns cluster c.
// chunk_cnt is rewritten in place with each chunk's first output row for
// cluster c (cluster offset + rows of that cluster in earlier chunks).
__global__ void __launch_bounds__(1024) sort_scan_kernel(int32_t *__restrict__ chunk_cnt, int N,
                                                         int C, int nch,
                                                         int32_t *__restrict__ offsets) {
  __shared__ int warp_tot[32];
  const int h = blockIdx.x, c = threadIdx.x;
  int32_t *cc = chunk_cnt + static_cast<size_t>(h) * nch * C;
  int total = 0;
  if (c < C) {
    for (int k0 = 0; k0 < nch; k0 += 8) {   // eight loads in flight, then the running sum
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = k0 + u < nch ? cc[static_cast<size_t>(k0 + u) * C + c] : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (k0 + u < nch) cc[static_cast<size_t>(k0 + u) * C + c] = total;
        total += v[u];
      }
    }
  }
  // exclusive scan of totals over clusters
  const int lane = c & 31, w = c >> 5;
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    int t = warp_tot[lane];
    int ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    warp_tot[lane] = ti - t;  // exclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = warp_tot[w] + incl - total;
  if (c < C) {
    offsets[static_cast<size_t>(h) * (C + 1) + c] = excl;
    for (int k0 = 0; k0 < nch; k0 += 8) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = k0 + u < nch ? cc[static_cast<size_t>(k0 + u) * C + c] : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (k0 + u < nch) cc[static_cast<size_t>(k0 + u) * C + c] = v[u] + excl;
    }
  }
  if (c == 0) offsets[static_cast<size_t>(h) * (C + 1) + C] = N;
}

// One warp per chunk: stable ranks inside each 32-token group via match_any.
// The chunk's ids are loaded up front (kChunk / 32 per lane), so the ordered
// walk over the groups waits on no global load.
__global__ void __launch_bounds__(32) sort_scatter_kernel(const int32_t *__restrict__ assign,
                                                          int N, int C,
                                                          const int32_t *__restrict__ chunk_base,
                                                          int32_t *__restrict__ perm) {
  __shared__ int cursor[kMaxClusters];
  const int h = blockIdx.y, chunk = blockIdx.x, nch = gridDim.x;
  const int lane = threadIdx.x;
  const int32_t *base = chunk_base + (static_cast<size_t>(h) * nch + chunk) * C;
  for (int c = lane; c < C; c += 32) cursor[c] = base[c];
  __syncwarp();
  const int32_t *a = assign + static_cast<size_t>(h) * N;
  int32_t *p = perm + static_cast<size_t>(h) * N;
  const int n0 = chunk * kChunk, n1 = min(N, n0 + kChunk);
  const unsigned lt = (1u << lane) - 1u;
  int ids[kChunk / 32];
#pragma unroll
  for (int gi = 0; gi < kChunk / 32; ++gi) {
    const int n = n0 + gi * 32 + lane;
    ids[gi] = n < n1 ? a[n] : -1;
  }
#pragma unroll
  for (int gi = 0; gi < kChunk / 32; ++gi) {
    const int g = n0 + gi * 32;
    if (g >= n1) break;
    const int n = g + lane;
    int c = ids[gi];
    const bool ok = (c >= 0 && c < C);
    const unsigned live = __ballot_sync(0xffffffffu, ok);
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? c : -1) & live;
    if (ok) {
      const int rank = __popc(peers & lt);
      p[cursor[c] + rank] = n;
    }
    __syncwarp();
    if (ok && (peers >> lane) == 1u) cursor[c] += __popc(peers);  // highest peer updates
    __syncwarp();
  }
}

// ------------------------------------------------------------------ row moves
// Row gather (permute) / scatter (un-permute) of bf16 [BH, N, D] tensors with
// 16-byte vectors.  Every thread moves kVecPerThread vectors per tensor.
constexpr int kVecPerThread = 4;

struct RowMoveArgs {
  const uint4 *src[3];
  uint4 *dst[3];
};

template <bool kGather>
__global__ void __launch_bounds__(256) row_move_kernel(RowMoveArgs args, int ntensors,
                                                       const int32_t *__restrict__ perm, int BH,
                                                       int N, int vec_per_row) {
  const size_t total = static_cast<size_t>(BH) * N * vec_per_row;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x * kVecPerThread;
  for (size_t base = (static_cast<size_t>(blockIdx.x) * blockDim.x) * kVecPerThread + threadIdx.x;
       base < total; base += stride) {
    size_t src_idx[kVecPerThread], dst_idx[kVecPerThread];
    bool ok[kVecPerThread];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const size_t v = base + static_cast<size_t>(u) * blockDim.x;
      ok[u] = v < total;
      src_idx[u] = dst_idx[u] = 0;
      if (ok[u]) {
        const size_t row = v / vec_per_row;
        const int col = static_cast<int>(v - row * vec_per_row);
        const size_t h = row / N;
        const int r = static_cast<int>(row - h * N);
        const int t = perm[row];
        if (t < 0 || t >= N) {
          record_error(SVG_ERR_DEVICE_CHECK, SITE_PERMUTE_RANGE);
          ok[u] = false;
          continue;
        }
        const size_t moved = (h * N + t) * vec_per_row + col;
        const size_t fixed = (h * N + r) * vec_per_row + col;
        src_idx[u] = kGather ? moved : fixed;
        dst_idx[u] = kGather ? fixed : moved;
      }
    }
    for (int t = 0; t < ntensors; ++t) {
      uint4 val[kVecPerThread];
#pragma unroll
      for (int u = 0; u < kVecPerThread; ++u)
        if (ok[u]) val[u] = __ldcs(args.src[t] + src_idx[u]);
#pragma unroll
      for (int u = 0; u < kVecPerThread; ++u)
        if (ok[u]) __stcs(args.dst[t] + dst_idx[u], val[u]);
    }
  }
}

}  // namespace svg
