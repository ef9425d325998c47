// Centroid-based top-p block selection (Sparse VideoGen2, section 2(b):
// "Centroid approximation" scores cluster pairs through their centroids;
// "Top-p strategy" sorts clusters by estimated score and takes them until
// the cumulative score reaches p).
//
// One block per (head, group of kRowsPerBlock q-clusters).  Phase 1: every
// thread takes k-clusters j and computes the logits of all rows of the group
// (mu_k row read once per block).  Phase 2: one warp per row forms
// w_j = n_kj * exp(logit_j - max), sorts (w desc, j asc) with a bitonic
// network in shared memory, scans the sorted weights and keeps the shortest
// prefix with cumulative weight >= p * total; selected ids are written in
// ascending order.
#pragma once
#include "common.cuh"

namespace svg {

constexpr int kRowsPerBlock = 8;
constexpr int kMaxCk = 1024;

template <int D>
__global__ void __launch_bounds__(256) select_topp_kernel(
    const float *__restrict__ mu_q, const int32_t *__restrict__ n_q, const float *__restrict__ mu_k,
    const int32_t *__restrict__ n_k, int Cq, int Ck, float p, float scale,
    int32_t *__restrict__ sel_count, int32_t *__restrict__ sel_cols) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // layout: q rows [R][D] f32 | logits [R][Ck] f32 | keys [R][pow2(Ck)] u64
  float *sq = reinterpret_cast<float *>(smem_raw);
  float *slog = sq + kRowsPerBlock * D;
  int ck2 = 1;
  while (ck2 < Ck) ck2 <<= 1;
  uint64_t *skey = reinterpret_cast<uint64_t *>(
      smem_raw + ((kRowsPerBlock * D + kRowsPerBlock * Ck) * sizeof(float) + 15) / 16 * 16);

  const int h = blockIdx.y;
  const int i0 = blockIdx.x * kRowsPerBlock;
  const int nrows = min(kRowsPerBlock, Cq - i0);
  for (int t = threadIdx.x; t < kRowsPerBlock * D; t += blockDim.x) {
    const int r = t / D, d = t % D;
    sq[t] = r < nrows ? mu_q[(static_cast<size_t>(h) * Cq + i0 + r) * D + d] : 0.f;
  }
  __syncthreads();
  // phase 1: logits
  const float *mkh = mu_k + static_cast<size_t>(h) * Ck * D;
  for (int j = threadIdx.x; j < Ck; j += blockDim.x) {
    float acc[kRowsPerBlock];
#pragma unroll
    for (int r = 0; r < kRowsPerBlock; ++r) acc[r] = 0.f;
    const float4 *kr = reinterpret_cast<const float4 *>(mkh + static_cast<size_t>(j) * D);
#pragma unroll 4
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 kv = kr[d4];
#pragma unroll
      for (int r = 0; r < kRowsPerBlock; ++r) {
        const float4 qv = reinterpret_cast<const float4 *>(sq + r * D)[d4];
        acc[r] = fmaf(qv.x, kv.x, acc[r]);
        acc[r] = fmaf(qv.y, kv.y, acc[r]);
        acc[r] = fmaf(qv.z, kv.z, acc[r]);
        acc[r] = fmaf(qv.w, kv.w, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kRowsPerBlock; ++r) slog[r * Ck + j] = acc[r] * scale;
  }
  __syncthreads();
  // phase 2: one warp per row
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (w >= nrows) return;
  const int i = i0 + w;
  const size_t row_id = static_cast<size_t>(h) * Cq + i;
  const int32_t *nkh = n_k + static_cast<size_t>(h) * Ck;
  if (n_q[row_id] <= 0) {
    if (lane == 0) sel_count[row_id] = 0;
    return;
  }
  float *lg = slog + w * Ck;
  uint64_t *key = skey + static_cast<size_t>(w) * ck2;
  float mx = -INFINITY;
  int live = 0;
  for (int j = lane; j < Ck; j += 32)
    if (nkh[j] > 0) {
      mx = fmaxf(mx, lg[j]);
      ++live;
    }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    live += __shfl_xor_sync(0xffffffffu, live, o);
  }
  // weights -> sort keys; dead clusters and padding sort last
  for (int j = lane; j < ck2; j += 32) {
    uint64_t kv = ~0ull;
    if (j < Ck && nkh[j] > 0) {
      const float wj = static_cast<float>(nkh[j]) * expf(lg[j] - mx);
      lg[j] = wj;
      kv = (static_cast<uint64_t>(~__float_as_uint(wj)) << 32) | static_cast<uint32_t>(j);
    }
    key[j] = kv;
  }
  __syncwarp();
  for (int kk = 2; kk <= ck2; kk <<= 1) {
    for (int jj = kk >> 1; jj > 0; jj >>= 1) {
      for (int t = lane; t < ck2; t += 32) {
        const int u = t ^ jj;
        if (u > t) {
          const uint64_t a = key[t], b = key[u];
          const bool up = (t & kk) == 0;
          if ((a > b) == up) {
            key[t] = b;
            key[u] = a;
          }
        }
      }
      __syncwarp();
    }
  }
  // inclusive scan of sorted weights; total = sum over live
  int take = live;
  if (p < 1.f && live > 0) {
    float total = 0.f;
    for (int base = 0; base < live; base += 32) {
      const int t = base + lane;
      float v = t < live ? lg[static_cast<uint32_t>(key[t])] : 0.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
      }
      v += total;
      if (t < live) lg[static_cast<uint32_t>(key[t])] = v;  // weight slot now holds the prefix
      total = __shfl_sync(0xffffffffu, v, 31);
    }
    __syncwarp();
    const float thr = p * total;
    int first = live;
    for (int base = 0; base < live; base += 32) {
      const int t = base + lane;
      const bool hit = t < live && lg[static_cast<uint32_t>(key[t])] >= thr;
      const unsigned m = __ballot_sync(0xffffffffu, hit);
      if (m) {
        first = base + __ffs(m) - 1;
        break;
      }
    }
    take = min(live, first + 1);
  }
  // mark the first `take` sorted ids, emit ascending
  __syncwarp();
  for (int j = lane; j < Ck; j += 32) lg[j] = 0.f;
  __syncwarp();
  for (int t = lane; t < take; t += 32) lg[static_cast<uint32_t>(key[t])] = 1.f;
  __syncwarp();
  int32_t *out = sel_cols + row_id * Ck;
  int pos = 0;
  for (int base = 0; base < Ck; base += 32) {
    const int j = base + lane;
    const bool s = j < Ck && lg[j] != 0.f;
    const unsigned m = __ballot_sync(0xffffffffu, s);
    if (s) out[pos + __popc(m & ((1u << lane) - 1u))] = j;
    pos += __popc(m);
  }
  if (lane == 0) sel_count[row_id] = take;
}

inline size_t select_smem_bytes(int D, int Ck) {
  int ck2 = 1;
  while (ck2 < Ck) ck2 <<= 1;
  size_t f = (static_cast<size_t>(kRowsPerBlock) * D + static_cast<size_t>(kRowsPerBlock) * Ck) * 4;
  f = (f + 15) / 16 * 16;
  return f + static_cast<size_t>(kRowsPerBlock) * ck2 * 8;
}

}  // namespace svg
