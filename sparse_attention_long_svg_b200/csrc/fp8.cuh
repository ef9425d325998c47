// E4M3 quantisation of Q and K for the 8-bit Q K^T path of the attention
// kernel.  The page "TurboDiffusion" (section "SageAttention: low-bit
// quantization") runs attention on low-bit quantised operands to cut memory
// traffic and compute; it fixes no format or scale rule.  Here:
//   * E4M3 values (4 exponent bits, bias 7, 3 mantissa bits, largest finite
//     448), rounded to nearest with ties to even, saturating at +-448;
//   * Q: one float32 scale per token row, s = amax|row| / 448 (1 for an
//     all-zero row); K: one float32 scale per head over all its rows, so a key
//     tile gathered from any rows of the head shares it;
//   * the stored value is E4M3(x / s), the division in float32.
// The logits become scale * (q8 . k8) * s_q * s_k; P and V stay bf16.  Rows
// may be gathered through a permutation on the way (output row i of a head
// from source row perm[i]), so the permuted bf16 copies are never written.
#pragma once
#include <cuda_fp8.h>

#include "common.cuh"

namespace svg {

constexpr float kE4m3Max = 448.f;

__device__ __forceinline__ float e4m3_scale(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f;
}

__device__ __forceinline__ uint32_t e4m3_byte(float v, float s) {
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fdiv_rn(v, s), __NV_SATFINITE, __NV_E4M3));
}

// Source row of output row r (r = h * N + i): row i itself, or row perm[r] of
// the same head (gathered); -1 for a permutation entry outside [0, N), which
// is recorded and quantised as a zero row.
__device__ __forceinline__ long long quant_src_row(const int32_t *perm, size_t r, int N) {
  if (perm == nullptr) return static_cast<long long>(r);
  const int t = __ldg(perm + r);
  if (t < 0 || t >= N) {
    record_error(SVG_ERR_DEVICE_CHECK, SITE_PERMUTE_RANGE);
    return -1;
  }
  return static_cast<long long>(r - r % static_cast<size_t>(N)) + t;
}

// Quantisation of rows: each lane converts 8 consecutive channels (one
// 16-byte load), D / 8 lanes a row, so a warp covers 256 / D rows per pass
// and U passes are in flight per iteration.  PER_ROW: the row's amax (by
// shuffles) gives its scale, written to scales[r]; otherwise the head's amax
// is read from amax_bits[r / N].  With perm the source row is gathered.
template <int D, bool PER_ROW>
__global__ void __launch_bounds__(256) quant_e4m3_kernel(const __nv_bfloat16 *__restrict__ x,
                                                         const int32_t *__restrict__ perm, int N, size_t rows,
                                                         const int32_t *__restrict__ amax_bits,
                                                         uint8_t *__restrict__ x8, float *__restrict__ scales) {
  constexpr int LPR = D / 8;           // lanes per row
  constexpr int RPW = 32 / LPR;        // rows per warp pass
  constexpr int U = 4;                 // passes per iteration
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, c = lane % LPR;
  const size_t warp = static_cast<size_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const size_t warps = static_cast<size_t>(gridDim.x) * (blockDim.x >> 5);
  for (size_t r0 = warp * (RPW * U); r0 < rows; r0 += warps * (RPW * U)) {
    long long src[U];
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const size_t r = r0 + i * RPW + sub;
      src[i] = r < rows ? quant_src_row(perm, r, N) : -1;
    }
    uint4 u[U];
#pragma unroll
    for (int i = 0; i < U; ++i)
      u[i] = src[i] >= 0 ? __ldcs(reinterpret_cast<const uint4 *>(x + static_cast<size_t>(src[i]) * D) + c)
                         : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const size_t r = r0 + i * RPW + sub;
      const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
      float v[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&w[j]);
        v[2 * j] = __low2float(b);
        v[2 * j + 1] = __high2float(b);
      }
      float s;
      if constexpr (PER_ROW) {
        float m = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        s = e4m3_scale(m);
      } else {
        s = e4m3_scale(__int_as_float(__ldg(amax_bits + (r < rows ? r / N : 0))));
      }
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        lo |= e4m3_byte(v[e], s) << (8 * e);
        hi |= e4m3_byte(v[4 + e], s) << (8 * e);
      }
      if (r < rows) {
        reinterpret_cast<uint2 *>(x8 + r * D)[c] = make_uint2(lo, hi);
        if (PER_ROW && c == 0) scales[r] = s;
      }
    }
  }
}

// Per-head amax: blocks (chunk, head) reduce 8-channel groups of the head's
// N * D values and fold their maximum into amax_bits[head] (float bits of a
// non-negative value order like integers; amax_bits is zero on entry).
__global__ void __launch_bounds__(256) head_amax_kernel(const __nv_bfloat16 *__restrict__ x, size_t per_head,
                                                        int32_t *__restrict__ amax_bits) {
  const int h = blockIdx.y;
  const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(h) * per_head);
  const size_t groups = per_head / 8;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  float m = 0.f;
  for (size_t g0 = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; g0 < groups; g0 += 4 * stride) {
    uint4 u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const size_t g = g0 + k * stride;
      u[k] = g < groups ? __ldcs(src + g) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&w[i]);
        m = fmaxf(m, fmaxf(fabsf(__low2float(b)), fabsf(__high2float(b))));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[8];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) b = fmaxf(b, wmax[w]);
    atomicMax(amax_bits + h, __float_as_int(b));
  }
}

// amax_bits[h] (float bits) -> scale[h], in place.
__global__ void head_scale_kernel(int32_t *amax_bits, int BH) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < BH) reinterpret_cast<float *>(amax_bits)[h] = e4m3_scale(__int_as_float(amax_bits[h]));
}

}  // namespace svg
