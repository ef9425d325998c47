// k-means assign step on the tensor cores (Sparse VideoGen2, section 2(a)
// "Clustering").
//
// a_n = argmin_c (||mu_c||^2 - 2 x_n . mu_c), ties to the lowest c.
// x (bf16) is exact as an MMA operand; every fp32 centroid is split into a
// bf16 high part and a bf16 low part (mu = hi + lo + r, |r| <= 2^-17 |mu|
// per channel) and x . mu is accumulated as x . hi + x . lo in fp32 TMEM.
// The epilogue keeps the best two centroids; when they are closer than the
// tensor-core error allows to separate, the exact float32 distances decide.
//
// One CTA per (128-token tile, head), ~97 KB shared memory so two CTAs share
// an SM.  Warps 0-3: epilogue (thread t = token t of the tile = TMEM lane t);
// warp 4: TMA producer; warp 5: MMA issuer and TMEM owner.  Centroids stream
// in chunks of 128 (one smem stage); the two TMEM accumulators let the
// epilogue of chunk j overlap the MMAs of chunk j+1.
#pragma once
#include "common.cuh"

namespace svg {

template <int D>
struct KmCfg {
  static constexpr int BM = 128, NC = 128, DH = D / 64;
  static constexpr int X_BYTES = BM * D * 2, C_BYTES = NC * D * 2;
  static constexpr int HALF = 128 * 128;  // one 64-channel half of a 128-row tile
  static constexpr int OFF_X = 0, OFF_HI = X_BYTES, OFF_LO = OFF_HI + C_BYTES;
  static constexpr int OFF_BAR = OFF_LO + C_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
  static constexpr uint32_t TM_COLS = 256;
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, NC, false, false);
  static constexpr int THREADS = 192;
};

struct KmBarriers {
  uint64_t x_full, c_full, c_empty, acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

__device__ __forceinline__ bool km_wait(KmBarriers *b, uint64_t *bar, uint32_t parity, uint64_t ns,
                                        uint32_t site) {
  if (mbar_wait(bar, parity, ns)) return true;
  record_error(SVG_ERR_TIMEOUT, site);
  atomicExch(&b->abort_flag, 1);
  return false;
}

// Splits fp32 centroids into bf16 hi/lo parts and squared norms for chunks of
// NC rows; rows C..Cpad-1 get zero parts and +inf norm (never the argmin).
// Also clears the fp64 update sums [BH, C, D] for the first round.
__global__ void kmeans_split_kernel(const float *__restrict__ mu, int C, int Cpad, int D,
                                    __nv_bfloat16 *__restrict__ hi, __nv_bfloat16 *__restrict__ lo,
                                    float *__restrict__ norms, double *__restrict__ sums) {
  const int h = blockIdx.y;
  const int c = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (c >= Cpad) return;
  const size_t orow = (static_cast<size_t>(h) * Cpad + c) * D;
  float s = 0.f;
  for (int d = lane; d < D; d += 32) {
    float v = c < C ? mu[(static_cast<size_t>(h) * C + c) * D + d] : 0.f;
    const __nv_bfloat16 vh = __float2bfloat16_rn(v);
    const __nv_bfloat16 vl = __float2bfloat16_rn(v - __bfloat162float(vh));
    hi[orow + d] = vh;
    lo[orow + d] = vl;
    s = fmaf(v, v, s);
    if (c < C) sums[(static_cast<size_t>(h) * C + c) * D + d] = 0.0;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) norms[static_cast<size_t>(h) * Cpad + c] = c < C ? s : INFINITY;
}

template <int D>
__global__ void __launch_bounds__(KmCfg<D>::THREADS)
    kmeans_assign_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                            const __grid_constant__ CUtensorMap map_hi,
                            const __grid_constant__ CUtensorMap map_lo, int N, int C, int Cpad,
                            const float *__restrict__ norms, const float *__restrict__ mu,
                            int32_t *__restrict__ assign, uint64_t wait_ns) {
  using Cfg = KmCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sX = smem + Cfg::OFF_X;
  uint8_t *sHi = smem + Cfg::OFF_HI;
  uint8_t *sLo = smem + Cfg::OFF_LO;
  KmBarriers *B = reinterpret_cast<KmBarriers *>(smem + Cfg::OFF_BAR);
  const int warp = static_cast<int>(warp_id()), lane = static_cast<int>(lane_id());
  const int h = blockIdx.y, n0 = blockIdx.x * Cfg::BM;
  const int nchunks = Cpad / Cfg::NC;

  if (threadIdx.x == 0) {
    mbar_init(&B->x_full, 1);
    mbar_init(&B->c_full, 1);
    mbar_init(&B->c_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B->acc_full[s], 1);
      mbar_init(&B->acc_empty[s], 4);
    }
    mbar_init(&B->drain, 1);
    B->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&B->tmem_base, Cfg::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B->tmem_base;

  if (warp == 4) {
    if (lane == 0) {
      int j = 0;
      mbar_arrive_expect_tx(&B->x_full, Cfg::X_BYTES);
#pragma unroll
      for (int dh = 0; dh < Cfg::DH; ++dh)
        tma_load_2d(sX + dh * Cfg::HALF, &map_x, dh * 64, h * N + n0, &B->x_full);
      for (; j < nchunks; ++j) {
        if (j > 0 && !km_wait(B, &B->c_empty, (j - 1) & 1, wait_ns, SITE_KMEANS_MMA)) break;
        mbar_arrive_expect_tx(&B->c_full, 2 * Cfg::C_BYTES);
        const int crow = h * Cpad + j * Cfg::NC;
#pragma unroll
        for (int dh = 0; dh < Cfg::DH; ++dh) {
          tma_load_2d(sHi + dh * Cfg::HALF, &map_hi, dh * 64, crow, &B->c_full);
          tma_load_2d(sLo + dh * Cfg::HALF, &map_lo, dh * 64, crow, &B->c_full);
        }
      }
      // drain: the last issued chunk and x must have landed before exit
      mbar_wait(&B->x_full, 0, 1000000000ull);
      if (j > 0) mbar_wait(&B->c_full, (j - 1) & 1, 1000000000ull);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t xb = smem_u32(sX), hb = smem_u32(sHi), lb = smem_u32(sLo);
      if (km_wait(B, &B->x_full, 0, wait_ns, SITE_KMEANS_MMA)) {
        for (int j = 0; j < nchunks; ++j) {
          const int ab = j & 1;
          if (!km_wait(B, &B->c_full, j & 1, wait_ns, SITE_KMEANS_MMA)) break;
          if (j >= 2 && !km_wait(B, &B->acc_empty[ab], ((j >> 1) - 1) & 1, wait_ns, SITE_KMEANS_MMA))
            break;
          tc_fence_after();
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint32_t cb = part == 0 ? hb : lb;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t koff = (kk >> 2) * Cfg::HALF + (kk & 3) * 32;
              mma_bf16_ss(tmem + ab * Cfg::NC, smem_desc_sw128(xb + koff, 16, 1024),
                          smem_desc_sw128(cb + koff, 16, 1024), Cfg::IDESC,
                          (part == 0 && kk == 0) ? 0u : 1u);
            }
          }
          mma_commit(&B->c_empty);
          mma_commit(&B->acc_full[ab]);
        }
      }
      mma_commit(&B->drain);
      mbar_wait(&B->drain, 0, 1000000000ull);
    }
  } else {
    // epilogue: running best and runner-up over the chunks for token n0 + row
    const int row = threadIdx.x;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float *nh = norms + static_cast<size_t>(h) * Cpad;
    float best = INFINITY, second = INFINITY;
    int arg = 0, arg2 = -1;
    bool ok = true;
    for (int j = 0; j < nchunks; ++j) {
      const int ab = j & 1;
      const bool got = mbar_wait(&B->acc_full[ab], (j >> 1) & 1, wait_ns);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) {
          record_error(SVG_ERR_TIMEOUT, SITE_KMEANS_EPI);
          atomicExch(&B->abort_flag, 1);
        }
        ok = false;
        break;
      }
      tc_fence_after();
      float acc[128];
      tmem_ld128_sync(tmem + lane_off + ab * Cfg::NC, acc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B->acc_empty[ab]);
      const float *cn = nh + j * Cfg::NC;
#pragma unroll
      for (int c = 0; c < Cfg::NC; ++c) {
        const float score = fmaf(-2.f, acc[c], __ldg(cn + c));
        if (score < best) {
          second = best;
          arg2 = arg;
          best = score;
          arg = j * Cfg::NC + c;
        } else if (score < second) {
          second = score;
          arg2 = j * Cfg::NC + c;
        }
      }
    }
    if (ok && n0 + row < N) {
      // Near-tie: the tensor-core scores carry about 2^-15 ||x|| ||mu|| of
      // error (bf16 split residual plus fp32 accumulation).  When the runner-up
      // is within 2^-13 (||x||^2 + ||mu||^2) >= 2^-12 ||x|| ||mu||, decide with
      // the exact float32 distances sum_d (x_d - mu_d)^2 instead.
      float xr[D];
#pragma unroll
      for (int dh = 0; dh < Cfg::DH; ++dh)
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 u = *reinterpret_cast<const uint4 *>(
              sX + dh * Cfg::HALF + row * 128 + ((q ^ (row & 7)) << 4));
          const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(b2[e]);
            xr[dh * 64 + q * 8 + 2 * e] = f.x;
            xr[dh * 64 + q * 8 + 2 * e + 1] = f.y;
          }
        }
      float xx = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) xx = fmaf(xr[d], xr[d], xx);
      if (arg2 >= 0 && arg2 < C && second - best <= 0x1p-13f * (xx + __ldg(nh + arg))) {
        const float *m1 = mu + (static_cast<size_t>(h) * C + arg) * D;
        const float *m2 = mu + (static_cast<size_t>(h) * C + arg2) * D;
        float d1 = 0.f, d2 = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          const float a1 = xr[d] - __ldg(m1 + d), a2 = xr[d] - __ldg(m2 + d);
          d1 = fmaf(a1, a1, d1);
          d2 = fmaf(a2, a2, d2);
        }
        if (d2 < d1 || (d2 == d1 && arg2 < arg)) arg = arg2;
      }
      assign[static_cast<size_t>(h) * N + n0 + row] = arg;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TM_COLS);
  }
}

}  // namespace svg
