// k-means assign step on the tensor cores (Sparse VideoGen2, section 2(a)
// "Clustering").
//
// a_n = argmin_c (||mu_c||^2 - 2 x_n . mu_c), ties to the lowest c.
// x (bf16) is exact as an MMA operand; every fp32 centroid is split into a
// bf16 high part and a bf16 low part (mu = hi + lo + r, |r| <= 2^-17 |mu|
// per channel) and x . mu is accumulated as x . hi + x . lo in fp32 TMEM.
// The epilogue keeps the best two centroids; when they are closer than the
// tensor-core error allows to separate, the token goes on a near-tie list and
// kmeans_refine_kernel decides it with the exact float32 distances.  The
// epilogue also counts the members of every cluster (the refine step moves
// the tokens it reassigns), which the update step (kmeans.cuh) starts from.
//
// Persistent: one CTA per SM walks units (head, 128-token tile) in
// head-major order (the head's centroids stay hot in L2).  Warps 0-7:
// epilogue in two groups of four (thread t of a group = token t of the tile
// = TMEM lane t), taking alternate chunks; warp 8: TMA producer (x tiles,
// centroid chunks and their squared norms); warp 9: MMA issuer and TMEM
// owner.  x tiles (2-deep ring) and centroid chunks of 128 (hi and lo parts,
// 2-deep ring) stream through shared memory; four TMEM accumulators (two per
// epilogue group) let the MMAs run up to two chunks ahead of each group.
#pragma once
#include "common.cuh"

namespace svg {

template <int D>
struct KmCfg {
  static constexpr int BM = 128, NC = 128, DH = D / 64;
  static constexpr int XST = 2, CST = 2;  // x tile ring, centroid chunk ring
  static constexpr int X_BYTES = BM * D * 2, C_BYTES = NC * D * 2;
  static constexpr int HALF = 128 * 128;  // one 64-channel half of a 128-row tile
  static constexpr int OFF_X = 0;
  static constexpr int OFF_C = OFF_X + XST * X_BYTES;          // stage: hi part then lo part
  static constexpr int NST = 4, AST = 4;  // norms ring, TMEM accumulators
  static constexpr int OFF_NORM = OFF_C + CST * 2 * C_BYTES;   // NST x NC fp32 squared norms
  static constexpr int OFF_MERGE = OFF_NORM + NST * NC * 4;    // 2 x 128 x (best, arg, second, arg2)
  static constexpr int OFF_BAR = OFF_MERGE + 2 * 128 * 16;
  static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;
  static constexpr uint32_t TM_COLS = AST * NC;
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, NC, false, false);
  static constexpr int EPI_WARPS = 8;                          // two groups of four
  static constexpr int THREADS = (EPI_WARPS + 2) * 32;
  static constexpr int PRODUCER_WARP = EPI_WARPS, MMA_WARP = EPI_WARPS + 1;
};

struct KmBarriers {
  uint64_t x_full[2], x_empty[2], c_full[2], c_empty[2], acc_full[4], acc_empty[4];
  uint64_t n_full[4], n_empty[4], merge_full[2], merge_empty[2], drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

// One near-tie token: flat token index (h * N + n) and its two candidates.
struct KmTie {
  int32_t token, a, b, pad;
};


__device__ __forceinline__ bool km_wait(KmBarriers *b, uint64_t *bar, uint32_t parity, uint64_t ns,
                                        uint32_t site) {
  if (mbar_wait(bar, parity, ns)) return true;
  record_error(SVG_ERR_TIMEOUT, site);
  atomicExch(&b->abort_flag, 1);
  return false;
}

// Padding rows C..Cpad-1 of a chunk get zero parts and this squared norm: a
// finite score far above any real one, so they are never the argmin and their
// keys stay finite.
constexpr float kPadNorm = 0x1p100f;

// Splits fp32 centroids into bf16 hi/lo parts and squared norms for chunks of
// NC rows.  Also clears the near-tie counter and the per-cluster counters
// (sizes, bucket cursors, chunk arrivals) before the first assign step.
__global__ void kmeans_split_kernel(const float *__restrict__ mu, int C, int Cpad, int D,
                                    __nv_bfloat16 *__restrict__ hi, __nv_bfloat16 *__restrict__ lo,
                                    float *__restrict__ norms, int32_t *__restrict__ num_ties,
                                    int32_t *__restrict__ counters) {
  const int h = blockIdx.y;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *num_ties = 0;
  const int c = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (c >= Cpad) return;
  if (c < C && lane < 3)   // counters: three [BH, C] int32 arrays, back to back
    counters[(static_cast<size_t>(lane) * gridDim.y + h) * C + c] = 0;
  const size_t orow = (static_cast<size_t>(h) * Cpad + c) * D;
  float s = 0.f;
  for (int d = lane; d < D; d += 32) {
    float v = c < C ? mu[(static_cast<size_t>(h) * C + c) * D + d] : 0.f;
    const __nv_bfloat16 vh = __float2bfloat16_rn(v);
    const __nv_bfloat16 vl = __float2bfloat16_rn(v - __bfloat162float(vh));
    hi[orow + d] = vh;
    lo[orow + d] = vl;
    s = fmaf(v, v, s);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) norms[static_cast<size_t>(h) * Cpad + c] = c < C ? s : kPadNorm;
}

template <int D>
__global__ void __launch_bounds__(KmCfg<D>::THREADS, 1)
    kmeans_assign_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                            const __grid_constant__ CUtensorMap map_hi,
                            const __grid_constant__ CUtensorMap map_lo, int BH, int N, int C,
                            int Cpad, const float *__restrict__ norms,
                            const float *__restrict__ xnorm, int32_t *__restrict__ assign,
                            int32_t *__restrict__ counts, KmTie *__restrict__ ties,
                            int32_t *__restrict__ num_ties, uint64_t wait_ns) {
  using Cfg = KmCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  KmBarriers *B = reinterpret_cast<KmBarriers *>(smem + Cfg::OFF_BAR);
  float *sNorm = reinterpret_cast<float *>(smem + Cfg::OFF_NORM);
  float4 *sMerge = reinterpret_cast<float4 *>(smem + Cfg::OFF_MERGE);
  const int warp = static_cast<int>(warp_id()), lane = static_cast<int>(lane_id());
  const int tiles = (N + Cfg::BM - 1) / Cfg::BM;
  const int units = BH * tiles;              // unit u = (head u / tiles, tile u % tiles)
  const int nchunks = Cpad / Cfg::NC;
  const int grid = static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B->x_full[s], 1);
      mbar_init(&B->x_empty[s], 1);          // released by the MMA commit after a unit
      mbar_init(&B->c_full[s], 1);
      mbar_init(&B->c_empty[s], 1);
      mbar_init(&B->merge_full[s], 4);
      mbar_init(&B->merge_empty[s], 4);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&B->acc_full[s], 1);
      mbar_init(&B->acc_empty[s], 4);        // the four warps of the group that read it
      mbar_init(&B->n_full[s], 1);
      mbar_init(&B->n_empty[s], 4);
    }
    mbar_init(&B->drain, 1);
    B->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == Cfg::MMA_WARP) {
    tmem_alloc(&B->tmem_base, Cfg::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B->tmem_base;

  if (warp == Cfg::PRODUCER_WARP) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t nu = 0, gc = 0, gn = 0;   // x tiles, centroid chunks and norm rows issued
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += grid, ++nu) {
        const int h = u / tiles, n0 = (u % tiles) * Cfg::BM;
        const int xs = nu & 1;
        if (nu >= 2 && !km_wait(B, &B->x_empty[xs], ((nu >> 1) - 1) & 1, wait_ns, SITE_KMEANS_MMA)) break;
        mbar_arrive_expect_tx(&B->x_full[xs], Cfg::X_BYTES);
        uint8_t *xd = smem + Cfg::OFF_X + xs * Cfg::X_BYTES;
#pragma unroll
        for (int dh = 0; dh < Cfg::DH; ++dh)
          tma_load_2d(xd + dh * Cfg::HALF, &map_x, dh * 64, h * N + n0, &B->x_full[xs]);
        for (int j = 0; j < nchunks; ++j, ++gc) {
          const int cs = gc & 1, ns = gc & 3;
          if (gc >= 2 && !km_wait(B, &B->c_empty[cs], ((gc >> 1) - 1) & 1, wait_ns, SITE_KMEANS_MMA)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&B->c_full[cs], 2 * Cfg::C_BYTES);
          uint8_t *cd = smem + Cfg::OFF_C + cs * 2 * Cfg::C_BYTES;
          const int crow = h * Cpad + j * Cfg::NC;
#pragma unroll
          for (int dh = 0; dh < Cfg::DH; ++dh) {
            tma_load_2d(cd + dh * Cfg::HALF, &map_hi, dh * 64, crow, &B->c_full[cs]);
            tma_load_2d(cd + Cfg::C_BYTES + dh * Cfg::HALF, &map_lo, dh * 64, crow, &B->c_full[cs]);
          }
          if (gc >= 4 && !km_wait(B, &B->n_empty[ns], ((gc >> 2) - 1) & 1, wait_ns, SITE_KMEANS_MMA)) {
            ++gc;          // this chunk's centroid copies are in flight: the drain waits for them
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&B->n_full[ns], Cfg::NC * 4);
          bulk_load(sNorm + ns * Cfg::NC, norms + static_cast<size_t>(crow), Cfg::NC * 4, &B->n_full[ns]);
          ++gn;
        }
      }
      // drain: wait for the last issued copies of each ring slot
      if (*reinterpret_cast<volatile int32_t *>(&B->abort_flag)) {
        for (uint32_t k = nu >= 2 ? nu - 2 : 0; k < nu; ++k)
          mbar_wait(&B->x_full[k & 1], (k >> 1) & 1, 1000000000ull);
        for (uint32_t k = gc >= 2 ? gc - 2 : 0; k < gc; ++k)
          mbar_wait(&B->c_full[k & 1], (k >> 1) & 1, 1000000000ull);
        for (uint32_t k = gn >= 4 ? gn - 4 : 0; k < gn; ++k)
          mbar_wait(&B->n_full[k & 3], (k >> 2) & 1, 1000000000ull);
      }
    }
  } else if (warp == Cfg::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t nu = 0, gc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += grid, ++nu) {
        const int xs = nu & 1;
        if (!km_wait(B, &B->x_full[xs], (nu >> 1) & 1, wait_ns, SITE_KMEANS_MMA)) break;
        const uint32_t xb = smem_u32(smem + Cfg::OFF_X + xs * Cfg::X_BYTES);
        for (int j = 0; j < nchunks; ++j, ++gc) {
          const int cs = gc & 1, ab = gc & 3;
          if (!km_wait(B, &B->c_full[cs], (gc >> 1) & 1, wait_ns, SITE_KMEANS_MMA) ||
              (gc >= 4 && !km_wait(B, &B->acc_empty[ab], ((gc >> 2) - 1) & 1, wait_ns, SITE_KMEANS_MMA))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t cb = smem_u32(smem + Cfg::OFF_C + cs * 2 * Cfg::C_BYTES);
#pragma unroll
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t koff = (kk >> 2) * Cfg::HALF + (kk & 3) * 32;
              mma_bf16_ss(tmem + ab * Cfg::NC, smem_desc_sw128(xb + koff, 16, 1024),
                          smem_desc_sw128(cb + part * Cfg::C_BYTES + koff, 16, 1024), Cfg::IDESC,
                          (part == 0 && kk == 0) ? 0u : 1u);
            }
          }
          mma_commit(&B->c_empty[cs]);
          mma_commit(&B->acc_full[ab]);
        }
        if (ok) mma_commit(&B->x_empty[xs]);   // the unit's MMAs are the last readers of x
      }
      mma_commit(&B->drain);
      mbar_wait(&B->drain, 0, 1000000000ull);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Two groups of four warps; group g takes the chunks with (global chunk
    // index & 1) == g, from accumulator buffers g and g + 2 in turn.  Thread
    // `row` of a group = token n0 + row = TMEM lane row.
    //
    // Best two centroids per row with three min/max operations per score.
    // Every score s becomes a key: s with its low byte replaced by the
    // column's position in its 64-column half-chunk (a change of at most
    // 2^-15 |s|), so the keys of one half-chunk are distinct and each names
    // its column.  The half-chunk's two smallest keys follow
    //   m2 = min(m2, max(m1, k)),  m1 = min(m1, k)
    // in two interleaved chains, and are then merged into the running best
    // and runner-up with the half-chunk's first column (an equal key keeps the
    // earlier column).  When a unit has several chunks, group 1 hands its pair
    // to group 0 through shared memory and group 0 merges.
    // Near-tie rule: a key is within 2^-15 |s| of its score, and the
    // tensor-core score is within about 2^-16 (||x||^2 + ||mu||^2) of the
    // exact one (bf16 split residual and fp32 accumulation).  A runner-up
    // within 2^-14 (|key_1| + |key_2| + ||x||^2 + the larger ||mu||^2) of the
    // best (twice the key term, four times the tensor-core term) goes to the
    // exact float32 re-check.
    constexpr float kBig = 3.0e38f;
    const int grp = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // bytes 4r..4r+3 (column positions inside a half-chunk), one register per
    // four columns; opaque to the compiler so they stay in registers
    uint32_t colb[16];
#pragma unroll
    for (int r = 0; r < 16; ++r)
      asm volatile("mov.b32 %0, %1;" : "=r"(colb[r]) : "r"(0x03020100u + 0x04040404u * r));
    uint32_t nu = 0, gc = 0;
    for (int u = blockIdx.x; u < units; u += grid, ++nu) {
      const int h = u / tiles, n0 = (u % tiles) * Cfg::BM;
      const bool valid = n0 + row < N;
      float best = kBig, second = kBig;
      int arg = 0x7fffffff, arg2 = -1;
      bool ok = true, mine_any = false;
      for (int j = 0; j < nchunks; ++j, ++gc) {
        if (static_cast<int>(gc & 1) != grp) continue;
        const int ab = gc & 3;     // accumulator buffer and norms slot
        mine_any = true;
        const bool got = mbar_wait(&B->acc_full[ab], (gc >> 2) & 1, wait_ns) &&
                         mbar_wait(&B->n_full[ab], (gc >> 2) & 1, wait_ns);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) {
            record_error(SVG_ERR_TIMEOUT, SITE_KMEANS_EPI);
            atomicExch(&B->abort_flag, 1);
          }
          ok = false;
          break;
        }
        tc_fence_after();
        const float4 *nv4 = reinterpret_cast<const float4 *>(sNorm + ab * Cfg::NC);
        const uint32_t acc_addr = tmem + lane_off + ab * Cfg::NC;
        // 32-column pieces: the next piece's TMEM load is in flight while the
        // current one is reduced
        uint32_t buf[2][32];
        tmem_ld32_start(acc_addr, buf[0]);
        tmem_wait32(buf[0]);
        float p1 = kBig, p2 = kBig, q1 = kBig, q2 = kBig;
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          if (pc < 3) {
            tmem_ld32_start(acc_addr + (pc + 1) * 32, buf[(pc + 1) & 1]);
          } else {               // every piece is in registers: the MMAs may reuse the buffer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&B->acc_empty[ab]);
          }
          const uint32_t *acc = buf[pc & 1];
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 nv = nv4[pc * 8 + c4];
            const float nn[4] = {nv.x, nv.y, nv.z, nv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float sc = fmaf(-2.f, __uint_as_float(acc[4 * c4 + e]), nn[e]);
              const float k = __int_as_float(
                  __byte_perm(__float_as_int(sc), colb[(pc & 1) * 8 + c4], 0x3214 + e));
              if (e & 1) {
                q2 = fminf(q2, fmaxf(q1, k));
                q1 = fminf(q1, k);
              } else {
                p2 = fminf(p2, fmaxf(p1, k));
                p1 = fminf(p1, k);
              }
            }
          }
          if (pc & 1) {          // end of a 64-column half: merge its pair
            const float m1 = fminf(p1, q1);
            const float m2 = fminf(fmaxf(p1, q1), fminf(p2, q2));
            const int cbase = j * Cfg::NC + (pc >> 1) * 64;
            const int mc1 = cbase + (__float_as_int(m1) & 0xFF);
            const int mc2 = cbase + (__float_as_int(m2) & 0xFF);
            const bool n1 = m1 < best, n2 = m1 < second, s1 = m2 < best;
            const float ns = n1 ? (s1 ? m2 : best) : (n2 ? m1 : second);
            const int nsa = n1 ? (s1 ? mc2 : arg) : (n2 ? mc1 : arg2);
            best = n1 ? m1 : best;
            arg = n1 ? mc1 : arg;
            second = ns;
            arg2 = nsa;
            p1 = p2 = q1 = q2 = kBig;
          }
          if (pc < 3) tmem_wait32(buf[(pc + 1) & 1]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&B->n_empty[ab]);
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      // combine the two groups' pairs when both saw chunks of this unit
      bool owner = mine_any;
      if (nchunks >= 2) {
        const int ms = nu & 1;
        float4 *slot = sMerge + ms * 128 + row;
        if (grp == 1) {
          if (nu >= 2 && !__all_sync(0xffffffffu, mbar_wait(&B->merge_empty[ms], ((nu >> 1) - 1) & 1, wait_ns))) {
            if (lane == 0) {
              record_error(SVG_ERR_TIMEOUT, SITE_KMEANS_EPI);
              atomicExch(&B->abort_flag, 1);
            }
            break;
          }
          *slot = make_float4(best, __int_as_float(arg), second, __int_as_float(arg2));
          __syncwarp();
          if (lane == 0) mbar_arrive(&B->merge_full[ms]);
          owner = false;
        } else {
          if (!__all_sync(0xffffffffu, mbar_wait(&B->merge_full[ms], (nu >> 1) & 1, wait_ns))) {
            if (lane == 0) {
              record_error(SVG_ERR_TIMEOUT, SITE_KMEANS_EPI);
              atomicExch(&B->abort_flag, 1);
            }
            break;
          }
          const float4 o = *slot;
          __syncwarp();
          if (lane == 0) mbar_arrive(&B->merge_empty[ms]);
          const float ob = o.x, os = o.z;
          const int oa = __float_as_int(o.y), oa2 = __float_as_int(o.w);
          // top two (score, index) of the union of the two pairs
          if (ob < best || (ob == best && oa < arg)) {
            if (best < os || (best == os && arg < oa2)) {
              second = best;
              arg2 = arg;
            } else {
              second = os;
              arg2 = oa2;
            }
            best = ob;
            arg = oa;
          } else if (ob < second || (ob == second && oa < arg2)) {
            second = ob;
            arg2 = oa;
          }
          owner = true;
        }
      }
      if (!owner) continue;
      const float *nh = norms + static_cast<size_t>(h) * Cpad;
      const bool live = valid && arg >= 0 && arg < C;
      if (valid && !live) record_error(SVG_ERR_DEVICE_CHECK, SITE_KMEANS_RANGE);
      bool tie = false;
      if (live && arg2 >= 0 && arg2 < C) {
        const float xx = __ldg(xnorm + static_cast<size_t>(h) * N + n0 + row);
        const float mm = fmaxf(__ldg(nh + arg), __ldg(nh + arg2));
        tie = second - best <= 0x1p-14f * (fabsf(best) + fabsf(second) + xx + mm);
      }
      const unsigned tmask = __ballot_sync(0xffffffffu, tie);
      if (tmask) {   // warp-aggregated append to the near-tie list
        int base = 0;
        if (lane == 0) base = atomicAdd(num_ties, __popc(tmask));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (tie) {
          const int slot = base + __popc(tmask & ((1u << lane) - 1u));
          ties[slot] = KmTie{h * N + n0 + row, arg, arg2, 0};
        }
      }
      if (valid) assign[static_cast<size_t>(h) * N + n0 + row] = arg;
      // cluster sizes of this round, one atomic per distinct cluster of a warp
      const unsigned lmask = __ballot_sync(0xffffffffu, live);
      if (live) {
        const unsigned peers = __match_any_sync(lmask, arg);
        if (lane == __ffs(peers) - 1) atomicAdd(counts + static_cast<size_t>(h) * C + arg, __popc(peers));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TM_COLS);
  }
}

// ||x_n||^2 in fp32 for every token (x does not change across rounds); each
// thread squares one 16-byte vector, the D/8 threads of a row add theirs.
template <int D>
__global__ void __launch_bounds__(256) kmeans_xnorm_kernel(const __nv_bfloat16 *__restrict__ x,
                                                           size_t tokens, float *__restrict__ xnorm) {
  constexpr int VPR = D / 8;
  const size_t v = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t t = v / VPR;
  float s = 0.f;
  if (t < tokens) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(x) + v);
    const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(b2[e]);
      s = fmaf(f.x, f.x, s);
      s = fmaf(f.y, f.y, s);
    }
  }
#pragma unroll
  for (int o = VPR / 2; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (t < tokens && (threadIdx.x % VPR) == 0) xnorm[t] = s;
}

// Decides every listed near tie with the exact float32 distances
// sum_d (x_d - mu_d)^2 (ties to the lower index); one warp per token.  The
// assign step already stored and counted the first candidate.
template <int D>
__global__ void __launch_bounds__(256) kmeans_refine_kernel(const __nv_bfloat16 *__restrict__ x,
                                                            int N, int C, const float *__restrict__ mu,
                                                            const KmTie *__restrict__ ties,
                                                            const int32_t *__restrict__ num_ties,
                                                            int32_t *__restrict__ assign,
                                                            int32_t *__restrict__ counts) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const int nt = *num_ties;
  for (int e = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); e < nt;
       e += gridDim.x * (blockDim.x / 32)) {
    const KmTie t = ties[e];
    const int h = t.token / N;
    const __nv_bfloat16 *xr = x + static_cast<size_t>(t.token) * D + lane * PER;
    const float *m1 = mu + (static_cast<size_t>(h) * C + t.a) * D + lane * PER;
    const float *m2 = mu + (static_cast<size_t>(h) * C + t.b) * D + lane * PER;
    float d1 = 0.f, d2 = 0.f;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const float xv = __bfloat162float(xr[k]);
      const float a1 = xv - m1[k], a2 = xv - m2[k];
      d1 = fmaf(a1, a1, d1);
      d2 = fmaf(a2, a2, d2);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      d1 += __shfl_xor_sync(0xffffffffu, d1, o);
      d2 += __shfl_xor_sync(0xffffffffu, d2, o);
    }
    if (lane == 0 && (d2 < d1 || (d2 == d1 && t.b < t.a))) {   // the runner-up wins: move the token
      assign[t.token] = t.b;
      atomicSub(counts + static_cast<size_t>(h) * C + t.a, 1);
      atomicAdd(counts + static_cast<size_t>(h) * C + t.b, 1);
    }
  }
}

}  // namespace svg
