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
// Data movement is the limit of this step: a 128-token tile of x is 32 KB
// but one 128-centroid chunk (hi and lo parts) is 64 KB, and streaming every
// chunk from L2 for every tile saturates L2-to-shared-memory bandwidth long
// before the tensor cores.  So every CTA takes a contiguous range of
// (head, 128-token tile) units and reuses centroids across tiles:
//   * C <= 128 (one chunk, SINGLE): the chunk stays in shared memory while
//     the CTA's units belong to the same head; only x streams (4-deep ring);
//   * C > 128: consecutive tiles of one head are taken in pairs, and every
//     chunk (hi and lo parts through a 4-deep ring) feeds both tiles' MMA
//     chains before it is released, halving the centroid traffic per tile;
//     a third x slot lets the next pair's first tile load while the current
//     pair's last chunk is multiplied.
// Warps 0-7: epilogue in two groups of four; group g owns tile g of every
// pair (thread t of a group = token t of the tile = TMEM lane t) and keeps
// the running best pair over all chunks of its tile, so the groups never
// merge.  Warp 8: TMA producer.  Warps 9 and 10: one MMA issuer per tile of
// a pair (warp 9 owns TMEM); each (tile, chunk) is one chain of 2 x D/16 MMAs
// (hi then lo) into one of the group's two TMEM accumulators.  The issuing
// thread runs in step with the tensor pipe (a chain of 16 MMAs takes about as
// long to issue as to execute), so with one issuer every barrier wait
// between chains left the pipe idle; with two, one tile's chain executes
// while the other issuer waits.
#pragma once
#include "common.cuh"

namespace svg {

constexpr int kKmChunk = 128;   // centroids per chunk (MMA N)

template <int D, bool SINGLE>
struct KmCfg {
  static constexpr int BM = 128, NC = kKmChunk, DH = D / 64;
  static constexpr int XST = SINGLE ? 5 : 3;   // x tile ring (pairs: the next pair's first tile loads early)
  static constexpr int CST = SINGLE ? 2 : 4;   // centroid part ring (a part = hi or lo of a chunk)
  static constexpr int X_BYTES = BM * D * 2, C_BYTES = NC * D * 2;
  static constexpr int HALF = 128 * 128;       // one 64-channel half of a 128-row tile
  static constexpr int OFF_X = 0;
  static constexpr int OFF_C = OFF_X + XST * X_BYTES;
  static constexpr int OFF_BAR = OFF_C + CST * C_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;
  static constexpr int AST = 4;                // TMEM accumulators, two per epilogue group
  static constexpr uint32_t TM_COLS = AST * NC;
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, NC, false, false);
  static constexpr int EPI_WARPS = 8;          // two groups of four
  static constexpr int THREADS = (EPI_WARPS + 3) * 32;
  static constexpr int PRODUCER_WARP = EPI_WARPS, MMA_WARP = EPI_WARPS + 1, MMA_B_WARP = EPI_WARPS + 2;
  static_assert(XST <= 6 && CST <= 4, "barrier arrays");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

struct KmBarriers {   // x rings have at most 6 slots
  uint64_t x_full[6], x_empty[6], c_full[4], c_empty[4], acc_full[4], acc_empty[4], drain[2];
  uint32_t tmem_base;
  int32_t abort_flag;
};

// Tiles (1 or 2) of the pair of units starting at u: two when u + 1 is in the
// CTA's range and in the same head.
__device__ __forceinline__ int km_pair_tiles(int u, int u_end, int tiles) {
  return (u + 1 < u_end && (u + 1) / tiles == u / tiles) ? 2 : 1;
}

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

template <int D, bool SINGLE>
__global__ void __launch_bounds__(KmCfg<D, SINGLE>::THREADS, 1)
    kmeans_assign_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                            const __grid_constant__ CUtensorMap map_hi,
                            const __grid_constant__ CUtensorMap map_lo, int BH, int N, int C,
                            int Cpad, const float *__restrict__ norms,
                            float *__restrict__ xnorm, int32_t *__restrict__ assign,
                            int32_t *__restrict__ counts, KmTie *__restrict__ ties,
                            int32_t *__restrict__ num_ties, int make_xnorm, uint64_t wait_ns) {
  using Cfg = KmCfg<D, SINGLE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  KmBarriers *B = reinterpret_cast<KmBarriers *>(smem + Cfg::OFF_BAR);
  const int warp = static_cast<int>(warp_id()), lane = static_cast<int>(lane_id());
  const int tiles = (N + Cfg::BM - 1) / Cfg::BM;
  const int nchunks = Cpad / Cfg::NC;
  // this CTA's contiguous range of units u = (head u / tiles, tile u % tiles)
  const long long units = static_cast<long long>(BH) * tiles;
  const int u_begin = static_cast<int>(units * blockIdx.x / gridDim.x);
  const int u_end = static_cast<int>(units * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::XST; ++s) {
      mbar_init(&B->x_full[s], 1);
      mbar_init(&B->x_empty[s], 4);          // released by the four epilogue warps of the tile's group
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&B->c_full[s], 1);
      mbar_init(&B->c_empty[s], 2);          // both tiles' readers (see the MMA issuers)
      mbar_init(&B->acc_full[s], 1);
      mbar_init(&B->acc_empty[s], 4);        // the four warps of the group that read it
    }
    mbar_init(&B->drain[0], 1);
    mbar_init(&B->drain[1], 1);
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
  auto x_slot = [&](uint32_t n) { return smem + Cfg::OFF_X + (n % Cfg::XST) * Cfg::X_BYTES; };
  auto c_slot = [&](uint32_t n) { return smem + Cfg::OFF_C + (n % Cfg::CST) * Cfg::C_BYTES; };

  if (warp == Cfg::PRODUCER_WARP) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t nx = 0, nc = 0;   // x tiles and centroid parts issued
      bool ok = true;
      int cur_h = -1;
      auto load_x = [&](int u) {
        const uint32_t s = nx % Cfg::XST;
        if (nx >= static_cast<uint32_t>(Cfg::XST) &&
            !km_wait(B, &B->x_empty[s], ((nx / Cfg::XST) - 1) & 1, wait_ns, SITE_KMEANS_MMA))
          return false;
        mbar_arrive_expect_tx(&B->x_full[s], Cfg::X_BYTES);
#pragma unroll
        for (int dh = 0; dh < Cfg::DH; ++dh)
          tma_load_2d(x_slot(nx) + dh * Cfg::HALF, &map_x, dh * 64, (u / tiles) * N + (u % tiles) * Cfg::BM,
                      &B->x_full[s]);
        ++nx;
        return true;
      };
      // one centroid part (hi or lo) of chunk j of head h
      auto load_part = [&](int h, int j, int part) {
        const uint32_t s = nc % Cfg::CST;
        if (nc >= static_cast<uint32_t>(Cfg::CST) &&
            !km_wait(B, &B->c_empty[s], ((nc / Cfg::CST) - 1) & 1, wait_ns, SITE_KMEANS_MMA))
          return false;
        mbar_arrive_expect_tx(&B->c_full[s], Cfg::C_BYTES);
#pragma unroll
        for (int dh = 0; dh < Cfg::DH; ++dh)
          tma_load_2d(c_slot(nc) + dh * Cfg::HALF, part ? &map_lo : &map_hi, dh * 64, h * Cpad + j * Cfg::NC,
                      &B->c_full[s]);
        ++nc;
        return true;
      };
      for (int u = u_begin; u < u_end && ok; ) {
        const int nt = km_pair_tiles(u, u_end, tiles);
        const int h = u / tiles;
        if (SINGLE) {
          if (h != cur_h) {          // new head: its chunk replaces the resident one
            ok = load_part(h, 0, 0) && load_part(h, 0, 1);
            cur_h = h;
          }
          for (int t = 0; t < nt && ok; ++t) ok = load_x(u + t);
        } else {
          for (int j = 0; j < nchunks && ok; ++j) {
            ok = load_part(h, j, 0) && load_part(h, j, 1);
            if (j == 0)
              for (int t = 0; t < nt && ok; ++t) ok = load_x(u + t);
          }
        }
        u += nt;
      }
      // drain: wait for the last issued copies of each ring slot
      if (*reinterpret_cast<volatile int32_t *>(&B->abort_flag)) {
        for (uint32_t k = nx >= static_cast<uint32_t>(Cfg::XST) ? nx - Cfg::XST : 0; k < nx; ++k)
          mbar_wait(&B->x_full[k % Cfg::XST], (k / Cfg::XST) & 1, 1000000000ull);
        for (uint32_t k = nc >= static_cast<uint32_t>(Cfg::CST) ? nc - Cfg::CST : 0; k < nc; ++k)
          mbar_wait(&B->c_full[k % Cfg::CST], (k / Cfg::CST) & 1, 1000000000ull);
      }
    }
  } else if (warp == Cfg::MMA_WARP || warp == Cfg::MMA_B_WARP) {
    // ------------------------------------------------------------ MMA issuers
    // Issuer x takes tile x of every pair.  A commit covers only its own
    // thread's MMAs, so the centroid parts of a chunk are released by both
    // tiles' epilogue groups (c_empty counts two arrivals), and in the
    // one-chunk case both issuers commit the resident chunk's release when
    // the head changes.
    const int x = warp == Cfg::MMA_WARP ? 0 : 1;
    if (lane == 0) {
      uint32_t nx = 0, nc = 0, kacc = 0;
      bool ok = true;
      int cur_h = -1;
      // descriptors of x slot 0 and centroid slot 0, built once; a slot adds its offset
      const SmemDesc xd0 = make_desc_sw128(smem_u32(smem + Cfg::OFF_X), 16, 1024);
      const SmemDesc cd0 = make_desc_sw128(smem_u32(smem + Cfg::OFF_C), 16, 1024);
      for (int u = u_begin; u < u_end && ok; ) {
        const int nt = km_pair_tiles(u, u_end, tiles);
        const int h = u / tiles;
        if (SINGLE && h != cur_h) {   // the resident chunk of the previous head is no longer read
          if (nc > 0) {
            mma_commit(&B->c_empty[0]);
            mma_commit(&B->c_empty[1]);
          }
          if (!km_wait(B, &B->c_full[nc % Cfg::CST], (nc / Cfg::CST) & 1, wait_ns, SITE_KMEANS_MMA) ||
              !km_wait(B, &B->c_full[(nc + 1) % Cfg::CST], ((nc + 1) / Cfg::CST) & 1, wait_ns, SITE_KMEANS_MMA)) {
            ok = false;
            break;
          }
          nc += 2;
          cur_h = h;
        }
        if (x < nt) {
          const uint32_t xn = nx + x;
          for (int j = 0; j < nchunks && ok; ++j) {
            uint32_t c_hi = nc - 2, c_lo = nc - 1;   // SINGLE: the resident parts
            if (!SINGLE) {
              c_hi = nc + 2 * j;
              c_lo = c_hi + 1;
              if (!km_wait(B, &B->c_full[c_hi % Cfg::CST], (c_hi / Cfg::CST) & 1, wait_ns, SITE_KMEANS_MMA) ||
                  !km_wait(B, &B->c_full[c_lo % Cfg::CST], (c_lo / Cfg::CST) & 1, wait_ns, SITE_KMEANS_MMA)) {
                ok = false;
                break;
              }
            }
            const int ab = 2 * x + static_cast<int>(kacc & 1);
            if ((j == 0 && !km_wait(B, &B->x_full[xn % Cfg::XST], (xn / Cfg::XST) & 1, wait_ns,
                                    SITE_KMEANS_MMA)) ||
                (kacc >= 2 && !km_wait(B, &B->acc_empty[ab], ((kacc >> 1) - 1) & 1, wait_ns, SITE_KMEANS_MMA))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const SmemDesc xd{xd0.lo + (((xn % Cfg::XST) * Cfg::X_BYTES) >> 4), xd0.hi};
            const SmemDesc hd{cd0.lo + (((c_hi % Cfg::CST) * Cfg::C_BYTES) >> 4), cd0.hi};
            const SmemDesc ld{cd0.lo + (((c_lo % Cfg::CST) * Cfg::C_BYTES) >> 4), cd0.hi};
            mma_chain<D / 16, Cfg::HALF, 32, Cfg::HALF, 32>(tmem + ab * Cfg::NC, xd, hd, Cfg::IDESC, 0u);
            mma_chain<D / 16, Cfg::HALF, 32, Cfg::HALF, 32>(tmem + ab * Cfg::NC, xd, ld, Cfg::IDESC, 1u);
            mma_commit(&B->acc_full[ab]);   // the only commit of a chain (slots are released by the epilogue)
            ++kacc;
          }
        }
        if (!SINGLE) nc += 2 * nchunks;
        nx += nt;
        u += nt;
      }
      mma_commit(&B->drain[x]);
      mbar_wait(&B->drain[x], 0, 1000000000ull);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Group g owns tile g of every pair; thread `row` = token n0 + row = TMEM
    // lane row.  Accumulators 2g and 2g + 1 alternate.
    //
    // Best two centroids per row with five min/max operations per two scores.
    // Every score s becomes a key: s with its low byte replaced by the
    // column's position in its 64-column half-chunk (a change of at most
    // 2^-15 |s|), so the keys of one half-chunk are distinct and each names
    // its column.  The half-chunk's two smallest keys are kept in four
    // independent chains (the chains are latency-bound, so more of them keep
    // the ALU busy); a chain takes its keys two at a time:
    //   lo = min(a, b), hi = max(a, b),
    //   m2 = min(m2, hi, max(m1, lo)),  m1 = min(m1, lo).
    // The chains are then merged pairwise and into the running best and
    // runner-up with the half-chunk's first column (an equal key keeps the
    // earlier column, chunks are taken in ascending order).
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
    uint32_t k = 0;   // accumulators this group has read
    // Slot releases: an accumulator's commit tracks every earlier MMA of its
    // issuer (one issuer per tile), so once a group sees the accumulator of
    // its tile's last chunk, that tile's x slot is no longer read, and once
    // it sees chunk j, its tile no longer reads chunk j's parts (c_empty
    // counts both tiles).  The epilogue arrives on those barriers itself,
    // which leaves one commit per MMA chain.
    uint32_t nx_ep = 0, nc_ep = 0;   // x tiles and centroid parts of earlier pairs (the MMA issuer's counts)
    bool ok = true;
    for (int u0 = u_begin; u0 < u_end && ok; ) {
      const int nt = km_pair_tiles(u0, u_end, tiles);
      const int u = u0 + grp;
      u0 += nt;
      const uint32_t xn_tile = nx_ep + grp, nc_pair = nc_ep;
      nx_ep += nt;
      if (!SINGLE) nc_ep += 2 * nchunks;
      if (grp >= nt) continue;
      const int h = u / tiles, n0 = (u % tiles) * Cfg::BM;
      const bool valid = n0 + row < N;
      const float *nh = norms + static_cast<size_t>(h) * Cpad;
      // ||x||^2 of later rounds is read now: the load completes while the chunks are reduced
      const float xx_ld = !make_xnorm && valid ? __ldg(xnorm + static_cast<size_t>(h) * N + n0 + row) : 0.f;
      float best = kBig, second = kBig;
      int arg = 0x7fffffff, arg2 = -1;
      float xx = 0.f;   // ||x||^2 of this row (first round: from the x tile in shared memory)
      for (int j = 0; j < nchunks; ++j, ++k) {
        const int ab = 2 * grp + static_cast<int>(k & 1);
        if (!__all_sync(0xffffffffu, mbar_wait(&B->acc_full[ab], (k >> 1) & 1, wait_ns))) {
          if (lane == 0) {
            record_error(SVG_ERR_TIMEOUT, SITE_KMEANS_EPI);
            atomicExch(&B->abort_flag, 1);
          }
          ok = false;
          break;
        }
        tc_fence_after();
        if (threadIdx.x == static_cast<unsigned>(grp * 128)) {   // one thread of the group
          if (!SINGLE) {   // this tile no longer reads chunk j (the lone tile of a pair counts twice)
            for (int r = 0; r < (nt == 1 ? 2 : 1); ++r) {
              mbar_arrive(&B->c_empty[(nc_pair + 2 * j) % Cfg::CST]);
              mbar_arrive(&B->c_empty[(nc_pair + 2 * j + 1) % Cfg::CST]);
            }
          }
        }
        if (make_xnorm && j == 0) {
          // The x tile stays in its slot until this group releases it after
          // the tile's last chunk; its own barrier (no later phase can have
          // started) orders the copy before these reads.
          if (!__all_sync(0xffffffffu, mbar_wait(&B->x_full[xn_tile % Cfg::XST], (xn_tile / Cfg::XST) & 1,
                                                 wait_ns))) {
            if (lane == 0) {
              record_error(SVG_ERR_TIMEOUT, SITE_KMEANS_EPI);
              atomicExch(&B->abort_flag, 1);
            }
            ok = false;
            break;
          }
          const uint8_t *xr = smem + Cfg::OFF_X + (xn_tile % Cfg::XST) * Cfg::X_BYTES + row * 128;
#pragma unroll
          for (int dh = 0; dh < Cfg::DH; ++dh) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {   // 16-byte chunk c of the row sits at chunk c ^ (row % 8)
              const uint4 v = *reinterpret_cast<const uint4 *>(xr + dh * Cfg::HALF + ((c ^ (row & 7)) << 4));
              const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(b2[e]);
                xx = fmaf(f.x, f.x, xx);
                xx = fmaf(f.y, f.y, xx);
              }
            }
          }
          if (valid) xnorm[static_cast<size_t>(h) * N + n0 + row] = xx;
        }
        if (j == nchunks - 1) {   // every warp of the group is done with the x tile (x_empty counts four)
          __syncwarp();
          if (lane == 0) mbar_arrive(&B->x_empty[xn_tile % Cfg::XST]);
        }
        const float4 *nv4 = reinterpret_cast<const float4 *>(nh + j * Cfg::NC);
        const uint32_t acc_addr = tmem + lane_off + ab * Cfg::NC;
        // 32-column pieces: the next piece's TMEM load is in flight while the
        // current one is reduced
        uint32_t buf[2][32];
        tmem_ld32_start(acc_addr, buf[0]);
        tmem_wait32(buf[0]);
        float a1[4] = {kBig, kBig, kBig, kBig}, a2[4] = {kBig, kBig, kBig, kBig};   // four chains
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
            const float4 nv = __ldg(nv4 + pc * 8 + c4);
            const float nn[4] = {nv.x, nv.y, nv.z, nv.w};
            float kk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float sc = fmaf(-2.f, __uint_as_float(acc[4 * c4 + e]), nn[e]);
              kk[e] = __int_as_float(__byte_perm(__float_as_int(sc), colb[(pc & 1) * 8 + c4], 0x3214 + e));
            }
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {   // chain (c4 & 1) * 2 + pr takes keys 2 pr, 2 pr + 1
              const int ch = (c4 & 1) * 2 + pr;
              const float lo = fminf(kk[2 * pr], kk[2 * pr + 1]), hi = fmaxf(kk[2 * pr], kk[2 * pr + 1]);
              a2[ch] = min3f(a2[ch], hi, fmaxf(a1[ch], lo));
              a1[ch] = fminf(a1[ch], lo);
            }
          }
          if (pc & 1) {          // end of a 64-column half: merge the chains' pairs
            const float p1 = fminf(a1[0], a1[1]), p2 = fminf(fmaxf(a1[0], a1[1]), fminf(a2[0], a2[1]));
            const float q1 = fminf(a1[2], a1[3]), q2 = fminf(fmaxf(a1[2], a1[3]), fminf(a2[2], a2[3]));
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
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) a1[ch] = a2[ch] = kBig;
          }
          if (pc < 3) tmem_wait32(buf[(pc + 1) & 1]);
        }
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      const bool live = valid && arg >= 0 && arg < C;
      if (valid && !live) record_error(SVG_ERR_DEVICE_CHECK, SITE_KMEANS_RANGE);
      bool tie = false;
      if (live && arg2 >= 0 && arg2 < C) {
        if (!make_xnorm) xx = xx_ld;
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
