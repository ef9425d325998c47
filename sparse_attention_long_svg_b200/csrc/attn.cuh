// Varlen block-sparse attention over the selected (q-cluster, k-cluster)
// blocks (Sparse VideoGen2, section 2(c) "Customized attention kernel": the
// query rows of a cluster are contiguous after the permutation and are
// computed densely; the selected key clusters are scattered ranges of the
// permuted K/V and are gathered sparsely, without padding them to fixed
// block sizes).
//
// Work item: up to 256 consecutive permuted query rows of one q-cluster, as
// two 128-row tiles A and B that share every K/V tile (one K/V fetch feeds
// two tiles of MMAs).  The item's key list is the concatenation of its
// selected k-clusters' row ranges (touching ranges merged into runs), cut
// into 8-row slots; 8 slots form a 64-key tile.  A run of n rows costs
// ceil(n/8) slots and at most 7 masked rows, fetched with as few TMA boxes as
// possible (8, 16, 32 or 64 rows: the largest power of two that fits the rest
// of the run and of the tile).
//
// Per CTA (persistent, one per SM), 11 warps:
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread t owns
//              query row t of its tile (TMEM lane t)
//   warp 8     TMA producer: Q tiles, K and V boxes into 3-stage rings
//   warp 9     MMA issuer: S_x = Q_x K^T into TMEM (two buffers per tile) and
//              O_x += P_x V into TMEM, issuing whichever is ready; owns TMEM
//   warp 10    item loader: claims the next item of the cost-sorted list from a
//              counter shared by all CTAs and puts its header and key ranges
//              into a 2-slot ring that every other role reads
// P is written by the softmax warps to shared memory (bf16, 128-byte
// swizzled, K-major) so both MMAs read their operands from shared memory.
// O accumulates in TMEM across the item's key tiles; the softmax warps
// rescale it in place only when a row's running max grows by more than 2^8
// (exact: every probability is taken against the same reference max that O
// and the row sum use).
#pragma once
#include "common.cuh"

namespace svg {

constexpr int kItemRows = 256;     // query rows per work item (two 128-row tiles)
constexpr int kSlotsPerTile = 8;   // 8-row slots per 64-key tile

struct AttnItem {  // up to 256 query rows of one q-cluster; h < 0 ends the list
  int32_t h, i, q0, packed;  // packed = rows (<= 256) | key_tiles << 9
};

// Readers of an item slot that must release it before it is refilled: the
// producer, the MMA issuer and the eight softmax warps.
constexpr int kItemReaders = 10;

template <int D>
struct AttnCfg {
  static constexpr int BM = 128, BN = 64, SLOT = 8, NSLOT = BN / SLOT;
  static constexpr int DH = D / 64;  // 64-channel (128-byte) halves
  static constexpr int KST = 3, VST = 3;
  static constexpr int QT_BYTES = BM * D * 2;   // one Q tile
  static constexpr int KV_BYTES = BN * D * 2;   // one K or V tile
  static constexpr int P_BYTES = BM * BN * 2;   // one P tile
  static constexpr int HALF_Q = BM * 128;       // one 64-channel half of a Q tile
  static constexpr int HALF_KV = BN * 128;      // same for a K/V tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * QT_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_P = OFF_V + VST * KV_BYTES;
  static constexpr int MAX_SEL = 1024;                        // selected k-clusters per q-cluster
  static constexpr int OFF_RANGES = OFF_P + 2 * P_BYTES;      // 2 x int2 (first row, rows)
  static constexpr int OFF_BAR = OFF_RANGES + 2 * MAX_SEL * 8;
  static constexpr int SMEM_BYTES = OFF_BAR + 1024 + 1024;    // barriers/meta + alignment slack
  // TMEM: S of tile x in buffer b at x*128 + b*64 (64 columns); O of tile x at 256 + x*128
  static constexpr uint32_t TM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, false, true);
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, LOADER_WARP = 10;
  static constexpr int THREADS = 11 * 32;
  __device__ static constexpr uint32_t tm_s(int x, int b) { return x * 128 + b * 64; }
  __device__ static constexpr uint32_t tm_o(int x) { return 256 + x * 128; }
};

// TMA boxes of 8, 16, 32 and 64 rows (one tensor map each for K and V).
constexpr int kNumBoxSizes = 4;

struct AttnMaps {
  CUtensorMap q;
  CUtensorMap k[kNumBoxSizes];
  CUtensorMap v[kNumBoxSizes];
};

// Sets bits [first, first + count) of a 64-bit mask held in two registers.
__device__ __forceinline__ void set_bits(uint32_t (&m)[2], int first, int count) {
  const int last = first + count;
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const int lo = max(first, 32 * w), hi = min(last, 32 * w + 32);
    if (hi > lo) {
      const int n = hi - lo;
      const uint32_t bits = n >= 32 ? 0xFFFFFFFFu : ((1u << n) - 1u);
      m[w] |= bits << (lo - 32 * w);
    }
  }
}

struct AttnBarriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3], meta_full[3];
  uint64_t s_full[2][2], s_free[2][2];   // [tile][buffer]
  uint64_t p_full[2], o_full[2];         // [tile]
  uint64_t item_full[2], item_empty[2];
  uint64_t drain;
  AttnItem item[2];      // item ring written by the loader warp
  int32_t item_cnt[2];
  uint32_t meta[3][2];   // per V stage: 64-bit key validity mask of the tile
  uint32_t tmem_base;
  int32_t abort_flag;
};

struct AttnParams {
  const int32_t *q_off, *k_off, *sel_count, *sel_cols;
  const AttnItem *items;
  const int32_t *num_items;
  int32_t *next_item;    // work counter: CTAs claim items in list order (zero at launch)
  __nv_bfloat16 *op;
  float *lse;
  const int32_t *perm;   // optional: write row r of a head to row perm[r] (un-permuted output)
  int N, Cq, Ck, BH;
  float scale_log2;      // softmax scale * log2(e)
  uint64_t wait_ns;
  int fault;             // test hook: 1 = never load the query tiles (waits must run out)
};

__device__ __forceinline__ bool attn_wait(AttnBarriers *b, uint64_t *bar, uint32_t parity,
                                          uint64_t ns, uint32_t site) {
  if (mbar_wait(bar, parity, ns)) return true;
  record_error(SVG_ERR_TIMEOUT, site);
  atomicExch(&b->abort_flag, 1);
  return false;
}

__device__ __forceinline__ bool aborted(AttnBarriers *b) {
  return *reinterpret_cast<volatile int32_t *>(&b->abort_flag) != 0;
}

// Every lane waits; the warp proceeds only if all lanes saw the phase, so the
// .sync.aligned tcgen05 loads that follow always run on the full warp.
__device__ __forceinline__ bool attn_warp_wait(AttnBarriers *b, uint64_t *bar, uint32_t parity,
                                               uint64_t ns, uint32_t site) {
  const bool ok = mbar_wait(bar, parity, ns);
  const bool all = __all_sync(0xffffffffu, ok);
  if (!all && lane_id() == 0) {
    record_error(SVG_ERR_TIMEOUT, site);
    atomicExch(&b->abort_flag, 1);
  }
  return all;
}

__device__ __forceinline__ bool warp_aborted(AttnBarriers *b) {
  return __any_sync(0xffffffffu, aborted(b));
}

template <int D>
__global__ void __launch_bounds__(AttnCfg<D>::THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnParams P) {
  using Cfg = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem + Cfg::OFF_Q;
  uint8_t *sK = smem + Cfg::OFF_K;
  uint8_t *sV = smem + Cfg::OFF_V;
  uint8_t *sP = smem + Cfg::OFF_P;
  int2 *sRanges = reinterpret_cast<int2 *>(smem + Cfg::OFF_RANGES);
  AttnBarriers *B = reinterpret_cast<AttnBarriers *>(smem + Cfg::OFF_BAR);
  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());

  if (threadIdx.x == 0) {
    mbar_init(&B->q_full, 1);
    mbar_init(&B->q_empty, 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&B->k_full[s], 1);
      mbar_init(&B->k_empty[s], 1);
      mbar_init(&B->v_full[s], 1);
      mbar_init(&B->v_empty[s], 1);
      mbar_init(&B->meta_full[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(&B->s_full[x][b], 1);
        mbar_init(&B->s_free[x][b], 4);
      }
      mbar_init(&B->p_full[x], 4);
      mbar_init(&B->o_full[x], 1);
      mbar_init(&B->item_full[x], 1);
      mbar_init(&B->item_empty[x], kItemReaders);
    }
    mbar_init(&B->drain, 1);
    B->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == Cfg::MMA_WARP) {
    tmem_alloc(&B->tmem_base, Cfg::TM_COLS);
    tmem_relinquish();
  }
  if (warp == Cfg::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&maps.q);
    for (int b = 0; b < kNumBoxSizes; ++b) {
      tma_prefetch_desc(&maps.k[b]);
      tma_prefetch_desc(&maps.v[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B->tmem_base;
  const int total = *P.num_items;
  const uint64_t ns = P.wait_ns;

  if (warp == Cfg::LOADER_WARP) {
    // ------------------------------------------------------------ item loader
    // Claims the next item of the list (longest first) with an atomic counter,
    // so an SM that finishes early takes more work; after the last item it
    // publishes an end marker (h = -1).
    for (int n = 0;; ++n) {
      const int buf = n & 1;
      bool ok = true;
      if (lane == 0 && n >= 2)
        ok = attn_wait(B, &B->item_empty[buf], ((n >> 1) - 1) & 1, ns, SITE_ATTN_PRODUCER);
      if (!__shfl_sync(0xffffffffu, ok, 0) || warp_aborted(B)) break;
      int w = 0;
      if (lane == 0) w = atomicAdd(P.next_item, 1);
      w = __shfl_sync(0xffffffffu, w, 0);
      if (w >= total) {
        if (lane == 0) {
          B->item[buf] = AttnItem{-1, 0, 0, 0};
          B->item_cnt[buf] = 0;
          __threadfence_block();
          mbar_arrive(&B->item_full[buf]);
        }
        break;
      }
      const AttnItem it = P.items[w];
      const int cnt = min(P.sel_count[it.h * P.Cq + it.i], Cfg::MAX_SEL);
      const int32_t *cols = P.sel_cols + static_cast<size_t>(it.h * P.Cq + it.i) * P.Ck;
      const int32_t *koff = P.k_off + static_cast<size_t>(it.h) * (P.Ck + 1);
      int2 *dst = sRanges + buf * Cfg::MAX_SEL;
      for (int c = lane; c < cnt; c += 32) {
        const int j = cols[c];
        int2 r = make_int2(0, 0);  // out-of-range ids are flagged by the planning kernel
        if (j >= 0 && j < P.Ck) {
          r.x = koff[j];
          r.y = koff[j + 1] - r.x;
        }
        dst[c] = r;
      }
      __syncwarp();
      if (lane == 0) {   // merge touching ranges into runs (same rule as the planning kernel)
        int m = 0, run_end = -1;
        for (int c = 0; c < cnt; ++c) {
          const int2 r = dst[c];
          if (r.y <= 0) continue;
          if (m > 0 && r.x == run_end) {
            dst[m - 1].y += r.y;
          } else {
            dst[m++] = r;
          }
          run_end = r.x + r.y;
        }
        B->item[buf] = it;
        B->item_cnt[buf] = m;
      }
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B->item_full[buf]);
    }
  } else if (warp == Cfg::PRODUCER_WARP) {
    // ------------------------------------------------------------ TMA producer
    uint32_t g = 0;                  // global key-tile counter
    uint32_t nq = 0, gk = 0, gv = 0;  // Q loads, K tiles and V tiles issued (for the drain)
    int n_items = 0;
    if (lane == 0) {
      bool ok = true;
      for (; ok && !aborted(B); ++n_items) {
        const int buf = n_items & 1;
        if (!attn_wait(B, &B->item_full[buf], (n_items >> 1) & 1, ns, SITE_ATTN_PRODUCER)) break;
        const AttnItem it = B->item[buf];
        if (it.h < 0) {                     // end of the list
          mbar_arrive(&B->item_empty[buf]);
          break;
        }
        const int cnt = B->item_cnt[buf];
        const int2 *ranges = sRanges + buf * Cfg::MAX_SEL;
        const int ntk = it.packed >> 9;
        const bool has_b = (it.packed & 0x1FF) > Cfg::BM;
        if (n_items > 0 && !attn_wait(B, &B->q_empty, (n_items - 1) & 1, ns, SITE_ATTN_PRODUCER))
          break;
        if (P.fault != 1) {
          mbar_arrive_expect_tx(&B->q_full, Cfg::QT_BYTES * (has_b ? 2 : 1));
          const int qrow = it.h * P.N + it.q0;
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (x == 1 && !has_b) break;
#pragma unroll
            for (int dh = 0; dh < Cfg::DH; ++dh)
              tma_load_2d(sQ + x * Cfg::QT_BYTES + dh * Cfg::HALF_Q, &maps.q, dh * 64,
                          qrow + x * Cfg::BM, &B->q_full);
          }
          ++nq;
        }
        int ci = 0, cur = 0, left = 0;
        const int pad_row = it.h * P.N;  // unused slots re-read a valid row; they are masked
        for (int t = 0; t < ntk; ++t, ++g) {
          const int ks = static_cast<int>(g % 3);
          const uint32_t kph = (g / 3) & 1;
          // Cut the tile into boxes of 1, 2, 4 or 8 slots (8..64 rows): the
          // largest power of two that fits both the tile and the run rest.
          int box_row[Cfg::NSLOT], box_kind[Cfg::NSLOT], nbox = 0;
          uint32_t mask[2] = {0, 0};
          int sl = 0;
          while (sl < Cfg::NSLOT) {
            while (left <= 0 && ci < cnt) {
              const int2 r = ranges[ci++];
              cur = r.x;
              left = r.y;
            }
            const int space = Cfg::NSLOT - sl;
            const int need = left > 0 ? (left + Cfg::SLOT - 1) / Cfg::SLOT : space;
            int kind = 0;
            while (kind + 1 < kNumBoxSizes && (2 << kind) <= space && (2 << kind) <= need) ++kind;
            const int nsl = 1 << kind;
            if (left > 0) {
              set_bits(mask, sl * Cfg::SLOT, min(left, nsl * Cfg::SLOT));
              box_row[nbox] = it.h * P.N + cur;
              cur += nsl * Cfg::SLOT;
              left -= nsl * Cfg::SLOT;
            } else {
              box_row[nbox] = pad_row;   // no keys left: finite filler rows, masked out
            }
            box_kind[nbox] = kind | (sl << 8);
            ++nbox;
            sl += nsl;
          }
          if (g >= 3 && !attn_wait(B, &B->k_empty[ks], kph ^ 1, ns, SITE_ATTN_PRODUCER)) { ok = false; break; }
          mbar_arrive_expect_tx(&B->k_full[ks], Cfg::KV_BYTES);
          uint8_t *kdst = sK + ks * Cfg::KV_BYTES;
          for (int bx = 0; bx < nbox; ++bx) {
            const int kind = box_kind[bx] & 0xFF, at = box_kind[bx] >> 8;
#pragma unroll
            for (int dh = 0; dh < Cfg::DH; ++dh)
              tma_load_2d(kdst + dh * Cfg::HALF_KV + at * 1024, &maps.k[kind], dh * 64, box_row[bx],
                          &B->k_full[ks]);
          }
          gk = g + 1;
          if (g >= 3 && !attn_wait(B, &B->v_empty[ks], kph ^ 1, ns, SITE_ATTN_PRODUCER)) { ok = false; break; }
          B->meta[ks][0] = mask[0];
          B->meta[ks][1] = mask[1];
          mbar_arrive(&B->meta_full[ks]);
          mbar_arrive_expect_tx(&B->v_full[ks], Cfg::KV_BYTES);
          uint8_t *vdst = sV + ks * Cfg::KV_BYTES;
          for (int bx = 0; bx < nbox; ++bx) {
            const int kind = box_kind[bx] & 0xFF, at = box_kind[bx] >> 8;
#pragma unroll
            for (int dh = 0; dh < Cfg::DH; ++dh)
              tma_load_2d(vdst + dh * Cfg::HALF_KV + at * 1024, &maps.v[kind], dh * 64, box_row[bx],
                          &B->v_full[ks]);
          }
          gv = g + 1;
        }
        mbar_arrive(&B->item_empty[buf]);   // the ranges of this item are no longer read
      }
      // drain: every load issued above lands on a full barrier; wait for the
      // last phase of each so no copy is in flight when the CTA exits.
      if (aborted(B)) {
        if (nq > 0) mbar_wait(&B->q_full, (nq - 1) & 1, 1000000000ull);
        for (uint32_t k = (gk >= 3 ? gk - 3 : 0); k < gk; ++k)
          mbar_wait(&B->k_full[k % 3], (k / 3) & 1, 1000000000ull);
        for (uint32_t k = (gv >= 3 ? gv - 3 : 0); k < gv; ++k)
          mbar_wait(&B->v_full[k % 3], (k / 3) & 1, 1000000000ull);
      }
    }
  } else if (warp == Cfg::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    // Two cursors walk this CTA's key tiles: gs = next tile for S, gp = next
    // tile for PV; each tile has one S (and one PV) per query tile present.
    // Every pass issues whatever is ready (S first), so neither waits behind
    // the other's operands.  The S cursor takes item headers from the item
    // ring and queues them (hq) for the PV cursor, which trails it by up to
    // two items.
    if (lane == 0) {
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV),
                     p_base = smem_u32(sP);
      uint32_t n_hdr = 0, n_s = 0, n_pd = 0;   // headers read, items with all S / all PV issued
      int hq[4] = {0, 0, 0, 0};
      bool s_active = false, s_end = false;
      int ts = 0, tp = 0;
      int pk_s = 0;
      uint32_t gs = 0, gp = 0;
      uint32_t n_sx[2] = {0, 0}, n_px[2] = {0, 0};
      bool s_done[2] = {false, false}, p_done[2] = {false, false};
      bool q_ok = false;
      const long long limit = static_cast<long long>(ns) * 2;
      long long t_last = clock64();
      while (true) {
        bool progress = false;
        if (!s_active && !s_end &&
            mbar_test(&B->item_full[n_hdr & 1], (n_hdr >> 1) & 1)) {   // next item for the S cursor
          const AttnItem it = B->item[n_hdr & 1];
          mbar_arrive(&B->item_empty[n_hdr & 1]);
          ++n_hdr;
          if (it.h < 0) {
            s_end = true;
          } else {
            pk_s = it.packed;
            hq[n_s & 3] = pk_s;
            s_active = true;
            ts = 0;
            q_ok = false;
          }
          progress = true;
        }
        if (s_end && !s_active && n_pd == n_s) break;   // every started item is finished
        if (s_active) {
          const int ks = static_cast<int>(gs % 3);
          const bool has_b = (pk_s & 0x1FF) > Cfg::BM;
          if (!q_ok) q_ok = mbar_test(&B->q_full, n_s & 1);
          if (q_ok && mbar_test(&B->k_full[ks], (gs / 3) & 1)) {
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              if (s_done[x] || (x == 1 && !has_b)) continue;
              const int b = n_sx[x] & 1;
              if (n_sx[x] >= 2 && !mbar_test(&B->s_free[x][b], ((n_sx[x] >> 1) - 1) & 1)) continue;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff_q = (kk >> 2) * Cfg::HALF_Q + (kk & 3) * 32;
                const uint32_t koff_k = (kk >> 2) * Cfg::HALF_KV + (kk & 3) * 32;
                mma_bf16_ss(tmem + Cfg::tm_s(x, b),
                            smem_desc_sw128(q_base + x * Cfg::QT_BYTES + koff_q, 16, 1024),
                            smem_desc_sw128(k_base + ks * Cfg::KV_BYTES + koff_k, 16, 1024),
                            Cfg::IDESC_S, kk > 0 ? 1u : 0u);
              }
              mma_commit(&B->s_full[x][b]);
              ++n_sx[x];
              s_done[x] = true;
              progress = true;
            }
            if (s_done[0] && (s_done[1] || !has_b)) {
              mma_commit(&B->k_empty[ks]);
              if (++ts == (pk_s >> 9)) {         // last S of this item: Q may be replaced
                mma_commit(&B->q_empty);
                ++n_s;
                s_active = false;
              }
              ++gs;
              s_done[0] = s_done[1] = false;
            }
          }
        }
        if (gp < gs) {
          const int pk_p = hq[n_pd & 3];
          const int vs = static_cast<int>(gp % 3);
          const bool has_b = (pk_p & 0x1FF) > Cfg::BM;
          if (mbar_test(&B->v_full[vs], (gp / 3) & 1)) {
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              if (p_done[x] || (x == 1 && !has_b)) continue;
              if (!mbar_test(&B->p_full[x], n_px[x] & 1)) continue;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < Cfg::BN / 16; ++kk) {
                // A = P_x [128 q x 16 keys], K-major; B = V [16 keys x D], MN-major
                mma_bf16_ss(tmem + Cfg::tm_o(x),
                            smem_desc_sw128(p_base + x * Cfg::P_BYTES + kk * 32, 16, 1024),
                            smem_desc_sw128(v_base + vs * Cfg::KV_BYTES + kk * 2048, Cfg::HALF_KV, 1024),
                            Cfg::IDESC_PV, (tp == 0 && kk == 0) ? 0u : 1u);
              }
              mma_commit(&B->o_full[x]);
              ++n_px[x];
              p_done[x] = true;
              progress = true;
            }
            if (p_done[0] && (p_done[1] || !has_b)) {
              mma_commit(&B->v_empty[vs]);
              if (++tp == (pk_p >> 9)) {
                ++n_pd;
                tp = 0;
              }
              ++gp;
              p_done[0] = p_done[1] = false;
            }
          }
        }
        if (progress) {
          t_last = clock64();
        } else if (clock64() - t_last > limit) {
          record_error(SVG_ERR_TIMEOUT, SITE_ATTN_MMA);
          atomicExch(&B->abort_flag, 1);
          break;
        } else if (aborted(B)) {
          break;
        }
      }
      // make sure every issued MMA has retired before TMEM is released
      mma_commit(&B->drain);
      mbar_wait(&B->drain, 0, 1000000000ull);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // Group x = warp / 4 owns query tile x of every item; thread `row` owns
    // TMEM lane `row` (one query row of S_x and O_x).  Probabilities are taken
    // against a reference max m_ref that is raised only when a tile's max
    // exceeds it by more than kRescaleLog2; O_x (in TMEM) and l are rescaled
    // then.  P values stay below 2^kRescaleLog2.
    constexpr float kRescaleLog2 = 8.f;
    const int x = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t o_addr = tmem + lane_off + Cfg::tm_o(x);
    uint8_t *sPx = sP + x * Cfg::P_BYTES;
    const float sl2 = P.scale_log2;
    uint32_t g = 0, n_s = 0, n_o = 0;
    for (uint32_t n = 0; !warp_aborted(B); ++n) {
      if (!attn_warp_wait(B, &B->item_full[n & 1], (n >> 1) & 1, ns, SITE_ATTN_SOFTMAX)) break;
      const AttnItem it = B->item[n & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(&B->item_empty[n & 1]);
      if (it.h < 0) break;                  // end of the list
      const int ntk = it.packed >> 9;
      const int rows_total = it.packed & 0x1FF;
      const int nrows = x == 0 ? min(rows_total, Cfg::BM) : rows_total - Cfg::BM;
      if (nrows <= 0) {          // this item has no tile B
        g += ntk;
        continue;
      }
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int t = 0; t < ntk; ++t, ++g) {
        const int st = static_cast<int>(g % 3);
        const uint32_t ph = (g / 3) & 1;
        const int sb = n_s & 1;
        if (!attn_warp_wait(B, &B->s_full[x][sb], (n_s >> 1) & 1, ns, SITE_ATTN_SOFTMAX) ||
            !attn_warp_wait(B, &B->meta_full[st], ph, ns, SITE_ATTN_SOFTMAX)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t mk[2] = {B->meta[st][0], B->meta[st][1]};
        float sv[2][32];
        tmem_ld64_sync(tmem + lane_off + Cfg::tm_s(x, sb), reinterpret_cast<float(&)[64]>(sv));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B->s_free[x][sb]);   // S buffer may be overwritten now
        ++n_s;
        // masked raw scores and the tile max; the mask is warp-uniform.  The
        // scale (into the log2 domain) is applied once to the max and folded
        // into one FMA per probability below (scale > 0 keeps the order).
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (mk[c] != 0xFFFFFFFFu) {
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[c][e] = ((mk[c] >> e) & 1u) ? sv[c][e] : -INFINITY;
          }
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            mx4[(e >> 1) & 3] = max3f(mx4[(e >> 1) & 3], sv[c][e], sv[c][e + 1]);
        }
        const float mt = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
        float alpha = 1.f;
        if (mt > m_ref + kRescaleLog2) {   // also taken on the first tile (m_ref = -inf)
          alpha = ex2_approx(m_ref - mt);
          m_ref = mt;
        }
        // probabilities -> bf16 pairs, row sum
        // (pairs of scores go through one paired FMA and one paired add)
        float2 rs2 = make_float2(0.f, 0.f);
        uint32_t packed[32];
        const float2 sl2x2 = make_float2(sl2, sl2), nm2 = make_float2(-m_ref, -m_ref);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 a2 = fma_f32x2(make_float2(sv[c][e], sv[c][e + 1]), sl2x2, nm2);
            const float2 p2 = make_float2(ex2_approx(a2.x), ex2_approx(a2.y));
            rs2 = add_f32x2(rs2, p2);
            packed[c * 16 + (e >> 1)] = pack_bf16x2(p2.x, p2.y);
          }
        }
        if (t >= 1) {  // PV_x(t-1) must be done before P_x and O_x are touched
          if (!attn_warp_wait(B, &B->o_full[x], n_o & 1, ns, SITE_ATTN_SOFTMAX)) { ok = false; break; }
          tc_fence_after();
          ++n_o;
          if (__any_sync(0xffffffffu, alpha != 1.f)) {   // rescale O rows in TMEM
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              float ov[32];
              tmem_ld32_sync(o_addr + c * 32, ov);
#pragma unroll
              for (int e = 0; e < 32; ++e) ov[e] *= alpha;
              tmem_st32(o_addr + c * 32, ov);
            }
            tmem_st_wait();
          }
        }
        l = l * alpha + (rs2.x + rs2.y);
        // P row: 64 keys = one 128-byte swizzle row (K-major, 16-byte chunks ^ row % 8)
        uint8_t *prow = sPx + row * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t chunk = u ^ (row & 7);
          *reinterpret_cast<uint4 *>(prow + chunk * 16) =
              make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B->p_full[x]);
      }
      if (!ok) break;
      if (!attn_warp_wait(B, &B->o_full[x], n_o & 1, ns, SITE_ATTN_SOFTMAX)) break;
      tc_fence_after();
      ++n_o;
      const float inv = 1.f / l;
      size_t grow = static_cast<size_t>(it.h) * P.N + it.q0 + x * Cfg::BM + row;
      if (P.perm != nullptr && row < nrows) {   // un-permute fused into the store
        const int t = P.perm[grow];
        if (t >= 0 && t < P.N) {
          grow = static_cast<size_t>(it.h) * P.N + t;
        } else {
          record_error(SVG_ERR_DEVICE_CHECK, SITE_PERMUTE_RANGE);
          grow = static_cast<size_t>(-1);
        }
      }
      const bool store = row < nrows && grow != static_cast<size_t>(-1);
      uint4 *dst = reinterpret_cast<uint4 *>(P.op + (store ? grow : 0) * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float ov[32];
        tmem_ld32_sync(o_addr + c * 32, ov);
        if (store) {
#pragma unroll
          for (int v8 = 0; v8 < 4; ++v8)
            dst[c * 4 + v8] = make_uint4(pack_bf16x2(ov[8 * v8] * inv, ov[8 * v8 + 1] * inv),
                                         pack_bf16x2(ov[8 * v8 + 2] * inv, ov[8 * v8 + 3] * inv),
                                         pack_bf16x2(ov[8 * v8 + 4] * inv, ov[8 * v8 + 5] * inv),
                                         pack_bf16x2(ov[8 * v8 + 6] * inv, ov[8 * v8 + 7] * inv));
        }
      }
      tc_fence_before();
      if (store && P.lse) P.lse[grow] = (m_ref + log2f(l)) * 0.69314718055994531f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TM_COLS);
  }
}

// ------------------------------------------------------------------ planning
// Per (head, q-cluster): number of work items (256 query rows each) and of
// 64-key tiles per item.
__global__ void attn_plan_count_kernel(const int32_t *__restrict__ q_off,
                                       const int32_t *__restrict__ k_off,
                                       const int32_t *__restrict__ sel_count,
                                       const int32_t *__restrict__ sel_cols, int BH, int Cq, int Ck,
                                       int32_t *__restrict__ qtiles, int32_t *__restrict__ ktiles) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= BH * Cq) return;
  const int h = idx / Cq, i = idx % Cq;
  const int nq = q_off[h * (Cq + 1) + i + 1] - q_off[h * (Cq + 1) + i];
  const int cnt = sel_count[idx];
  const int32_t *cols = sel_cols + static_cast<size_t>(idx) * Ck;
  const int32_t *ko = k_off + static_cast<size_t>(h) * (Ck + 1);
  // Selected k-clusters whose row ranges touch (consecutive ids, or ids with
  // only empty clusters between them) form one run: slots are counted per
  // run, exactly as the attention kernel's item loader merges them.
  int slots = 0, run_end = -1, run_len = 0;
  for (int c = 0; c < cnt; ++c) {
    const int j = cols[c];
    if (j < 0 || j >= Ck) {
      record_error(SVG_ERR_DEVICE_CHECK, SITE_ATTN_EMPTY_ROW);
      continue;
    }
    const int r0 = ko[j], len = ko[j + 1] - r0;
    if (len <= 0) continue;
    if (r0 == run_end) {
      run_len += len;
    } else {
      slots += (run_len + 7) >> 3;
      run_len = len;
    }
    run_end = r0 + len;
  }
  slots += (run_len + 7) >> 3;
  int qt = nq > 0 ? (nq + kItemRows - 1) / kItemRows : 0;
  if (qt > 0 && slots == 0) {
    record_error(SVG_ERR_DEVICE_CHECK, SITE_ATTN_EMPTY_ROW);
    qt = 0;
  }
  qtiles[idx] = qt;
  ktiles[idx] = (slots + kSlotsPerTile - 1) / kSlotsPerTile;
}

// Single block: one AttnItem per 256 query rows, in descending order of
// estimated cost (key tiles x query tiles of the item; a counting sort over
// kAttnBuckets buckets).  The attention kernel's CTAs claim items in this
// order from a shared counter (greedy list scheduling, longest first), so an
// SM that drew short items takes more of them.  Also resets that counter.
constexpr int kAttnBuckets = 1024;

__device__ __forceinline__ int attn_item_bucket(int kt, int rows) {
  const int cost = kt * (rows > 128 ? 2 : 1);
  return kAttnBuckets - 1 - min(cost, kAttnBuckets - 1);   // descending cost
}

__global__ void __launch_bounds__(1024) attn_plan_emit_kernel(
    const int32_t *__restrict__ q_off, const int32_t *__restrict__ qtiles,
    const int32_t *__restrict__ ktiles, int BH, int Cq, AttnItem *__restrict__ items,
    int32_t *__restrict__ num_items, int32_t *__restrict__ next_item) {
  __shared__ int hist[kAttnBuckets];
  __shared__ int warp_tot[32];
  const int total = BH * Cq;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  hist[threadIdx.x] = 0;
  if (threadIdx.x == 0) *next_item = 0;
  __syncthreads();
  for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
    const int qt = qtiles[idx];
    if (qt <= 0) continue;
    const int kt = ktiles[idx];
    const int h = idx / Cq, i = idx % Cq;
    const int row0 = q_off[h * (Cq + 1) + i], row1 = q_off[h * (Cq + 1) + i + 1];
    for (int t = 0; t < qt; ++t)
      atomicAdd(&hist[attn_item_bucket(kt, min(kItemRows, row1 - row0 - t * kItemRows))], 1);
  }
  __syncthreads();
  // exclusive scan of the buckets (one per thread)
  const int v = hist[threadIdx.x];
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int t = warp_tot[lane];
    int ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    warp_tot[lane] = ti - t;
  }
  __syncthreads();
  const int excl = warp_tot[w] + incl - v;
  __syncthreads();
  hist[threadIdx.x] = excl;                       // now: next free rank of each bucket
  if (threadIdx.x == kAttnBuckets - 1) *num_items = excl + v;
  __syncthreads();
  for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
    const int qt = qtiles[idx];
    if (qt <= 0) continue;
    const int kt = ktiles[idx];
    const int h = idx / Cq, i = idx % Cq;
    const int row0 = q_off[h * (Cq + 1) + i], row1 = q_off[h * (Cq + 1) + i + 1];
    for (int t = 0; t < qt; ++t) {
      const int q0 = row0 + t * kItemRows;
      const int rows = min(kItemRows, row1 - q0);
      const int rank = atomicAdd(&hist[attn_item_bucket(kt, rows)], 1);
      items[rank] = AttnItem{h, i, q0, rows | (kt << 9)};
    }
  }
}

}  // namespace svg
