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
// into 8-row slots; 16 slots form a 128-key tile.  A run of n rows costs
// ceil(n/8) slots and at most 7 masked rows, fetched with as few TMA boxes as
// possible (8 to 128 rows: the largest power of two that fits the rest of the
// run and of the tile).
//
// Tensor-core shape: every MMA chain accumulates into one TMEM accumulator
// (S = Q K^T: M=128, N=128 keys, D/16 steps; O += P V: M=128, N=D, 8 steps).
// Measured on B200, a chain of M=128 MMAs into one accumulator runs at ~97 %
// of the dense bf16 rate for N >= 128 (~63 % at N = 64), while alternating
// accumulators instruction by instruction costs ~150 cycles per MMA; so the
// kernel issues whole chains and never interleaves them.
//
// Per CTA (persistent, one per SM), 11 warps:
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread t owns
//              query row t of its tile (TMEM lane t)
//   warp 8     TMA producer: Q tiles; K and V tiles through one ring, in the
//              order the MMAs consume them: K0, K1, V0, K2, V1, ..., V(n-1)
//   warp 9     MMA issuer: walks the same sequence; for a K entry issues
//              S_x = Q_x K^T of both tiles, for a V entry O_x += P_x V; owns TMEM
//   warp 10    item loader: claims the next item from a counter shared by all
//              CTAs (list sorted by head group, then longest first), prefetches
//              its query rows into L2, merges its key ranges into runs
// S_x has one TMEM buffer per tile; the softmax copies it to registers and
// releases it at once, so S_x(t+1) runs on the tensor cores while the softmax
// of tile t computes.  P is written by the softmax warps to shared memory
// (bf16, 128-byte swizzled, K-major), so both MMAs read shared memory.  O
// accumulates in TMEM across the item's key tiles; the softmax warps rescale
// it in place only when a row's running max grows by more than 2^8 (exact:
// every probability is taken against the same reference max that O and the
// row sum use).
#pragma once
#include "common.cuh"

namespace svg {

constexpr int kItemRows = 256;     // query rows per work item (two 128-row tiles)
constexpr int kSlotsPerTile = 16;  // 8-row slots per 128-key tile
constexpr int kMetaRing = 8;       // key-validity masks in flight

struct AttnItem {  // up to 256 query rows of one q-cluster; h < 0 ends the list
  int32_t h, i, q0, packed;  // packed = rows (<= 256) | key_tiles << 9
};

// Readers of an item header slot that must release it before it is refilled:
// the producer, the MMA issuer and the eight softmax warps.
constexpr int kItemReaders = 10;

template <int D>
struct AttnCfg {
  static constexpr int BM = 128, BN = 128, SLOT = 8, NSLOT = BN / SLOT;
  static constexpr int DH = D / 64;                   // 64-channel (128-byte) halves
  static constexpr int KVST = D == 128 ? 2 : 4;       // K/V ring slots
  static constexpr int QT_BYTES = BM * D * 2;         // one Q tile
  static constexpr int KV_BYTES = BN * D * 2;         // one K or V tile
  static constexpr int P_BYTES = BM * BN * 2;         // one P tile
  static constexpr int HALF_Q = BM * 128;             // one 64-channel half of a Q tile
  static constexpr int HALF_KV = BN * 128;            // same for a K/V tile
  static constexpr int HALF_P = BM * 128;             // one 64-key half of a P tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + 2 * QT_BYTES;
  static constexpr int OFF_P = OFF_KV + KVST * KV_BYTES;
  static constexpr int MAX_SEL = 1024;                // selected k-clusters per q-cluster
  static constexpr int OFF_RANGES = OFF_P + 2 * P_BYTES;   // int2 (first row, rows) per run
  static constexpr int OFF_BAR = OFF_RANGES + MAX_SEL * 8;
  static constexpr int SMEM_BYTES = OFF_BAR + 1024 + 1024;  // barriers/meta + alignment slack
  // TMEM: S of tile x at x*128 (128 columns); O of tile x at 256 + x*128
  static constexpr uint32_t TM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, false, true);
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, LOADER_WARP = 10;
  static constexpr int THREADS = 11 * 32;
  __device__ static constexpr uint32_t tm_s(int x) { return x * 128; }
  __device__ static constexpr uint32_t tm_o(int x) { return 256 + x * 128; }
};

// TMA boxes of 8, 16, 32, 64 and 128 rows (one tensor map each for K and V).
constexpr int kNumBoxSizes = 5;

struct AttnMaps {
  CUtensorMap q;
  CUtensorMap k[kNumBoxSizes];
  CUtensorMap v[kNumBoxSizes];
};

// Entry e of an item with n key tiles in the ring order K0, K1, V0, K2, V1,
// ..., K(n-1), V(n-2), V(n-1): returns the key tile and sets is_k.
__device__ __forceinline__ int attn_entry(int n, int e, bool &is_k) {
  if (e == 0) { is_k = true; return 0; }
  if (e == 2 * n - 1) { is_k = false; return n - 1; }
  is_k = (e & 1) != 0;
  return is_k ? (e + 1) >> 1 : (e >> 1) - 1;
}

// Sets bits [first, first + count) of a 128-bit mask held in four registers.
__device__ __forceinline__ void set_bits(uint32_t (&m)[4], int first, int count) {
  const int last = first + count;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
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
  uint64_t kv_full[4], kv_empty[4];
  uint64_t meta_full[kMetaRing];
  uint64_t s_full[2], s_free[2], p_full[2], o_full[2];   // [tile]
  uint64_t item_full[2], item_empty[2];
  uint64_t ranges_full, ranges_empty;
  uint64_t drain;
  AttnItem item[2];      // item header ring written by the loader warp
  int32_t ranges_cnt;    // runs of the item whose ranges are in shared memory
  uint32_t meta[kMetaRing][4];   // per key tile: 128-bit key validity mask
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
  unsigned long long *issued;   // optional: += (query tile, key tile) pairs issued
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

// Number of selected k-clusters of a block-list row, clamped to [0, limit];
// a count outside that range is recorded as a device check failure.
__device__ __forceinline__ int attn_sel_count(const int32_t *sel_count, size_t row, int limit) {
  const int c = sel_count[row];
  if (c < 0 || c > limit) {
    record_error(SVG_ERR_DEVICE_CHECK, SITE_ATTN_EMPTY_ROW);
    return c < 0 ? 0 : limit;
  }
  return c;
}

template <int D>
__global__ void __launch_bounds__(AttnCfg<D>::THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnParams P) {
  using Cfg = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem + Cfg::OFF_Q;
  uint8_t *sKV = smem + Cfg::OFF_KV;
  uint8_t *sP = smem + Cfg::OFF_P;
  int2 *sRanges = reinterpret_cast<int2 *>(smem + Cfg::OFF_RANGES);
  AttnBarriers *B = reinterpret_cast<AttnBarriers *>(smem + Cfg::OFF_BAR);
  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());

  if (threadIdx.x == 0) {
    mbar_init(&B->q_full, 1);
    mbar_init(&B->q_empty, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&B->kv_full[s], 1);
      mbar_init(&B->kv_empty[s], 1);
    }
    for (int s = 0; s < kMetaRing; ++s) mbar_init(&B->meta_full[s], 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&B->s_full[x], 1);
      mbar_init(&B->s_free[x], 4);
      mbar_init(&B->p_full[x], 4);
      mbar_init(&B->o_full[x], 1);
      mbar_init(&B->item_full[x], 1);
      mbar_init(&B->item_empty[x], kItemReaders);
    }
    mbar_init(&B->ranges_full, 1);
    mbar_init(&B->ranges_empty, 1);
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
    // Claims the next item of the list with an atomic counter, so an SM that
    // finishes early takes more work; after the last item it publishes an end
    // marker (h = -1).  The key ranges have one shared-memory slot: the
    // ranges of item n are written once the producer has finished item n-1.
    const int max_sel = min(P.Ck, Cfg::MAX_SEL);
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
          __threadfence_block();
          mbar_arrive(&B->item_full[buf]);
        }
        break;
      }
      const AttnItem it = P.items[w];
      if (lane < 2 * Cfg::DH && (lane / Cfg::DH) * Cfg::BM < (it.packed & 0x1FF))   // query rows -> L2
        tma_prefetch_l2_2d(&maps.q, (lane % Cfg::DH) * 64, it.h * P.N + it.q0 + (lane / Cfg::DH) * Cfg::BM);
      const size_t row = static_cast<size_t>(it.h) * P.Cq + it.i;
      const int cnt = attn_sel_count(P.sel_count, row, max_sel);
      const int32_t *cols = P.sel_cols + row * P.Ck;
      const int32_t *koff = P.k_off + static_cast<size_t>(it.h) * (P.Ck + 1);
      ok = true;
      if (lane == 0 && n >= 1) ok = attn_wait(B, &B->ranges_empty, (n - 1) & 1, ns, SITE_ATTN_PRODUCER);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      for (int c = lane; c < cnt; c += 32) {
        const int j = cols[c];
        int2 r = make_int2(0, 0);  // out-of-range ids are flagged by the planning kernel
        if (j >= 0 && j < P.Ck) {
          r.x = koff[j];
          r.y = koff[j + 1] - r.x;
        }
        sRanges[c] = r;
      }
      __syncwarp();
      if (lane == 0) {   // merge touching ranges into runs (same rule as the planning kernel)
        int m = 0, run_end = -1;
        for (int c = 0; c < cnt; ++c) {
          const int2 r = sRanges[c];
          if (r.y <= 0) continue;
          if (m > 0 && r.x == run_end) {
            sRanges[m - 1].y += r.y;
          } else {
            sRanges[m++] = r;
          }
          run_end = r.x + r.y;
        }
        B->ranges_cnt = m;
        B->item[buf] = it;
        __threadfence_block();
        mbar_arrive(&B->ranges_full);
        mbar_arrive(&B->item_full[buf]);
      }
      __syncwarp();
    }
  } else if (warp == Cfg::PRODUCER_WARP) {
    // ------------------------------------------------------------ TMA producer
    uint32_t g = 0;         // global key-tile counter
    uint32_t e = 0;         // global ring-entry counter (K and V tiles issued)
    uint32_t nq = 0;        // Q loads issued (for the drain)
    if (lane == 0) {
      bool ok = true;
      for (int n = 0; ok && !aborted(B); ++n) {
        const int buf = n & 1;
        if (!attn_wait(B, &B->item_full[buf], (n >> 1) & 1, ns, SITE_ATTN_PRODUCER)) break;
        const AttnItem it = B->item[buf];
        if (it.h < 0) {                     // end of the list
          mbar_arrive(&B->item_empty[buf]);
          break;
        }
        if (!attn_wait(B, &B->ranges_full, n & 1, ns, SITE_ATTN_PRODUCER)) break;
        const int cnt = B->ranges_cnt;
        const int ntk = it.packed >> 9;
        const bool has_b = (it.packed & 0x1FF) > Cfg::BM;
        if (n > 0 && !attn_wait(B, &B->q_empty, (n - 1) & 1, ns, SITE_ATTN_PRODUCER)) break;
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
        // box lists of the last two key tiles (a V tile is issued after the
        // next tile's K): row and (kind | slot << 8) of every box
        int box_row[2][Cfg::NSLOT], box_kind[2][Cfg::NSLOT], nbox[2] = {0, 0};
        int ci = 0, cur = 0, left = 0;
        const int pad_row = it.h * P.N;  // unused slots re-read a valid row; they are masked
        for (int en = 0; en < 2 * ntk && ok; ++en) {
          bool is_k;
          const int t = attn_entry(ntk, en, is_k);
          const int lb = t & 1;
          if (is_k) {
            // cut tile t into boxes of 1..16 slots (8..128 rows): the largest
            // power of two that fits both the tile and the rest of the run
            uint32_t mask[4] = {0, 0, 0, 0};
            int sl = 0, nb = 0;
            while (sl < Cfg::NSLOT) {
              while (left <= 0 && ci < cnt) {
                const int2 r = sRanges[ci++];
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
                box_row[lb][nb] = it.h * P.N + cur;
                cur += nsl * Cfg::SLOT;
                left -= nsl * Cfg::SLOT;
              } else {
                box_row[lb][nb] = pad_row;   // no keys left: finite filler rows, masked out
              }
              box_kind[lb][nb] = kind | (sl << 8);
              ++nb;
              sl += nsl;
            }
            nbox[lb] = nb;
            if (t == ntk - 1) mbar_arrive(&B->ranges_empty);   // the ranges are no longer read
            const int mi = static_cast<int>(g % kMetaRing);
#pragma unroll
            for (int w = 0; w < 4; ++w) B->meta[mi][w] = mask[w];
            mbar_arrive(&B->meta_full[mi]);
            ++g;
          }
          const int slot = static_cast<int>(e % Cfg::KVST);
          if (e >= static_cast<uint32_t>(Cfg::KVST) &&
              !attn_wait(B, &B->kv_empty[slot], ((e / Cfg::KVST) - 1) & 1, ns, SITE_ATTN_PRODUCER)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&B->kv_full[slot], Cfg::KV_BYTES);
          uint8_t *dst = sKV + slot * Cfg::KV_BYTES;
          const CUtensorMap *maps_t = is_k ? maps.k : maps.v;
          for (int bx = 0; bx < nbox[lb]; ++bx) {
            const int kind = box_kind[lb][bx] & 0xFF, at = box_kind[lb][bx] >> 8;
#pragma unroll
            for (int dh = 0; dh < Cfg::DH; ++dh)
              tma_load_2d(dst + dh * Cfg::HALF_KV + at * 1024, &maps_t[kind], dh * 64, box_row[lb][bx],
                          &B->kv_full[slot]);
          }
          ++e;
        }
        mbar_arrive(&B->item_empty[buf]);
      }
      // drain: every load issued above lands on a full barrier; wait for the
      // last phase of each so no copy is in flight when the CTA exits.
      if (aborted(B)) {
        if (nq > 0) mbar_wait(&B->q_full, (nq - 1) & 1, 1000000000ull);
        for (uint32_t k = (e >= static_cast<uint32_t>(Cfg::KVST) ? e - Cfg::KVST : 0); k < e; ++k)
          mbar_wait(&B->kv_full[k % Cfg::KVST], (k / Cfg::KVST) & 1, 1000000000ull);
      }
    }
  } else if (warp == Cfg::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    // Walks the ring entries in the producer's order.  For a K entry it
    // issues S_x = Q_x K^T for each present tile x once S_x's buffer has been
    // read by the softmax; for a V entry O_x += P_x V once P_x is written.
    // The two tiles of an entry are issued independently (whichever is ready
    // first); the ring slot is released when both have been issued.
    if (lane == 0) {
      // descriptors built once: Q and P tiles (per query tile), ring slot 0 as a
      // K operand (K-major) and as a V operand (MN-major); a slot adds its offset
      const SmemDesc qd[2] = {make_desc_sw128(smem_u32(sQ), 16, 1024),
                              make_desc_sw128(smem_u32(sQ) + Cfg::QT_BYTES, 16, 1024)};
      const SmemDesc pd[2] = {make_desc_sw128(smem_u32(sP), 16, 1024),
                              make_desc_sw128(smem_u32(sP) + Cfg::P_BYTES, 16, 1024)};
      const SmemDesc kd0 = make_desc_sw128(smem_u32(sKV), 16, 1024);
      const SmemDesc vd0 = make_desc_sw128(smem_u32(sKV), Cfg::HALF_KV, 1024);
      uint32_t n_hdr = 0, n_item = 0, e = 0;
      uint32_t n_s[2] = {0, 0}, n_pv[2] = {0, 0};
      bool have = false, finished = false, q_ok = false;
      bool done[2] = {false, false};
      int ntk = 0, en = 0;
      bool has_b = false;
      unsigned long long pairs = 0;
      const long long limit = static_cast<long long>(ns) * 2;
      long long t_last = clock64();
      while (!finished) {
        bool progress = false;
        if (!have && mbar_test(&B->item_full[n_hdr & 1], (n_hdr >> 1) & 1)) {
          const AttnItem it = B->item[n_hdr & 1];
          mbar_arrive(&B->item_empty[n_hdr & 1]);
          ++n_hdr;
          if (it.h < 0) {
            finished = true;
            break;
          }
          ntk = it.packed >> 9;
          has_b = (it.packed & 0x1FF) > Cfg::BM;
          en = 0;
          q_ok = false;
          have = true;
          progress = true;
        }
        if (have) {
          bool is_k;
          const int t = attn_entry(ntk, en, is_k);
          const int slot = static_cast<int>(e % Cfg::KVST);
          if (mbar_test(&B->kv_full[slot], (e / Cfg::KVST) & 1)) {
            const uint32_t slot_off = (slot * Cfg::KV_BYTES) >> 4;
            if (is_k && !q_ok) q_ok = mbar_test(&B->q_full, n_item & 1);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              if (done[x] || (x == 1 && !has_b)) continue;
              if (is_k) {
                if (!q_ok) continue;
                if (n_s[x] >= 1 && !mbar_test(&B->s_free[x], (n_s[x] - 1) & 1)) continue;
                tc_fence_after();
                mma_chain<D / 16, Cfg::HALF_Q, 32, Cfg::HALF_KV, 32>(
                    tmem + Cfg::tm_s(x), qd[x], SmemDesc{kd0.lo + slot_off, kd0.hi}, Cfg::IDESC_S, 0u);
                mma_commit(&B->s_full[x]);
                ++n_s[x];
              } else {
                if (!mbar_test(&B->p_full[x], n_pv[x] & 1)) continue;
                tc_fence_after();
                // A = P_x [128 q x 128 keys], K-major in two 64-key halves; B = V [128 keys x D],
                // MN-major, 16 keys = 2048 bytes per K-step
                mma_chain<Cfg::BN / 16, Cfg::HALF_P, 32, 4 * 2048, 2048>(
                    tmem + Cfg::tm_o(x), pd[x], SmemDesc{vd0.lo + slot_off, vd0.hi}, Cfg::IDESC_PV,
                    t > 0 ? 1u : 0u);
                mma_commit(&B->o_full[x]);
                ++n_pv[x];
                ++pairs;
              }
              done[x] = true;
              progress = true;
            }
            if (done[0] && (done[1] || !has_b)) {
              mma_commit(&B->kv_empty[slot]);
              if (is_k && t == ntk - 1) mma_commit(&B->q_empty);   // the item's last S: Q may be replaced
              ++e;
              done[0] = done[1] = false;
              if (++en == 2 * ntk) {
                have = false;
                ++n_item;
              }
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
      if (P.issued != nullptr && pairs > 0) atomicAdd(P.issued, pairs);
      // make sure every issued MMA has retired before TMEM is released
      mma_commit(&B->drain);
      mbar_wait(&B->drain, 0, 1000000000ull);
    }
  } else if (warp < 8) {
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
        const int mi = static_cast<int>(g % kMetaRing);
        if (!attn_warp_wait(B, &B->s_full[x], n_s & 1, ns, SITE_ATTN_SOFTMAX) ||
            !attn_warp_wait(B, &B->meta_full[mi], (g / kMetaRing) & 1, ns, SITE_ATTN_SOFTMAX)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t mk[4] = {B->meta[mi][0], B->meta[mi][1], B->meta[mi][2], B->meta[mi][3]};
        float sv[128];
        tmem_ld128_sync(tmem + lane_off + Cfg::tm_s(x), sv);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B->s_free[x]);   // S buffer may be overwritten now
        ++n_s;
        // masked raw scores and the tile max; the mask is warp-uniform.  The
        // scale (into the log2 domain) is applied once to the max and folded
        // into one FMA per probability below (scale > 0 keeps the order).
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (mk[c] != 0xFFFFFFFFu) {
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[c * 32 + e] = ((mk[c] >> e) & 1u) ? sv[c * 32 + e] : -INFINITY;
          }
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            mx4[(e >> 1) & 3] = max3f(mx4[(e >> 1) & 3], sv[c * 32 + e], sv[c * 32 + e + 1]);
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
        uint32_t packed[64];
        const float2 sl2x2 = make_float2(sl2, sl2), nm2 = make_float2(-m_ref, -m_ref);
#pragma unroll
        for (int e = 0; e < 128; e += 2) {
          const float2 a2 = fma_f32x2(make_float2(sv[e], sv[e + 1]), sl2x2, nm2);
          const float2 p2 = make_float2(ex2_approx(a2.x), ex2_approx(a2.y));
          rs2 = add_f32x2(rs2, p2);
          packed[e >> 1] = pack_bf16x2(p2.x, p2.y);
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
        // P row: two 64-key halves, each one 128-byte swizzle row (K-major,
        // 16-byte chunks XOR row % 8)
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
          uint8_t *prow = sPx + kh * Cfg::HALF_P + row * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t chunk = u ^ (row & 7);
            const int b = kh * 32 + 4 * u;
            *reinterpret_cast<uint4 *>(prow + chunk * 16) =
                make_uint4(packed[b], packed[b + 1], packed[b + 2], packed[b + 3]);
          }
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
// 128-key tiles per item.
__global__ void attn_plan_count_kernel(const int32_t *__restrict__ q_off,
                                       const int32_t *__restrict__ k_off,
                                       const int32_t *__restrict__ sel_count,
                                       const int32_t *__restrict__ sel_cols, int BH, int Cq, int Ck,
                                       int max_sel, int32_t *__restrict__ qtiles,
                                       int32_t *__restrict__ ktiles) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= BH * Cq) return;
  const int h = idx / Cq, i = idx % Cq;
  const int nq = q_off[h * (Cq + 1) + i + 1] - q_off[h * (Cq + 1) + i];
  const int cnt = attn_sel_count(sel_count, idx, max_sel);
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

// Single block: one AttnItem per 256 query rows, ordered by head group, then
// by descending estimated cost inside a group (key tiles x query tiles; a
// counting sort over kAttnBuckets buckets).  The attention kernel's CTAs
// claim items in this order from a shared counter: a group's K/V (a few heads)
// stays in L2 while its items run, and inside the group the longest items go
// first (greedy list scheduling), so an SM that drew short items takes more
// of them.  Also resets that counter.
constexpr int kAttnBuckets = 1024;
constexpr int kAttnGroups = 16;                            // head groups
constexpr int kAttnCostBuckets = kAttnBuckets / kAttnGroups;

__device__ __forceinline__ int attn_item_bucket(int h, int heads_per_group, int kt, int rows) {
  const int cost = kt * (rows > 128 ? 2 : 1);
  const int grp = min(h / heads_per_group, kAttnGroups - 1);
  return grp * kAttnCostBuckets + kAttnCostBuckets - 1 - min(cost, kAttnCostBuckets - 1);
}

__global__ void __launch_bounds__(1024) attn_plan_emit_kernel(
    const int32_t *__restrict__ q_off, const int32_t *__restrict__ qtiles,
    const int32_t *__restrict__ ktiles, int BH, int Cq, AttnItem *__restrict__ items,
    int32_t *__restrict__ num_items, int32_t *__restrict__ next_item) {
  __shared__ int hist[kAttnBuckets];
  __shared__ int warp_tot[32];
  const int total = BH * Cq;
  const int hpg = (BH + kAttnGroups - 1) / kAttnGroups;
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
      atomicAdd(&hist[attn_item_bucket(h, hpg, kt, min(kItemRows, row1 - row0 - t * kItemRows))], 1);
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
      const int rank = atomicAdd(&hist[attn_item_bucket(h, hpg, kt, rows)], 1);
      items[rank] = AttnItem{h, i, q0, rows | (kt << 9)};
    }
  }
}

}  // namespace svg
