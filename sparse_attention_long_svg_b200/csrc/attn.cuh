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
// Per CTA (persistent, one per SM), 12 warps:
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread t owns
//              query row t of its tile (TMEM lane t)
//   warp 8     TMA producer: Q tiles; K and V tiles of every key tile into
//              two rings (two slots each at D = 128)
//   warps 9, 11 MMA issuers, one per query tile (warp 9 owns TMEM): the
//              sequence S(0), PV(0), S(1), PV(1), ... with S_x = Q_x K^T (A and
//              B in shared memory) and O_x += P_x V (A = P in tensor memory)
//   warp 10    item loader: claims the next item from a counter shared by all
//              CTAs (list sorted by head group, then longest first), prefetches
//              its query rows into L2, merges its key ranges into runs
// Tensor memory per query tile x: S_x (128 fp32 columns) and O_x (D
// columns).  The softmax reads S_x(t) into registers and writes P_x(t) as
// bf16 pairs over the first 64 columns of S_x, where the PV MMA takes it as
// its A operand; S_x(t+1) is issued after PV_x(t), and MMAs run in issue
// order, so it overwrites P only after PV has read it.  The two query tiles
// alternate on the tensor pipe: one tile's MMAs run while the other's
// softmax computes.  O accumulates in TMEM across the item's key tiles; the
// softmax warps rescale it in place only when a row's running max grows by
// more than 2^8 (exact: every probability is taken against the same
// reference max that O and the row sum use).
#pragma once
#include "common.cuh"

namespace svg {

#ifndef SVG_EXP_POLY_PAIRS
#define SVG_EXP_POLY_PAIRS 0
#endif
#ifndef SVG_PACK_INT
#define SVG_PACK_INT 0
#endif

constexpr int kItemRows = 256;     // query rows per work item (two 128-row tiles)
constexpr int kSlotsPerTile = 16;  // 8-row slots per 128-key tile
constexpr int kMetaRing = 8;       // key-validity masks in flight

struct AttnItem {  // up to 256 query rows of one q-cluster; h < 0 ends the list
  int32_t h, i, q0, packed;  // packed = rows (<= 256) | key_tiles << 9
};

// Readers of an item header slot that must release it before it is refilled:
// the producer, the two MMA issuers and the eight softmax warps.
constexpr int kItemReaders = 11;

template <int D>
struct AttnCfg {
  static constexpr int BM = 128, BN = 128, SLOT = 8, NSLOT = BN / SLOT;
  static constexpr int DH = D / 64;                   // 64-channel (128-byte) halves
  static constexpr int KST = D == 128 ? 2 : 4;        // K ring slots (same for V)
  static constexpr int QT_BYTES = BM * D * 2;         // one Q tile
  static constexpr int KV_BYTES = BN * D * 2;         // one K or V tile
  static constexpr int HALF_Q = BM * 128;             // one 64-channel half of a Q tile
  static constexpr int HALF_KV = BN * 128;            // same for a K/V tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * QT_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int MAX_SEL = 1024;                // selected k-clusters per q-cluster
  static constexpr int OFF_RANGES = OFF_V + KST * KV_BYTES;   // int2 (first row, rows) per run
  static constexpr int OFF_BAR = OFF_RANGES + MAX_SEL * 8;
  static constexpr int SMEM_BYTES = OFF_BAR + 1024 + 1024;  // barriers/meta + alignment slack
  // TMEM: S (then P) of tile x at x*128 (128 columns); O of tile x at 256 + x*128
  static constexpr uint32_t TM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, false, true);
  // warp 9 issues tile A's MMAs (and owns TMEM), warp 11 tile B's
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, LOADER_WARP = 10, MMA_B_WARP = 11;
  static constexpr int THREADS = 12 * 32;
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
  uint64_t q_full, q_empty[2];                      // q_empty: [tile]
  uint64_t k_full[4], v_full[4];
  uint64_t k_empty[2][4], v_empty[2][4];            // [tile][slot]: released by that tile's MMAs
  uint64_t meta_full[kMetaRing];
  uint64_t s_full[2], p_full[2], o_full[2];   // [tile]
  uint64_t exp_done[2];                       // [tile]: its four softmax warps finished a step's exponentials
  uint64_t item_full[2], item_empty[2];
  uint64_t ranges_full, ranges_empty;
  uint64_t drain[2];
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
  uint8_t *sK = smem + Cfg::OFF_K;
  uint8_t *sV = smem + Cfg::OFF_V;
  int2 *sRanges = reinterpret_cast<int2 *>(smem + Cfg::OFF_RANGES);
  AttnBarriers *B = reinterpret_cast<AttnBarriers *>(smem + Cfg::OFF_BAR);
  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());

  if (threadIdx.x == 0) {
    mbar_init(&B->q_full, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&B->k_full[s], 1);
      mbar_init(&B->v_full[s], 1);
      for (int x = 0; x < 2; ++x) {
        mbar_init(&B->k_empty[x][s], 1);
        mbar_init(&B->v_empty[x][s], 1);
      }
    }
    for (int s = 0; s < kMetaRing; ++s) mbar_init(&B->meta_full[s], 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&B->s_full[x], 1);
      mbar_init(&B->p_full[x], 4);
      mbar_init(&B->exp_done[x], 4);
      mbar_init(&B->o_full[x], 1);
      mbar_init(&B->item_full[x], 1);
      mbar_init(&B->item_empty[x], kItemReaders);
      mbar_init(&B->q_empty[x], 1);
      mbar_init(&B->drain[x], 1);
    }
    mbar_init(&B->ranges_full, 1);
    mbar_init(&B->ranges_empty, 1);
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
    // Per item: the Q tiles, then K(t) and V(t) of every key tile t (both
    // through the same box list).  K(t + KST) waits for S(t) of both query
    // tiles, V(t + KST) for PV(t).
    uint32_t g = 0;         // global key-tile counter
    uint32_t nq = 0;        // Q loads issued (for the drain)
    uint32_t gk = 0, gv = 0;   // K and V tiles issued (for the drain)
    // A slot (and Q) is reused once every query tile of its last occupant has
    // released it: tile A is in every item, tile B only in items of > 128
    // rows; slot_b[s] = whether the slot's last occupant had tile B,
    // rel_b[s] / nq_b = tile-B releases of the slot / of Q expected so far.
    bool slot_b[4] = {false, false, false, false}, prev_b = false;
    uint32_t rel_b[4] = {0, 0, 0, 0}, nq_b = 0;
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
        if (n > 0 && (!attn_wait(B, &B->q_empty[0], (n - 1) & 1, ns, SITE_ATTN_PRODUCER) ||
                      (prev_b && !attn_wait(B, &B->q_empty[1], (nq_b - 1) & 1, ns, SITE_ATTN_PRODUCER))))
          break;
        prev_b = has_b;
        if (has_b) ++nq_b;
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
        for (int t = 0; t < ntk && ok; ++t, ++g) {
          // cut tile t into boxes of 1..16 slots (8..128 rows): the largest
          // power of two that fits both the tile and the rest of the run
          int box_row[Cfg::NSLOT], box_kind[Cfg::NSLOT], nb = 0;
          uint32_t mask[4] = {0, 0, 0, 0};
          int sl = 0;
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
              box_row[nb] = it.h * P.N + cur;
              cur += nsl * Cfg::SLOT;
              left -= nsl * Cfg::SLOT;
            } else {
              box_row[nb] = pad_row;   // no keys left: finite filler rows, masked out
            }
            box_kind[nb] = kind | (sl << 8);
            ++nb;
            sl += nsl;
          }
          if (t == ntk - 1) mbar_arrive(&B->ranges_empty);   // the ranges are no longer read
          const int mi = static_cast<int>(g % kMetaRing);
#pragma unroll
          for (int w = 0; w < 4; ++w) B->meta[mi][w] = mask[w];
          mbar_arrive(&B->meta_full[mi]);
          const int slot = static_cast<int>(g % Cfg::KST);
          const uint32_t ph = ((g / Cfg::KST) - 1) & 1;
          const bool reuse_b = g >= static_cast<uint32_t>(Cfg::KST) && slot_b[slot];
          const uint32_t ph_b = (rel_b[slot] - 1) & 1;
#pragma unroll
          for (int kv = 0; kv < 2; ++kv) {     // K(t), then V(t)
            uint64_t *full = kv ? &B->v_full[slot] : &B->k_full[slot];
            if (g >= static_cast<uint32_t>(Cfg::KST) &&
                (!attn_wait(B, kv ? &B->v_empty[0][slot] : &B->k_empty[0][slot], ph, ns, SITE_ATTN_PRODUCER) ||
                 (reuse_b && !attn_wait(B, kv ? &B->v_empty[1][slot] : &B->k_empty[1][slot], ph_b, ns,
                                        SITE_ATTN_PRODUCER)))) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(full, Cfg::KV_BYTES);
            uint8_t *dst = (kv ? sV : sK) + slot * Cfg::KV_BYTES;
            const CUtensorMap *maps_t = kv ? maps.v : maps.k;
            for (int bx = 0; bx < nb; ++bx) {
              const int kind = box_kind[bx] & 0xFF, at = box_kind[bx] >> 8;
#pragma unroll
              for (int dh = 0; dh < Cfg::DH; ++dh)
                tma_load_2d(dst + dh * Cfg::HALF_KV + at * 1024, &maps_t[kind], dh * 64, box_row[bx], full);
            }
            if (kv)
              gv = g + 1;
            else
              gk = g + 1;
          }
          slot_b[slot] = has_b;
          if (has_b) ++rel_b[slot];
        }
        mbar_arrive(&B->item_empty[buf]);
      }
      // drain: every load issued above lands on a full barrier; wait for the
      // last phase of each so no copy is in flight when the CTA exits.
      if (aborted(B)) {
        if (nq > 0) mbar_wait(&B->q_full, (nq - 1) & 1, 1000000000ull);
        for (uint32_t k = (gk >= static_cast<uint32_t>(Cfg::KST) ? gk - Cfg::KST : 0); k < gk; ++k)
          mbar_wait(&B->k_full[k % Cfg::KST], (k / Cfg::KST) & 1, 1000000000ull);
        for (uint32_t k = (gv >= static_cast<uint32_t>(Cfg::KST) ? gv - Cfg::KST : 0); k < gv; ++k)
          mbar_wait(&B->v_full[k % Cfg::KST], (k / Cfg::KST) & 1, 1000000000ull);
      }
    }
  } else if (warp == Cfg::MMA_WARP || warp == Cfg::MMA_B_WARP) {
    // ------------------------------------------------------------ MMA issuers
    // One thread per query tile x issues that tile's sequence S(0), PV(0),
    // S(1), PV(1), ... of every item that has the tile: S_x(t) once K(t) (and
    // Q) has landed, PV_x(t) once the softmax has written P_x(t) and V(t) has
    // landed.  It releases each K/V slot and Q for its own tile; the producer
    // reuses them when every present tile has released them.  Two issuers let
    // one tile's chain queue on the tensor pipe while the other's executes.
    const int x = warp == Cfg::MMA_WARP ? 0 : 1;
    if (lane == 0) {
      const SmemDesc qd = make_desc_sw128(smem_u32(sQ) + x * Cfg::QT_BYTES, 16, 1024);
      const SmemDesc kd0 = make_desc_sw128(smem_u32(sK), 16, 1024);
      const SmemDesc vd0 = make_desc_sw128(smem_u32(sV), Cfg::HALF_KV, 1024);
      uint32_t g0 = 0, n_pv = 0;   // key tiles of earlier items; PV chains issued
      unsigned long long pairs = 0;
      for (uint32_t n = 0; !aborted(B); ++n) {
        if (!attn_wait(B, &B->item_full[n & 1], (n >> 1) & 1, ns, SITE_ATTN_MMA)) break;
        const AttnItem it = B->item[n & 1];
        mbar_arrive(&B->item_empty[n & 1]);
        if (it.h < 0) break;
        const int ntk = it.packed >> 9;
        if (x == 1 && (it.packed & 0x1FF) <= Cfg::BM) {   // no tile B in this item
          g0 += ntk;
          continue;
        }
        if (!attn_wait(B, &B->q_full, n & 1, ns, SITE_ATTN_MMA)) break;
        bool ok = true;
        for (int t = 0; t < ntk && ok; ++t) {
          const uint32_t gt = g0 + t;
          const int slot = static_cast<int>(gt % Cfg::KST);
          const uint32_t ph = (gt / Cfg::KST) & 1;
          const uint32_t slot_off = (slot * Cfg::KV_BYTES) >> 4;
          if (!attn_wait(B, &B->k_full[slot], ph, ns, SITE_ATTN_MMA)) { ok = false; break; }
          tc_fence_after();
          mma_chain<D / 16, Cfg::HALF_Q, 32, Cfg::HALF_KV, 32>(
              tmem + Cfg::tm_s(x), qd, SmemDesc{kd0.lo + slot_off, kd0.hi}, Cfg::IDESC_S, 0u);
          mma_commit(&B->s_full[x]);
          mma_commit(&B->k_empty[x][slot]);
          if (t == ntk - 1) mma_commit(&B->q_empty[x]);   // the item's last S: Q may be replaced
          if (!attn_wait(B, &B->p_full[x], n_pv & 1, ns, SITE_ATTN_MMA) ||
              !attn_wait(B, &B->v_full[slot], ph, ns, SITE_ATTN_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // A = P_x [128 q x 128 keys] in TMEM (the first 64 columns of S_x);
          // B = V [128 keys x D], MN-major, 16 keys = 2048 bytes per K-step
          mma_chain_ts<Cfg::BN / 16, 4 * 2048, 2048>(tmem + Cfg::tm_o(x), tmem + Cfg::tm_s(x),
                                                     SmemDesc{vd0.lo + slot_off, vd0.hi}, Cfg::IDESC_PV,
                                                     t > 0 ? 1u : 0u);
          if (t == ntk - 1) mma_commit(&B->o_full[x]);   // the item's O of tile x is final
          mma_commit(&B->v_empty[x][slot]);
          ++n_pv;
          ++pairs;
        }
        if (!ok) break;
        g0 += ntk;
      }
      if (P.issued != nullptr && pairs > 0) atomicAdd(P.issued, pairs);
      // make sure every issued MMA has retired before TMEM is released
      mma_commit(&B->drain[x]);
      mbar_wait(&B->drain[x], 0, 1000000000ull);
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
    const uint32_t s_addr = tmem + lane_off + Cfg::tm_s(x);
    const float sl2 = P.scale_log2;
    uint32_t g = 0, n_s = 0, n_o = 0;
    // Exponentials take turns between the two tiles of an item (A(t), B(t),
    // A(t+1), ...), so one tile's exponentials overlap the other tile's MMAs
    // instead of competing for the same MUFU units.  exp_done[y] completes
    // once per step of tile y; other_before counts the other tile's steps in
    // earlier items (tile A runs every item, tile B only items of > 128 rows).
    // Neither tile can get two completions ahead of the other's wait: tile B
    // waits for A(t) before finishing B(t), A waits for B(t-1) before A(t),
    // and an item's first S is issued only after both tiles' last PV.
    uint32_t other_before = 0;
    for (uint32_t n = 0; !warp_aborted(B); ++n) {
      if (!attn_warp_wait(B, &B->item_full[n & 1], (n >> 1) & 1, ns, SITE_ATTN_SOFTMAX)) break;
      const AttnItem it = B->item[n & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(&B->item_empty[n & 1]);
      if (it.h < 0) break;                  // end of the list
      const int ntk = it.packed >> 9;
      const int rows_total = it.packed & 0x1FF;
      const int nrows = x == 0 ? min(rows_total, Cfg::BM) : rows_total - Cfg::BM;
      const bool pair = rows_total > Cfg::BM;   // both tiles present: take turns
      if (nrows <= 0) {          // this item has no tile B
        g += ntk;
        other_before += ntk;     // tile A's steps of this item
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
        tmem_ld128_sync(s_addr, sv);
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
        // wait for the turn: tile A's step t after tile B's step t-1, tile B's
        // step t after tile A's step t
        if (pair && (x == 1 || t > 0)) {
          const uint32_t want = other_before + t - (x == 0 ? 1 : 0);   // index of the other's step
          if (!attn_warp_wait(B, &B->exp_done[x ^ 1], want & 1, ns, SITE_ATTN_SOFTMAX)) {
            ok = false;
            break;
          }
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
          float2 p2;
          if ((e >> 1) % 64 < SVG_EXP_POLY_PAIRS)   // a share of the pairs on the FMA pipe
            p2 = exp2_poly_x2(a2);
          else
            p2 = make_float2(ex2_approx(a2.x), ex2_approx(a2.y));
          rs2 = add_f32x2(rs2, p2);
          packed[e >> 1] = SVG_PACK_INT ? pack_bf16x2_int(p2.x, p2.y) : pack_bf16x2(p2.x, p2.y);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&B->exp_done[x]);
        // S_x(t) completing implies PV_x(t-1) completed (MMAs run in issue
        // order), so O_x is stable here
        if (t >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {   // rescale O rows in TMEM
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float ov[32];
            tmem_ld32_sync(o_addr + c * 32, ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] *= alpha;
            tmem_st32(o_addr + c * 32, ov);
          }
        }
        l = l * alpha + (rs2.x + rs2.y);
        // P row: 128 keys as 64 bf16 pairs over the first 64 columns of S_x
        tmem_st64(s_addr, packed);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B->p_full[x]);
      }
      if (!ok) break;
      if (x == 1 || pair) other_before += ntk;   // the other tile's steps of this item
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

// Single block: one AttnItem per 256 query rows, in claiming order (a
// counting sort over kAttnBuckets buckets of the estimated cost = key tiles x
// query tiles).  Long items (cost >= kAttnBigCost: q-clusters whose centroid
// scores are flat select most of the keys) come first, longest first across
// all heads, so none of them starts late and sets the tail; the rest follow
// by head group (a few heads, whose K/V stay in L2 while their items run),
// longest first inside a group.  The attention kernel's CTAs claim items in
// this order from a shared counter (greedy list scheduling), so an SM that
// drew short items takes more of them.  Also resets that counter.
constexpr int kAttnBuckets = 1024;
constexpr int kAttnBigCost = 32;
constexpr int kAttnBigBuckets = 256;                       // costs 32 .. 287 and above
constexpr int kAttnGroups = 16;                            // head groups of the short items
constexpr int kAttnCostBuckets = (kAttnBuckets - kAttnBigBuckets) / kAttnGroups;   // 48 > kAttnBigCost

__device__ __forceinline__ int attn_item_bucket(int h, int heads_per_group, int kt, int rows) {
  const int cost = kt * (rows > 128 ? 2 : 1);
  if (cost >= kAttnBigCost)
    return kAttnBigBuckets - 1 - min(cost - kAttnBigCost, kAttnBigBuckets - 1);
  const int grp = min(h / heads_per_group, kAttnGroups - 1);
  return kAttnBigBuckets + grp * kAttnCostBuckets + kAttnCostBuckets - 1 - cost;
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
