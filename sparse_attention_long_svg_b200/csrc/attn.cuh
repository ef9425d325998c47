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
//              sequence S(0), S(1), PV(0), S(2), PV(1), ... with S_x = Q_x K^T
//              and O_x += P V (operands in shared memory)
//   warp 10    item loader: claims the next item from a counter shared by all
//              CTAs (list sorted by head group, then longest first), prefetches
//              its query rows into L2, merges its key ranges into runs
// Tensor memory per query tile x: S_x (128 fp32 columns) and O_x (D
// columns).  The softmax copies S_x(t) to registers and releases it at once,
// so S_x(t+1) runs on the tensor cores while the softmax of step t computes.
// The two query tiles take turns on their exponentials (the MUFU-bound part),
// so one tile's exponentials overlap the other tile's MMAs; the turns also
// let both tiles share one P buffer in shared memory (bf16, 128-byte
// swizzled, K-major): P_x(t) is written once the previous PV (the other
// tile's) has read it.  With 8-bit Q and K (E4M3 Q K^T, kind::f8f6f4) the
// smaller Q/K tiles leave room for one P buffer per query tile, and P_x(t)
// waits only for PV_x(t-1).  O accumulates in TMEM across the item's key tiles;
// the softmax warps rescale it in place only when a row's running max grows
// by more than 2^8 (exact: every probability is taken against the same
// reference max that O and the row sum use).  The merged key ranges of the
// CTA's next two items live in two global scratch slots of the workspace,
// one per header slot.
#pragma once
#include "common.cuh"

namespace svg {

constexpr int kItemRows = 256;     // query rows per work item (two 128-row tiles)
constexpr int kSlotsPerTile = 16;  // 8-row slots per 128-key tile
constexpr int kMetaRing = 8;       // key-validity masks in flight

struct AttnItem {  // up to 256 consecutive query rows; h < 0 ends the list
  // i = the q-cluster whose block list the rows use (the rows may span a group
  // of consecutive q-clusters with identical block lists)
  int32_t h, i, q0, packed;  // packed = rows (<= 256) | key_tiles << 9
};

// Readers of an item header slot that must release it before it is refilled:
// the producer, the two MMA issuers and the eight softmax warps.
constexpr int kItemReaders = 11;

// Instruction descriptor for kind::f8f6f4 with E4M3 A/B (format code 0 in
// both operand fields), fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                   // D format: f32
         | (0u << 7) | (0u << 10)                    // A, B format: E4M3
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((static_cast<uint32_t>(N) >> 3) << 17) | ((static_cast<uint32_t>(M) >> 4) << 24);
}

// D[tmem] (+)= A * B^T with 8-bit operands (kind::f8f6f4): one MMA covers 32
// elements (32 bytes) of K.  Descriptors as halves plus 16-byte offsets.
__device__ __forceinline__ void mma_f8_ss_off(uint32_t d_tmem, SmemDesc a, uint32_t a_off, SmemDesc b,
                                              uint32_t b_off, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 ad, bd;\n\t"
      "mov.b64 ad, {%1, %2};\n\tmov.b64 bd, {%3, %4};\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], ad, bd, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a.lo + a_off), "r"(a.hi), "r"(b.lo + b_off), "r"(b.hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The 8-bit counterpart of mma_chain: STEPS MMAs of 32 bytes of K each, K-step
// k at byte offset k * 32 of a 128-byte swizzle row (STEPS <= 4).
template <int STEPS, uint32_t A_K, uint32_t B_K>
__device__ __forceinline__ void mma_chain_f8(uint32_t d_tmem, SmemDesc a, SmemDesc b, uint32_t idesc,
                                             uint32_t accumulate_first) {
  static_assert(STEPS <= 4, "one 128-byte block of K");
#pragma unroll
  for (int k = 0; k < STEPS; ++k)
    mma_f8_ss_off(d_tmem, a, (k * A_K) >> 4, b, (k * B_K) >> 4, idesc, k > 0 ? 1u : accumulate_first);
}

// FP8: Q and K are E4M3 (one byte per channel, a 128-channel row is one
// 128-byte swizzle row) and S = Q K^T runs as kind::f8f6f4 MMAs; P and V stay
// bf16.  Supported at D = 128.
template <int D, bool FP8 = false>
struct AttnCfg {
  static constexpr int BM = 128, BN = 128, SLOT = 8, NSLOT = BN / SLOT;
  static constexpr int HEAD_DIM = D;
  static constexpr int QE = FP8 ? 1 : 2;              // bytes per Q/K element
  static constexpr int QK_BLOCK = 128 / QE;           // Q/K channels per 128-byte block
  static constexpr int DHQ = D * QE / 128;            // 128-byte blocks of a Q/K row
  static constexpr int DH = D / 64;                   // 128-byte (64-channel) blocks of a V row
  static constexpr int KST = D == 128 ? 2 : 4;        // K ring slots (same for V)
  static constexpr int QT_BYTES = BM * D * QE;        // one Q tile
  static constexpr int K_BYTES = BN * D * QE;         // one K tile
  static constexpr int V_BYTES = BN * D * 2;          // one V tile
  static constexpr int HALF_Q = BM * 128;             // one 128-byte column block of a Q tile
  static constexpr int HALF_K = BN * 128;             // same for a K tile
  static constexpr int HALF_V = BN * 128;             // same for a V tile
  static constexpr int P_BYTES = BM * BN * 2;         // one P tile
  static constexpr int HALF_P = BM * 128;             // one 64-key half of it
  // P buffers: one shared by both query tiles, or (FP8, whose 8-bit Q and K
  // tiles leave the room) one per query tile
  static constexpr int NP = FP8 ? 2 : 1;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = OFF_Q + 2 * QT_BYTES;
  static constexpr int OFF_K = OFF_P + NP * P_BYTES;
  static constexpr int OFF_V = OFF_K + KST * K_BYTES;
  static constexpr int MAX_SEL = 1024;                // selected k-clusters per q-cluster
  static constexpr int OFF_BAR = OFF_V + KST * V_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 1024 + 1024;  // barriers/meta + alignment slack
  // TMEM: S of tile x at x*128 (128 columns); O of tile x at 256 + x*128
  static constexpr uint32_t TM_COLS = 512;
  static constexpr uint32_t IDESC_S =
      FP8 ? idesc_e4m3_f32(BM, BN, false, false) : idesc_bf16_f32(BM, BN, false, false);
  static constexpr int S_STEPS = D * QE / 32;         // MMAs of one S chain (32 bytes of K each)
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, false, true);
  static_assert(!FP8 || D == 128, "8-bit Q/K tiles need 128-byte rows");
  // warp 9 issues tile A's MMAs (and owns TMEM), warp 11 tile B's
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, LOADER_WARP = 10, MMA_B_WARP = 11;
  static constexpr int THREADS = 12 * 32;
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  __device__ static constexpr uint32_t tm_s(int x) { return x * 128; }
  __device__ static constexpr uint32_t tm_o(int x) { return 256 + x * 128; }
};

// TMA boxes of 8, 16, 32, 64 and 128 rows (one tensor map each for K and V).
constexpr int kNumBoxSizes = 5;

// Box mode (K and V already permuted): k[b], v[b] have boxes of 8 << b rows.
// Gather mode (K and V in token order, rows fetched through the K
// permutation with 16-byte asynchronous copies): k and v are unused.
struct AttnMaps {
  CUtensorMap q;
  CUtensorMap k[kNumBoxSizes];
  CUtensorMap v[kNumBoxSizes];
};

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
  uint64_t q_full[2], q_empty[2];                   // [tile]
  uint64_t k_full[4], v_full[4];
  uint64_t k_empty[2][4], v_empty[2][4];            // [tile][slot]: released by that tile's MMAs
  uint64_t meta_full[kMetaRing];
  uint64_t s_full[2], s_free[2], p_full[2], o_full[2];   // [tile]
  uint64_t p_free[2];                         // [tile]: a PV of that tile (reading P) has completed
  uint64_t item_full[2], item_empty[2];
  uint64_t drain[2];
  AttnItem item[2];      // item header ring written by the loader warp
  int32_t ranges_cnt[2]; // merged runs of the item in header slot [b]
  uint32_t meta[kMetaRing][4];   // per key tile: 128-bit key validity mask
  uint32_t exp_steps[2]; // [tile]: 4 x the steps whose exponentials that tile has finished (one add per warp)
  uint32_t v_seen;       // two P buffers: V tiles whose landing tile A's MMA issuer has seen (all tiles, in order)
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
  const int32_t *perm_k; // gather mode: permuted key row r of a head is row perm_k[r] of K and V
  const __nv_bfloat16 *kg, *vg;   // gather mode: K and V [BH, N, D] in token order
  const float *q_scale;  // FP8: per permuted query row [BH, N]; the logits carry q_scale * k_scale
  const float *k_scale;  // FP8: per head [BH]
  unsigned long long *issued;   // optional: += (query tile, key tile) pairs issued
  int2 *ranges;          // per CTA: 2 x MAX_SEL merged key runs (first row, rows), one slot per header slot
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

// Warp-wide wait until a shared-memory progress counter reaches `target`
// (wrap-safe comparison); lane 0 polls, bounded like the barrier waits.
__device__ __forceinline__ bool attn_warp_wait_count(AttnBarriers *b, const uint32_t *ctr, uint32_t target,
                                                     uint64_t ns, uint32_t site) {
  int ok = 1;
  if (lane_id() == 0) {
    const volatile uint32_t *c = ctr;
    if (static_cast<int32_t>(*c - target) < 0) {
      const long long t0 = clock64();
      const long long limit = static_cast<long long>(ns) * 2;
      while (static_cast<int32_t>(*c - target) < 0) {
        if (clock64() - t0 > limit) {
          ok = 0;
          record_error(SVG_ERR_TIMEOUT, site);
          atomicExch(&b->abort_flag, 1);
          break;
        }
      }
    }
  }
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// One thread waits until a shared-memory progress counter reaches `target`
// (wrap-safe comparison), bounded like the barrier waits.
__device__ __forceinline__ bool attn_wait_count(AttnBarriers *b, const uint32_t *ctr, uint32_t target, uint64_t ns,
                                                uint32_t site) {
  const volatile uint32_t *c = ctr;
  if (static_cast<int32_t>(*c - target) >= 0) return true;
  const long long t0 = clock64();
  const long long limit = static_cast<long long>(ns) * 2;
  while (static_cast<int32_t>(*c - target) < 0) {
    if (clock64() - t0 > limit) {
      record_error(SVG_ERR_TIMEOUT, site);
      atomicExch(&b->abort_flag, 1);
      return false;
    }
  }
  return true;
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

// Gather mode: one 128-row key tile (K or V) into a ring slot, in the same
// 128-byte-swizzled K-major layout the tensor-map loads produce (row r,
// 16-byte chunk c of 64-channel half h at h * HALF_V + 128 r + 16 (c ^ r % 8)).
// Lane l holds the global rows of tile rows 4 l .. 4 l + 3 in `rows`; each
// warp instruction copies D / 8 consecutive 16-byte chunks of 32 / (D / 8)
// rows (coalesced), the rows taken from their owners by shuffles.
template <class Cfg>
__device__ __forceinline__ void gather_rows(uint32_t slot_addr, const __nv_bfloat16 *__restrict__ src, int4 rows,
                                            int lane) {
  constexpr int LPR = Cfg::HEAD_DIM / 8;   // lanes (16-byte chunks) per row
  constexpr int RPI = 32 / LPR;        // rows per instruction
  const int sub = lane / LPR, c = lane % LPR;
  const uint32_t half_off = static_cast<uint32_t>((c >> 3) * Cfg::HALF_V);
  const int cc = c & 7;
#pragma unroll
  for (int i = 0; i < Cfg::BN / RPI; ++i) {
    const int r0 = i * RPI;            // tile rows r0 .. r0 + RPI - 1 (one owner lane per 4 rows)
    int v[RPI];
#pragma unroll
    for (int k = 0; k < RPI; ++k) {
      const int r = r0 + k;
      const int comp = r & 3;
      v[k] = __shfl_sync(0xffffffffu, comp == 0 ? rows.x : comp == 1 ? rows.y : comp == 2 ? rows.z : rows.w, r >> 2);
    }
    int g = v[0];
#pragma unroll
    for (int k = 1; k < RPI; ++k)
      if (sub == k) g = v[k];
    const int r = r0 + sub;
    const uint32_t dst = slot_addr + half_off + static_cast<uint32_t>(r * 128) +
                         (static_cast<uint32_t>(cc ^ (r & 7)) << 4);
    cp_async_16(dst, src + static_cast<size_t>(g) * Cfg::HEAD_DIM + c * 8);
  }
}

template <int D, bool GATHER, bool FP8 = false>
__global__ void __launch_bounds__(AttnCfg<D, FP8>::THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnParams P) {
  using Cfg = AttnCfg<D, FP8>;
  static_assert(!(GATHER && FP8), "gather mode copies bf16 rows");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem + Cfg::OFF_Q;
  uint8_t *sP = smem + Cfg::OFF_P;
  uint8_t *sK = smem + Cfg::OFF_K;
  uint8_t *sV = smem + Cfg::OFF_V;
  int2 *gRanges = P.ranges + static_cast<size_t>(blockIdx.x) * 2 * Cfg::MAX_SEL;
  AttnBarriers *B = reinterpret_cast<AttnBarriers *>(smem + Cfg::OFF_BAR);
  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());

  if (threadIdx.x == 0) {
    for (int s = 0; s < 4; ++s) {
      mbar_init(&B->k_full[s], GATHER ? 32 : 1);   // gather mode: one arrival per producer lane
      mbar_init(&B->v_full[s], GATHER ? 32 : 1);
      for (int x = 0; x < 2; ++x) {
        mbar_init(&B->k_empty[x][s], 1);
        mbar_init(&B->v_empty[x][s], 1);
      }
    }
    for (int s = 0; s < kMetaRing; ++s) mbar_init(&B->meta_full[s], 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&B->s_full[x], 1);
      mbar_init(&B->s_free[x], 4);
      mbar_init(&B->p_full[x], 4);
      mbar_init(&B->q_full[x], 1);
      B->exp_steps[x] = 0;
      B->v_seen = 0;
      mbar_init(&B->o_full[x], 1);
      mbar_init(&B->item_full[x], 1);
      mbar_init(&B->item_empty[x], kItemReaders);
      mbar_init(&B->q_empty[x], 1);
      mbar_init(&B->drain[x], 1);
    }
    mbar_init(&B->p_free[0], 1);
    mbar_init(&B->p_free[1], 1);
    B->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == Cfg::MMA_WARP) {
    tmem_alloc(&B->tmem_base, Cfg::TM_COLS);
    tmem_relinquish();
  }
  if (warp == Cfg::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&maps.q);
    for (int b = 0; b < (GATHER ? 0 : kNumBoxSizes); ++b) {
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
    // marker (h = -1).  The key ranges of item n go to the range slot of its
    // header slot n & 1, free once every reader has released item n - 2 (the
    // producer releases it after its last key tile).
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
      if (lane < 2 * Cfg::DHQ && (lane / Cfg::DHQ) * Cfg::BM < (it.packed & 0x1FF))   // query rows -> L2
        tma_prefetch_l2_2d(&maps.q, (lane % Cfg::DHQ) * Cfg::QK_BLOCK,
                           it.h * P.N + it.q0 + (lane / Cfg::DHQ) * Cfg::BM);
      const size_t row = static_cast<size_t>(it.h) * P.Cq + it.i;
      const int cnt = attn_sel_count(P.sel_count, row, max_sel);
      const int32_t *cols = P.sel_cols + row * P.Ck;
      const int32_t *koff = P.k_off + static_cast<size_t>(it.h) * (P.Ck + 1);
      // Merge touching ranges into runs (same rule as the planning kernel),
      // 32 selected clusters at a time, one per lane: a non-empty range opens
      // a run unless it starts where the previous non-empty range (in
      // selection order) ended.  The open run is carried between chunks.
      int2 *rng = gRanges + buf * Cfg::MAX_SEL;
      int m = 0, open_x = 0, open_end = -1;   // runs opened so far; the open run
      for (int c0 = 0; c0 < cnt; c0 += 32) {
        const int c = c0 + lane;
        int x = 0, len = 0;   // out-of-range ids are flagged by the planning kernel
        if (c < cnt) {
          const int j = cols[c];
          if (j >= 0 && j < P.Ck) {
            x = koff[j];
            len = koff[j + 1] - x;
          }
        }
        const bool valid = len > 0;
        const int end = x + len;
        const unsigned below_mask = (1u << lane) - 1u;
        const unsigned vmask = __ballot_sync(0xffffffffu, valid);
        const unsigned vb = vmask & below_mask;
        const int pv = vb ? 31 - __clz(vb) : 0;
        const int pv_end = __shfl_sync(0xffffffffu, end, pv);
        const int prev_end = vb ? pv_end : open_end;   // end of the previous non-empty range
        const bool opens = valid && x != prev_end;
        const unsigned smask = __ballot_sync(0xffffffffu, opens);
        const unsigned sb = smask & below_mask;
        const int ps = sb ? 31 - __clz(sb) : 0;
        const int ps_x = __shfl_sync(0xffffffffu, x, ps);
        if (opens) {   // close the previous run: it ends at prev_end
          const int idx = m + __popc(sb);
          const int run_x = sb ? ps_x : open_x;
          if (idx > 0) rng[idx - 1] = make_int2(run_x, prev_end - run_x);
        }
        if (smask) open_x = __shfl_sync(0xffffffffu, x, 31 - __clz(smask));
        if (vmask) open_end = __shfl_sync(0xffffffffu, end, 31 - __clz(vmask));
        m += __popc(smask);
      }
      if (lane == 0) {
        if (m > 0) rng[m - 1] = make_int2(open_x, open_end - open_x);
        __threadfence_block();
        B->ranges_cnt[buf] = m;
        B->item[buf] = it;
        __threadfence_block();
        mbar_arrive(&B->item_full[buf]);
      }
      __syncwarp();
    }
  } else if (warp == Cfg::PRODUCER_WARP) {
    // ------------------------------------------------------------ TMA producer
    // Two streams, issued by one thread that polls both: the K side takes the
    // items in order (Q tiles, then K(t) of every key tile t, cutting each
    // tile into boxes), the V side issues V(t) from the same box list.  Each
    // load is issued as soon as its ring slot is free: K(t + KST) once both
    // present query tiles' S(t) are done, V(t + KST) once their PV(t) are, so
    // a slot held by the slower tile never holds up the other ring.  Box
    // lists of key tiles whose V is not yet issued stay in a small ring.
    // A slot (and Q) is reused once every query tile of its last occupant has
    // released it: tile A is in every item, tile B only in items of > 128
    // rows; slot_b[r][s] = whether slot s of ring r (0 = K, 1 = V) last held a
    // tile with tile B, rel_b[r][s] / nq_b = tile-B releases expected so far.
    // The whole warp runs the loop with identical control flow (barrier tests
    // are made by lane 0 and broadcast); lane 0 issues the arrivals and the
    // Q copies, lane b the copies of box b of a key tile.  Key ranges are
    // read 32 at a time into a register window; every other piece of state
    // is in registers (no local memory).
    constexpr int kBoxRing = Cfg::KST + 2;   // box lists of tiles whose V is not yet issued
    auto test = [&](uint64_t *bar, uint32_t parity) {
      return __shfl_sync(0xffffffffu, lane == 0 ? (mbar_test(bar, parity) ? 1 : 0) : 0, 0) != 0;
    };
    int2 win = make_int2(0, 0);
    int win_base = -1;
    const int2 *rng = gRanges;
    {
      // bit 4r + s: slot s of ring r last held a tile with tile B / parity of
      // the tile-B releases of that slot expected so far
      uint32_t slot_b = 0, rel_b = 0, nq_b = 0;
      uint32_t tile_b = 0;               // bit e: box-ring entry e has tile B
      // box mode: this lane's box of each entry (row, kind | slot << 8; -1: none);
      // gather mode: this lane's four key rows of each entry (rows 4 lane .. +3 of the tile)
      int box_row[kBoxRing], box_code[kBoxRing];
      int4 grow[GATHER ? kBoxRing : 1];
#pragma unroll
      for (int e = 0; e < kBoxRing; ++e) box_row[e] = box_code[e] = -1;
#pragma unroll
      for (int e = 0; e < (GATHER ? kBoxRing : 1); ++e) grow[e] = make_int4(0, 0, 0, 0);
      const int32_t *perm_k = P.perm_k;
      bool pre = false;                  // gather mode: the next key tile's rows are looked up
      uint32_t pre_mask[4] = {0, 0, 0, 0};
      int4 pre_src = make_int4(0, 0, 0, 0);
      uint32_t gk = 0, gv = 0, nq = 0, nq1 = 0;   // K and V tiles issued, Q loads issued (all, tile B)
      int n = 0;                         // next item (header slot n & 1)
      bool k_active = false, k_done = false, prev_b = false;
      AttnItem it{};
      int ntk = 0, tk = 0, cnt = 0, ci = 0, cur = 0, left = 0;
      bool has_b = false;
      const long long limit = static_cast<long long>(ns) * 2;
      long long t_last = clock64();
      while (!(k_done && gv == gk)) {
        bool progress = false;
        // ---- K side: start the next item
        if (!k_active && !k_done && test(&B->item_full[n & 1], (n >> 1) & 1)) {
          it = B->item[n & 1];
          if (it.h < 0) {                   // end of the list
            if (lane == 0) mbar_arrive(&B->item_empty[n & 1]);
            k_done = true;
            progress = true;
          } else if ((n == 0 || (test(&B->q_empty[0], (n - 1) & 1) &&
                                 (!prev_b || test(&B->q_empty[1], (nq_b - 1) & 1))))) {
            cnt = B->ranges_cnt[n & 1];
            rng = gRanges + (n & 1) * Cfg::MAX_SEL;
            ntk = it.packed >> 9;
            has_b = (it.packed & 0x1FF) > Cfg::BM;
            prev_b = has_b;
            if (has_b) ++nq_b;
            if (P.fault != 1 && lane == 0) {
              const int qrow = it.h * P.N + it.q0;
#pragma unroll
              for (int x = 0; x < 2; ++x) {
                if (x == 1 && !has_b) break;
                mbar_arrive_expect_tx(&B->q_full[x], Cfg::QT_BYTES);
#pragma unroll
                for (int dh = 0; dh < Cfg::DHQ; ++dh)
                  tma_load_2d(sQ + x * Cfg::QT_BYTES + dh * Cfg::HALF_Q, &maps.q, dh * Cfg::QK_BLOCK,
                              qrow + x * Cfg::BM, &B->q_full[x]);
              }
            }
            if (P.fault != 1) {
              ++nq;
              if (has_b) ++nq1;
            }
            tk = 0;
            win_base = -1;
            ci = cur = left = 0;
            k_active = true;
            progress = true;
          }
        }
        // ---- K side: the next key tile of the item
        if constexpr (GATHER) {
          // gather mode: the next key tile's rows are looked up (the loads of
          // its K-permutation entries issued) as soon as it may be built, so
          // they are in registers by the time its slot frees
          if (k_active && !pre && gk - gv < static_cast<uint32_t>(kBoxRing)) {
            pre_mask[0] = pre_mask[1] = pre_mask[2] = pre_mask[3] = 0;
            int my_p0 = 0, my_nv = 0;    // first permuted row and valid rows of this lane's slot
            for (int sl = 0; sl < Cfg::NSLOT; ++sl) {
              while (left <= 0 && ci < cnt) {
                if ((ci & ~31) != win_base) {   // refill the window: ranges [ci & ~31, +32)
                  win_base = ci & ~31;
                  win = win_base + lane < cnt ? __ldcg(rng + win_base + lane) : make_int2(0, 0);
                }
                cur = __shfl_sync(0xffffffffu, win.x, ci & 31);
                left = __shfl_sync(0xffffffffu, win.y, ci & 31);
                ++ci;
              }
              const int nv = left > 0 ? min(left, Cfg::SLOT) : 0;
              if ((lane >> 1) == sl) {   // padding slots re-read row 0; they are masked
                my_p0 = nv > 0 ? cur : 0;
                my_nv = nv;
              }
              if (nv > 0) {
                set_bits(pre_mask, sl * Cfg::SLOT, nv);
                cur += Cfg::SLOT;
                left -= Cfg::SLOT;
              }
            }
            const int32_t *pk = perm_k + static_cast<size_t>(it.h) * P.N;
            const int o = 4 * (lane & 1);
            pre_src.x = __ldg(pk + my_p0 + (o < my_nv ? o : 0));
            pre_src.y = __ldg(pk + my_p0 + (o + 1 < my_nv ? o + 1 : 0));
            pre_src.z = __ldg(pk + my_p0 + (o + 2 < my_nv ? o + 2 : 0));
            pre_src.w = __ldg(pk + my_p0 + (o + 3 < my_nv ? o + 3 : 0));
            pre = true;
          }
        }
        if (k_active && (!GATHER || pre) && gk - gv < static_cast<uint32_t>(kBoxRing)) {
          const int slot = static_cast<int>(gk % Cfg::KST);
          const uint32_t sbit = 1u << slot;
          const bool free_slot =
              gk < static_cast<uint32_t>(Cfg::KST) ||
              (test(&B->k_empty[0][slot], ((gk / Cfg::KST) - 1) & 1) &&
               (!(slot_b & sbit) || test(&B->k_empty[1][slot], (rel_b & sbit) ? 0u : 1u)));
          if (free_slot) {
            if constexpr (GATHER) {
              const int rb = static_cast<int>(gk % kBoxRing);
              const int src[4] = {pre_src.x, pre_src.y, pre_src.z, pre_src.w};
              int rr[4];
              bool bad = false;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const bool out = src[i] < 0 || src[i] >= P.N;
                bad |= out;
                rr[i] = it.h * P.N + (out ? 0 : src[i]);
              }
              if (bad) record_error(SVG_ERR_DEVICE_CHECK, SITE_ATTN_PRODUCER);
              pre = false;
              const int4 r4 = make_int4(rr[0], rr[1], rr[2], rr[3]);
#pragma unroll
              for (int e = 0; e < kBoxRing; ++e)
                if (e == rb) grow[e] = r4;
              tile_b = has_b ? (tile_b | (1u << rb)) : (tile_b & ~(1u << rb));
              const int mi = static_cast<int>(gk % kMetaRing);
              slot_b = has_b ? (slot_b | sbit) : (slot_b & ~sbit);
              if (has_b) rel_b ^= sbit;
              if (lane == 0) {
#pragma unroll
                for (int w = 0; w < 4; ++w) B->meta[mi][w] = pre_mask[w];
                mbar_arrive(&B->meta_full[mi]);
              }
              gather_rows<Cfg>(smem_u32(sK + slot * Cfg::K_BYTES), P.kg, r4, lane);
              cp_async_arrive(&B->k_full[slot]);
            } else {
              // cut the tile into boxes of 1..16 slots (8..128 rows): the largest
              // power of two that fits both the tile and the rest of the run
              const int rb = static_cast<int>(gk % kBoxRing);
              const int pad_row = it.h * P.N;  // unused slots re-read a valid row; they are masked
              uint32_t mask[4] = {0, 0, 0, 0};
              int sl = 0, nb = 0, my_row = -1, my_code = -1;
              while (sl < Cfg::NSLOT) {
                while (left <= 0 && ci < cnt) {
                  if ((ci & ~31) != win_base) {   // refill the window: ranges [ci & ~31, +32)
                    win_base = ci & ~31;
                    win = win_base + lane < cnt ? __ldcg(rng + win_base + lane) : make_int2(0, 0);
                  }
                  cur = __shfl_sync(0xffffffffu, win.x, ci & 31);
                  left = __shfl_sync(0xffffffffu, win.y, ci & 31);
                  ++ci;
                }
                const int space = Cfg::NSLOT - sl;
                const int need = left > 0 ? (left + Cfg::SLOT - 1) / Cfg::SLOT : space;
                int kind = 0;
                while (kind + 1 < kNumBoxSizes && (2 << kind) <= space && (2 << kind) <= need) ++kind;
                const int nsl = 1 << kind;
                if (lane == nb) {
                  my_row = left > 0 ? it.h * P.N + cur : pad_row;
                  my_code = kind | (sl << 8);
                }
                if (left > 0) {
                  set_bits(mask, sl * Cfg::SLOT, min(left, nsl * Cfg::SLOT));
                  cur += nsl * Cfg::SLOT;
                  left -= nsl * Cfg::SLOT;
                }
                ++nb;
                sl += nsl;
              }
  #pragma unroll
              for (int e = 0; e < kBoxRing; ++e) {
                if (e == rb) {
                  box_row[e] = my_row;
                  box_code[e] = my_code;
                }
              }
              tile_b = has_b ? (tile_b | (1u << rb)) : (tile_b & ~(1u << rb));
              const int mi = static_cast<int>(gk % kMetaRing);
              slot_b = has_b ? (slot_b | sbit) : (slot_b & ~sbit);
              if (has_b) rel_b ^= sbit;
              if (lane == 0) {
  #pragma unroll
                for (int w = 0; w < 4; ++w) B->meta[mi][w] = mask[w];
                mbar_arrive(&B->meta_full[mi]);
                mbar_arrive_expect_tx(&B->k_full[slot], Cfg::K_BYTES);
              }
              __syncwarp();
              if (my_code >= 0) {
                const int kind = my_code & 0xFF, at = my_code >> 8;
  #pragma unroll
                for (int dh = 0; dh < Cfg::DHQ; ++dh)
                  tma_load_2d(sK + slot * Cfg::K_BYTES + dh * Cfg::HALF_K + at * 1024, &maps.k[kind],
                              dh * Cfg::QK_BLOCK, my_row, &B->k_full[slot]);
              }
            }
            ++gk;
            progress = true;
            if (++tk == ntk) {             // the item's ranges and header are no longer read
              if (lane == 0) {
                mbar_arrive(&B->item_empty[n & 1]);
              }
              ++n;
              k_active = false;
            }
          }
        }
        // ---- V side
        if (gv < gk) {
          const int slot = static_cast<int>(gv % Cfg::KST);
          const uint32_t sbit = 1u << (4 + slot);
          const bool free_slot =
              gv < static_cast<uint32_t>(Cfg::KST) ||
              (test(&B->v_empty[0][slot], ((gv / Cfg::KST) - 1) & 1) &&
               (!(slot_b & sbit) || test(&B->v_empty[1][slot], (rel_b & sbit) ? 0u : 1u)));
          if (free_slot) {
            const int rb = static_cast<int>(gv % kBoxRing);
            const bool tb = (tile_b >> rb) & 1u;
            slot_b = tb ? (slot_b | sbit) : (slot_b & ~sbit);
            if (tb) rel_b ^= sbit;
            if constexpr (GATHER) {
              int4 r4 = grow[0];
#pragma unroll
              for (int e = 1; e < kBoxRing; ++e)
                if (e == rb) r4 = grow[e];
              gather_rows<Cfg>(smem_u32(sV + slot * Cfg::V_BYTES), P.vg, r4, lane);
              cp_async_arrive(&B->v_full[slot]);
            } else {
              int my_row = -1, my_code = -1;
  #pragma unroll
              for (int e = 0; e < kBoxRing; ++e) {
                if (e == rb) {
                  my_row = box_row[e];
                  my_code = box_code[e];
                }
              }
              if (lane == 0) mbar_arrive_expect_tx(&B->v_full[slot], Cfg::V_BYTES);
              __syncwarp();
              if (my_code >= 0) {
                const int kind = my_code & 0xFF, at = my_code >> 8;
  #pragma unroll
                for (int dh = 0; dh < Cfg::DH; ++dh)
                  tma_load_2d(sV + slot * Cfg::V_BYTES + dh * Cfg::HALF_V + at * 1024, &maps.v[kind], dh * 64,
                              my_row, &B->v_full[slot]);
              }
            }
            ++gv;
            progress = true;
          }
        }
        if (progress) {
          t_last = clock64();
        } else if (__shfl_sync(0xffffffffu, clock64() - t_last > limit ? 1 : 0, 0)) {
          if (lane == 0) {
            record_error(SVG_ERR_TIMEOUT, SITE_ATTN_PRODUCER);
            atomicExch(&B->abort_flag, 1);
          }
          break;
        } else if (warp_aborted(B)) {
          break;
        }
      }
      // drain: every load issued above lands on a full barrier; wait for the
      // last phase of each so no copy is in flight when the CTA exits.
      if (lane == 0 && aborted(B)) {
        if (nq > 0) mbar_wait(&B->q_full[0], (nq - 1) & 1, 1000000000ull);
        if (nq1 > 0) mbar_wait(&B->q_full[1], (nq1 - 1) & 1, 1000000000ull);
        for (uint32_t k = (gk >= static_cast<uint32_t>(Cfg::KST) ? gk - Cfg::KST : 0); k < gk; ++k)
          mbar_wait(&B->k_full[k % Cfg::KST], (k / Cfg::KST) & 1, 1000000000ull);
        for (uint32_t k = (gv >= static_cast<uint32_t>(Cfg::KST) ? gv - Cfg::KST : 0); k < gv; ++k)
          mbar_wait(&B->v_full[k % Cfg::KST], (k / Cfg::KST) & 1, 1000000000ull);
      }
    }
  } else if (warp == Cfg::MMA_WARP || warp == Cfg::MMA_B_WARP) {
    // ------------------------------------------------------------ MMA issuers
    // One thread per query tile x issues that tile's chains for every item
    // that has the tile, in the order S(0), S(1), PV(0), S(2), PV(1), ...:
    // S_x(t) once K(t) (and Q) has landed and the softmax has read S_x(t-1)
    // out of TMEM; PV_x(t) once the softmax has written P_x(t) and V(t) has
    // landed.  It releases each K/V slot and Q for its own tile; the producer
    // reuses them when every present tile has released them.  With two
    // issuers one tile's chain queues on the tensor pipe while the other's
    // executes.  Tile B skips items without tile B, yet its parity waits on
    // the shared K/V slot barriers cannot pass on an older phase: its Q tile
    // of an item (own barrier, one phase per tile-B item) is loaded only
    // after tile A's last S of the previous item, so every earlier K tile has
    // landed, and its first P write of the item waits for tile A's first PV
    // of the item, so every earlier V tile has landed.
    const int x = warp == Cfg::MMA_WARP ? 0 : 1;
    if (lane == 0) {
      const SmemDesc qd = make_desc_sw128(smem_u32(sQ) + x * Cfg::QT_BYTES, 16, 1024);
      const SmemDesc pd = make_desc_sw128(smem_u32(sP) + (Cfg::NP == 2 ? x * Cfg::P_BYTES : 0), 16, 1024);
      const SmemDesc kd0 = make_desc_sw128(smem_u32(sK), 16, 1024);
      const SmemDesc vd0 = make_desc_sw128(smem_u32(sV), Cfg::HALF_V, 1024);
      uint32_t g0 = 0, n_s = 0, n_pv = 0, n_q = 0;   // key tiles of earlier items; S, PV chains issued; Q tiles used
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
        if (!attn_wait(B, &B->q_full[x], n_q & 1, ns, SITE_ATTN_MMA)) break;
        ++n_q;
        bool ok = true;
        // op 2t issues S(t + 1) (S(0) before the loop), op 2t + 1 issues PV(t)
        for (int op = -1; op < 2 * ntk && ok; ++op) {
          const bool is_s = op < 0 || (op & 1) == 0;
          const int t = op < 0 ? 0 : (is_s ? (op >> 1) + 1 : op >> 1);
          if (is_s && t >= ntk) continue;
          const uint32_t gt = g0 + t;
          const int slot = static_cast<int>(gt % Cfg::KST);
          const uint32_t ph = (gt / Cfg::KST) & 1;
          const uint32_t k_off = (slot * Cfg::K_BYTES) >> 4, v_off = (slot * Cfg::V_BYTES) >> 4;
          if (is_s) {
            if (!attn_wait(B, &B->k_full[slot], ph, ns, SITE_ATTN_MMA) ||
                (n_s > 0 && !attn_wait(B, &B->s_free[x], (n_s - 1) & 1, ns, SITE_ATTN_MMA))) {
              ok = false;
              break;
            }
            if constexpr (GATHER) fence_proxy_async_smem();   // cp.async writes -> tensor-core reads
            tc_fence_after();
            if constexpr (FP8)
              mma_chain_f8<Cfg::S_STEPS, 32, 32>(tmem + Cfg::tm_s(x), qd, SmemDesc{kd0.lo + k_off, kd0.hi},
                                                 Cfg::IDESC_S, 0u);
            else
              mma_chain<Cfg::S_STEPS, Cfg::HALF_Q, 32, Cfg::HALF_K, 32>(
                  tmem + Cfg::tm_s(x), qd, SmemDesc{kd0.lo + k_off, kd0.hi}, Cfg::IDESC_S, 0u);
            mma_commit(&B->s_full[x]);
            mma_commit(&B->k_empty[x][slot]);
            if (t == ntk - 1) mma_commit(&B->q_empty[x]);   // the item's last S: Q may be replaced
            ++n_s;
          } else {
            // with two P buffers tile B's P write no longer waits for tile A's
            // PV; its first V wait of an item then waits first for tile A to
            // have seen every earlier V tile land, so the slot barrier is at
            // most one phase behind the awaited one
            if (!attn_wait(B, &B->p_full[x], n_pv & 1, ns, SITE_ATTN_MMA) ||
                (Cfg::NP == 2 && x == 1 && t == 0 && !attn_wait_count(B, &B->v_seen, g0, ns, SITE_ATTN_MMA)) ||
                !attn_wait(B, &B->v_full[slot], ph, ns, SITE_ATTN_MMA)) {
              ok = false;
              break;
            }
            if constexpr (Cfg::NP == 2) {
              if (x == 0) *reinterpret_cast<volatile uint32_t *>(&B->v_seen) = gt + 1;
            }
            if constexpr (GATHER) fence_proxy_async_smem();
            tc_fence_after();
            // A = P [128 q x 128 keys], K-major in two 64-key halves; B = V [128 keys x D],
            // MN-major, 16 keys = 2048 bytes per K-step
            mma_chain<Cfg::BN / 16, Cfg::HALF_P, 32, 4 * 2048, 2048>(
                tmem + Cfg::tm_o(x), pd, SmemDesc{vd0.lo + v_off, vd0.hi}, Cfg::IDESC_PV, t > 0 ? 1u : 0u);
            mma_commit(&B->p_free[x]);                     // the shared P buffer may be rewritten
            if (t == ntk - 1) mma_commit(&B->o_full[x]);   // the item's O of tile x is final
            mma_commit(&B->v_empty[x][slot]);
            ++n_pv;
            ++pairs;
          }
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
    float sl2 = P.scale_log2;   // FP8: times this row's Q scale and the head's K scale (set per item)
    uint32_t g = 0, n_s = 0, n_o = 0;
    // Exponentials take turns between the two tiles (A(t), B(t), A(t+1), ...),
    // so one tile's exponentials overlap the other tile's MMAs instead of
    // competing for the same MUFU units: B(t) starts once A has finished t+1
    // steps of the item, A(t) once B has finished all its steps before B(t)
    // (in an item without tile B: all of B's steps so far).  Progress is a
    // monotonic counter per tile (exp_steps, 4 per step), not a barrier
    // parity, because tile B skips items and a parity would alias once one
    // tile runs two steps ahead of the other's wait.  other_before counts the
    // other tile's steps in earlier items (tile A runs every item, tile B
    // only items of > 128 rows).
    uint32_t other_before = 0;
    // P writes to the shared buffer happen in the order A(0), B(0), A(1), ...
    // (A(0), A(1), ... in items without tile B).  A write waits for the PV of
    // the previous write, on the p_free barrier of the tile that made it, by
    // that tile's PV count: pv_before[y] = PVs of tile y in earlier items.  A
    // waiter is never two completions behind on that barrier (the previous PV
    // of the same tile finished before the write that preceded ours), so the
    // phase parity cannot alias.
    uint32_t pv_before[2] = {0, 0};
    bool have_prev = false, prev_pair = false;
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
      if constexpr (FP8) {
        if (nrows > 0) {
          const size_t gq = static_cast<size_t>(it.h) * P.N + it.q0 + x * Cfg::BM + row;
          sl2 = P.scale_log2 * (row < nrows ? __ldg(P.q_scale + gq) : 1.f) * __ldg(P.k_scale + it.h);
        }
      }
      if (nrows <= 0) {          // this item has no tile B
        g += ntk;
        other_before += ntk;     // tile A's steps of this item
        pv_before[0] += ntk;     // and its PVs
        have_prev = true;
        prev_pair = false;
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
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B->s_free[x]);   // S_x(t + 1) may overwrite the buffer
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
        // wait for the turn: tile B's step t after tile A's step t, tile A's
        // step t after tile B's step t-1 (or B's last step of earlier items)
        {
          const uint32_t want = x == 1 ? other_before + t + 1 : other_before + (pair ? t : 0);
          if (want > 0 && !attn_warp_wait_count(B, &B->exp_steps[x ^ 1], 4u * want, ns, SITE_ATTN_SOFTMAX)) {
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
          const float2 p2 = make_float2(ex2_approx(a2.x), ex2_approx(a2.y));
          rs2 = add_f32x2(rs2, p2);
          packed[e >> 1] = pack_bf16x2(p2.x, p2.y);
        }
        __syncwarp();
        if (lane == 0) atomicAdd(&B->exp_steps[x], 1u);
        // a P buffer is free once the PV of its previous write has completed
        // (shared buffer: that PV was issued after PV_x(t - 1) completed, so
        // O_x is stable too; a buffer per tile: it is PV_x(t - 1) itself)
        int py = -1;              // tile whose PV read P last, and that PV's index
        uint32_t pidx = 0;
        if constexpr (Cfg::NP == 2) {   // own buffer: free once this tile's previous PV has completed
          if (pv_before[x] + t > 0) {
            py = x;
            pidx = pv_before[x] + t - 1;
          }
        } else if (x == 1) {
          py = 0;
          pidx = pv_before[0] + t;                          // A(t)
        } else if (t > 0) {
          py = pair ? 1 : 0;
          pidx = pv_before[py] + t - 1;                     // B(t-1), or A(t-1)
        } else if (have_prev) {
          py = prev_pair ? 1 : 0;
          pidx = pv_before[py] - 1;                         // the previous item's last write
        }
        if (py >= 0 && !attn_warp_wait(B, &B->p_free[py], pidx & 1, ns, SITE_ATTN_SOFTMAX)) {
          ok = false;
          break;
        }
        tc_fence_after();
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
        // P row: two 64-key halves, each one 128-byte swizzle row (K-major,
        // 16-byte chunks XOR row % 8)
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
          uint8_t *prow = sP + (Cfg::NP == 2 ? x * Cfg::P_BYTES : 0) + kh * Cfg::HALF_P + row * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t chunk = u ^ (row & 7);
            const int b = kh * 32 + 4 * u;
            *reinterpret_cast<uint4 *>(prow + chunk * 16) =
                make_uint4(packed[b], packed[b + 1], packed[b + 2], packed[b + 3]);
          }
        }
        tmem_st_wait();           // O rescale stores (if any) have landed
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B->p_full[x]);
      }
      if (!ok) break;
      if (x == 1 || pair) other_before += ntk;   // the other tile's steps of this item
      pv_before[0] += ntk;
      if (pair) pv_before[1] += ntk;
      have_prev = true;
      prev_pair = pair;
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
// Per (head, q-cluster): whether its block list equals the previous
// q-cluster's (same non-empty count, same ids).  Such neighbours attend to the
// same keys, so their consecutive permuted rows are planned as one row range:
// the query tiles then pack rows of several clusters instead of padding each
// cluster's tail.
__global__ void attn_plan_merge_kernel(const int32_t *__restrict__ q_off, const int32_t *__restrict__ sel_count,
                                       const int32_t *__restrict__ sel_cols, int BH, int Cq, int Ck, int max_sel,
                                       int32_t *__restrict__ same_prev) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= BH * Cq) return;
  const int h = idx / Cq, i = idx % Cq;
  int same = 0;
  if (i > 0) {
    const int32_t *qo = q_off + h * (Cq + 1);
    const int c0 = sel_count[idx - 1], c1 = sel_count[idx];
    if (c0 == c1 && c1 > 0 && c1 <= max_sel && qo[i] > qo[i - 1] && qo[i + 1] > qo[i]) {
      const int32_t *a = sel_cols + static_cast<size_t>(idx - 1) * Ck, *b = sel_cols + static_cast<size_t>(idx) * Ck;
      same = 1;
      for (int c = 0; c < c1 && same; ++c) same = a[c] == b[c];
    }
  }
  same_prev[idx] = same;
}

// Per (head, q-cluster): number of work items (256 query rows each) and of
// 128-key tiles per item; one warp per (head, q-cluster).  A q-cluster whose
// block list equals its predecessor's has no items of its own: the first
// cluster of such a group plans the group's rows (q_end = the group's last
// row + 1).  Selected k-clusters whose row ranges touch (consecutive ids, or
// ids with only empty clusters between them) form one run, and slots are
// counted per run, 32 selected clusters at a time with the same ballot rule
// the attention kernel's item loader merges them by.
__global__ void __launch_bounds__(256) attn_plan_count_kernel(const int32_t *__restrict__ q_off,
                                                              const int32_t *__restrict__ k_off,
                                                              const int32_t *__restrict__ sel_count,
                                                              const int32_t *__restrict__ sel_cols, int BH, int Cq,
                                                              int Ck, int max_sel,
                                                              const int32_t *__restrict__ same_prev,
                                                              int32_t *__restrict__ qtiles,
                                                              int32_t *__restrict__ ktiles,
                                                              int32_t *__restrict__ q_end) {
  const int lane = threadIdx.x & 31;
  const int idx = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (idx >= BH * Cq) return;   // warp-uniform
  const int h = idx / Cq, i = idx % Cq;
  if (same_prev[idx]) {   // planned by the first cluster of its group
    if (lane == 0) {
      qtiles[idx] = 0;
      ktiles[idx] = 0;
      q_end[idx] = 0;
    }
    return;
  }
  const int cnt = attn_sel_count(sel_count, idx, max_sel);
  const int32_t *cols = sel_cols + static_cast<size_t>(idx) * Ck;
  const int32_t *ko = k_off + static_cast<size_t>(h) * (Ck + 1);
  int slots = 0, m = 0, open_x = 0, open_end = -1;   // slots of closed runs; runs opened; the open run
  for (int c0 = 0; c0 < cnt; c0 += 32) {
    const int c = c0 + lane;
    int x = 0, len = 0;
    if (c < cnt) {
      const int j = cols[c];
      if (j >= 0 && j < Ck) {
        x = ko[j];
        len = ko[j + 1] - x;
      } else {
        record_error(SVG_ERR_DEVICE_CHECK, SITE_ATTN_EMPTY_ROW);
      }
    }
    const bool valid = len > 0;
    const int end = x + len;
    const unsigned below_mask = (1u << lane) - 1u;
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    const unsigned vb = vmask & below_mask;
    const int pv_end = __shfl_sync(0xffffffffu, end, vb ? 31 - __clz(vb) : 0);
    const int prev_end = vb ? pv_end : open_end;   // end of the previous non-empty range
    const bool opens = valid && x != prev_end;
    const unsigned smask = __ballot_sync(0xffffffffu, opens);
    const unsigned sb = smask & below_mask;
    const int ps_x = __shfl_sync(0xffffffffu, x, sb ? 31 - __clz(sb) : 0);
    int closed = 0;   // slots of the run this lane closes (the run before the one it opens)
    if (opens && m + __popc(sb) > 0) {
      const int run_x = sb ? ps_x : open_x;
      closed = (prev_end - run_x + 7) >> 3;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) closed += __shfl_xor_sync(0xffffffffu, closed, o);
    slots += closed;
    if (smask) open_x = __shfl_sync(0xffffffffu, x, 31 - __clz(smask));
    if (vmask) open_end = __shfl_sync(0xffffffffu, end, 31 - __clz(vmask));
    m += __popc(smask);
  }
  if (m > 0) slots += (open_end - open_x + 7) >> 3;
  if (lane == 0) {
    int last = i;
    while (last + 1 < Cq && same_prev[idx + (last + 1 - i)]) ++last;
    const int row_end = q_off[h * (Cq + 1) + last + 1];
    q_end[idx] = row_end;
    const int nq = row_end - q_off[h * (Cq + 1) + i];
    int qt = nq > 0 ? (nq + kItemRows - 1) / kItemRows : 0;
    if (qt > 0 && slots == 0) {
      record_error(SVG_ERR_DEVICE_CHECK, SITE_ATTN_EMPTY_ROW);
      qt = 0;
    }
    qtiles[idx] = qt;
    ktiles[idx] = (slots + kSlotsPerTile - 1) / kSlotsPerTile;
  }
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
    const int32_t *__restrict__ ktiles, const int32_t *__restrict__ q_end, int BH, int Cq,
    AttnItem *__restrict__ items,
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
    const int row0 = q_off[h * (Cq + 1) + i], row1 = q_end[idx];
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
    const int row0 = q_off[h * (Cq + 1) + i], row1 = q_end[idx];
    for (int t = 0; t < qt; ++t) {
      const int q0 = row0 + t * kItemRows;
      const int rows = min(kItemRows, row1 - q0);
      const int rank = atomicAdd(&hist[attn_item_bucket(h, hpg, kt, rows)], 1);
      items[rank] = AttnItem{h, i, q0, rows | (kt << 9)};
    }
  }
}

}  // namespace svg
