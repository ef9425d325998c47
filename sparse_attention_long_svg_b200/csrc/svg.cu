// libsvg.so: host side of the C ABI declared in include/svg.h.
// One translation unit, so every kernel shares one device error word.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "attn.cuh"
#include "common.cuh"
#include "dynrad.cuh"
#include "fp8.cuh"
#include "kmeans.cuh"
#include "kmeans_tc.cuh"
#include "select.cuh"
#include "sort.cuh"

using namespace svg;

namespace {

constexpr uint64_t kDefaultWaitNs = 2000000000ull;
uint64_t g_wait_ns = kDefaultWaitNs;
int g_fault = 0;

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Text of the last CUDA failure a call reported (what failed and CUDA's message).
char g_cuda_error[256] = "";
std::mutex g_cuda_error_mu;

inline svg_status cuda_status(cudaError_t e, const char *what = "CUDA call") {
  if (e == cudaSuccess) return SVG_OK;
  std::lock_guard<std::mutex> lock(g_cuda_error_mu);
  std::snprintf(g_cuda_error, sizeof(g_cuda_error), "%s: %s", what, cudaGetErrorString(e));
  return SVG_ERR_CUDA;
}

inline svg_status launch_status(const char *what = "kernel launch") {
  return cuda_status(cudaGetLastError(), what);
}

// --------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// 2-D view [rows, D] of a bf16 (or, with u8, a one-byte-per-channel)
// tensor; boxes of 128 bytes of channels x box_rows rows, 128-byte swizzle
// (the tcgen05 K-major / MN-major canonical layout).
bool make_map_2d(CUtensorMap *map, const void *base, uint64_t rows, int D, int box_rows, bool u8 = false) {
  auto enc = encoder();
  if (!enc) return false;
  const int eb = u8 ? 1 : 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * eb};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / eb), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int g_num_sms = 0;
int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

template <typename F>
bool set_smem(F kernel, size_t bytes) {
  return cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(bytes)),
                     "shared-memory size attribute") == SVG_OK;
}

// --------------------------------------------------------------- workspace carving
struct Carve {
  uint8_t *p;
  size_t used = 0;
  template <typename T>
  T *take(size_t count) {
    T *r = reinterpret_cast<T *>(p ? p + used : nullptr);
    used += align256(count * sizeof(T));
    return r;
  }
};

inline int kmeans_cpad(int C) { return (C + kKmChunk - 1) / kKmChunk * kKmChunk; }

struct KmeansWs {
  double *partial;
  float *norms, *xnorm;
  __nv_bfloat16 *hi, *lo;
  KmTie *ties;
  KmChunk *chunks;
  int32_t *bucket, *offsets, *counters, *num_chunks, *num_ties;
  int32_t *sizes(int BH, int C) const { return counters; }
  int32_t *cursor(int BH, int C) const { return counters + static_cast<size_t>(BH) * C; }
  int32_t *arrive(int BH, int C) const { return counters + 2 * static_cast<size_t>(BH) * C; }
};
KmeansWs carve_kmeans(void *ws, int BH, int N, int D, int C, size_t *bytes) {
  Carve c{static_cast<uint8_t *>(ws)};
  KmeansWs w;
  const size_t cp = static_cast<size_t>(BH) * kmeans_cpad(C);
  const size_t maxch = static_cast<size_t>(BH) * max_accum_chunks(N, C);
  w.partial = c.take<double>(maxch * D);
  w.chunks = c.take<KmChunk>(maxch);
  w.num_chunks = c.take<int32_t>(BH);
  w.xnorm = c.take<float>(static_cast<size_t>(BH) * N);
  w.ties = c.take<KmTie>(static_cast<size_t>(BH) * N);
  w.num_ties = c.take<int32_t>(1);
  w.norms = c.take<float>(cp);
  w.hi = c.take<__nv_bfloat16>(cp * D);
  w.lo = c.take<__nv_bfloat16>(cp * D);
  w.bucket = c.take<int32_t>(static_cast<size_t>(BH) * N);
  w.offsets = c.take<int32_t>(static_cast<size_t>(BH) * (C + 1));
  w.counters = c.take<int32_t>(3 * static_cast<size_t>(BH) * C);   // sizes, cursors, arrivals
  *bytes = c.used;
  return w;
}

// The attention kernel runs at most this many CTAs (one per SM); each has
// two slots of merged key ranges in the workspace (one per item in flight).
constexpr int kAttnMaxCtas = 160;

struct AttnWs {
  int32_t *num_items, *next_item, *qtiles, *ktiles, *same_prev, *q_end;
  AttnItem *items;
  int2 *ranges;
};
AttnWs carve_attn(void *ws, int BH, int N, int Cq, size_t *bytes) {
  Carve c{static_cast<uint8_t *>(ws)};
  AttnWs w;
  w.num_items = c.take<int32_t>(1);
  w.next_item = c.take<int32_t>(1);
  w.qtiles = c.take<int32_t>(static_cast<size_t>(BH) * Cq);
  w.ktiles = c.take<int32_t>(static_cast<size_t>(BH) * Cq);
  w.same_prev = c.take<int32_t>(static_cast<size_t>(BH) * Cq);
  w.q_end = c.take<int32_t>(static_cast<size_t>(BH) * Cq);
  w.items = c.take<AttnItem>(static_cast<size_t>(BH) * ((N + kItemRows - 1) / kItemRows + Cq));
  w.ranges = c.take<int2>(static_cast<size_t>(kAttnMaxCtas) * 2 * AttnCfg<128>::MAX_SEL);
  *bytes = c.used;
  return w;
}

bool sizes_ok(int BH, int N) {
  return BH > 0 && N > 0 && static_cast<int64_t>(BH) * N < (1ll << 31) - 1;
}

// Stable counting sort of assign[BH,N] by cluster: perm, offsets (and counts).
svg_status run_sort(const int32_t *assign, int BH, int N, int C, int32_t *perm, int32_t *offsets,
                    int32_t *chunk, cudaStream_t s) {
  const int nch = num_chunks(N);
  sort_hist_kernel<<<dim3(nch, BH), 256, 0, s>>>(assign, N, C, chunk);
  sort_scan_kernel<<<BH, 1024, 0, s>>>(chunk, N, C, nch, offsets);
  sort_scatter_kernel<<<dim3(nch, BH), 32, 0, s>>>(assign, N, C, chunk, perm);
  return launch_status();
}

svg_status run_row_move(bool gather, int ntensors, const void *const *src, void *const *dst,
                        const int32_t *perm, int BH, int N, int D, cudaStream_t s) {
  RowMoveArgs a{};
  for (int t = 0; t < ntensors; ++t) {
    a.src[t] = static_cast<const uint4 *>(src[t]);
    a.dst[t] = static_cast<uint4 *>(dst[t]);
  }
  const int vpr = D / 8;
  const size_t total = static_cast<size_t>(BH) * N * vpr;
  const size_t per_block = 256 * kVecPerThread;
  size_t blocks = (total + per_block - 1) / per_block;
  const size_t cap = static_cast<size_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks == 0) blocks = 1;
  if (gather)
    row_move_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, s>>>(a, ntensors, perm, BH, N,
                                                                        vpr);
  else
    row_move_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, s>>>(a, ntensors, perm, BH, N,
                                                                         vpr);
  return launch_status();
}

// --------------------------------------------------------------- kernel timing
// Event pairs recorded around the assign and attention launches while
// profiling is enabled (see svg_profile_enable in svg.h).
constexpr int kProfKernels = 2, kProfSlots = 1024;
struct ProfState {
  bool on = false, created = false;
  cudaEvent_t ev[kProfKernels][kProfSlots][2];
  int used[kProfKernels] = {0, 0};
  int dropped[kProfKernels] = {0, 0};
};
ProfState g_prof;
std::mutex g_prof_mutex;

// Returns the event pair to record around one launch, or nullptr.
cudaEvent_t *prof_slot(int kernel) {
  if (!g_prof.on) return nullptr;
  std::lock_guard<std::mutex> lock(g_prof_mutex);
  if (g_prof.used[kernel] >= kProfSlots) {
    ++g_prof.dropped[kernel];
    return nullptr;
  }
  return g_prof.ev[kernel][g_prof.used[kernel]++];
}

// (query tile, key tile) pairs the attention kernel issued MMAs for while
// profiling was on; one counter per device (module-scope device storage).
__device__ unsigned long long g_attn_issued_pairs = 0;

constexpr int kMaxDevices = 64;
void *g_issued_ptr[kMaxDevices] = {};

// Device address of g_attn_issued_pairs on the current device (nullptr on failure).
void *issued_pairs_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_prof_mutex);
  if (g_issued_ptr[dev] == nullptr) {
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_attn_issued_pairs);
    if (e != cudaSuccess) {
      cuda_status(e, "cudaGetSymbolAddress(attention pair counter)");
      cudaGetLastError();
      return nullptr;
    }
    g_issued_ptr[dev] = ptr;
  }
  return g_issued_ptr[dev];
}

}  // namespace

extern "C" {

svg_status svg_profile_attn_pairs(uint64_t *pairs) {
  if (!pairs) return SVG_ERR_INVALID_ARG;
  unsigned long long v = 0, zero = 0;
  svg_status st = cuda_status(cudaMemcpyFromSymbol(&v, g_attn_issued_pairs, sizeof(v)),
                              "cudaMemcpyFromSymbol(attention pair counter)");
  if (st != SVG_OK) return st;
  st = cuda_status(cudaMemcpyToSymbol(g_attn_issued_pairs, &zero, sizeof(zero)),
                   "cudaMemcpyToSymbol(attention pair counter)");
  if (st != SVG_OK) return st;
  *pairs = v;
  return SVG_OK;
}

svg_status svg_profile_enable(int on) {
  std::lock_guard<std::mutex> lock(g_prof_mutex);
  if (on && !g_prof.created) {
    for (int k = 0; k < kProfKernels; ++k)
      for (int i = 0; i < kProfSlots; ++i)
        for (int j = 0; j < 2; ++j)
          if (cudaEventCreate(&g_prof.ev[k][i][j]) != cudaSuccess) return SVG_ERR_CUDA;
    g_prof.created = true;
  }
  g_prof.on = on != 0;
  return SVG_OK;
}

svg_status svg_profile_read(int kernel, double *ms, int *launches, int *dropped) {
  if (kernel < 0 || kernel >= kProfKernels || !ms || !launches) return SVG_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_prof_mutex);
  double total = 0.0;
  for (int i = 0; i < g_prof.used[kernel]; ++i) {
    if (cudaEventSynchronize(g_prof.ev[kernel][i][1]) != cudaSuccess) return SVG_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, g_prof.ev[kernel][i][0], g_prof.ev[kernel][i][1]) != cudaSuccess)
      return SVG_ERR_CUDA;
    total += t;
  }
  *ms = total;
  *launches = g_prof.used[kernel];
  if (dropped) *dropped = g_prof.dropped[kernel];
  g_prof.used[kernel] = 0;
  g_prof.dropped[kernel] = 0;
  return SVG_OK;
}

const char *svg_status_string(svg_status s) {
  switch (s) {
    case SVG_OK: return "SVG_OK";
    case SVG_ERR_INVALID_ARG: return "SVG_ERR_INVALID_ARG";
    case SVG_ERR_UNSUPPORTED: return "SVG_ERR_UNSUPPORTED";
    case SVG_ERR_WORKSPACE: return "SVG_ERR_WORKSPACE";
    case SVG_ERR_CUDA: return "SVG_ERR_CUDA";
    case SVG_ERR_TIMEOUT: return "SVG_ERR_TIMEOUT";
    case SVG_ERR_DEVICE_CHECK: return "SVG_ERR_DEVICE_CHECK";
  }
  return "SVG_ERR_UNKNOWN";
}

const char *svg_last_cuda_error(void) {
  std::lock_guard<std::mutex> lock(g_cuda_error_mu);
  static thread_local char copy[sizeof(g_cuda_error)];
  std::memcpy(copy, g_cuda_error, sizeof(copy));
  return copy;
}

const char *svg_version(void) { return "svg-b200 0.2 (sm_100a)"; }

void svg_set_wait_timeout_ns(uint64_t ns) { g_wait_ns = ns ? ns : kDefaultWaitNs; }

void svg_debug_set_fault(int fault) { g_fault = fault; }

svg_status svg_get_error_detail(svg_stream_t stream, int32_t *site, int32_t *block) {
  if (site) *site = 0;
  if (block) *block = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SVG_ERR_CUDA;
  uint32_t word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return SVG_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return SVG_ERR_CUDA;
  if (site) *site = static_cast<int32_t>((word >> 8) & 0xFFu);
  if (block) *block = static_cast<int32_t>(word >> 16);
  return static_cast<svg_status>(word & 0xFFu);
}

svg_status svg_get_error(svg_stream_t stream) { return svg_get_error_detail(stream, nullptr, nullptr); }

// ------------------------------------------------------------------ k-means
size_t svg_kmeans_workspace_size(int BH, int N, int D, int C) {
  if (!sizes_ok(BH, N) || C <= 0 || D <= 0) return 0;
  size_t bytes = 0;
  carve_kmeans(nullptr, BH, N, D, C, &bytes);
  return bytes;
}

svg_status svg_kmeans(const void *x, int BH, int N, int D, int C, int iters, float *centroids,
                      int32_t *assign, int32_t *counts, void *ws, size_t ws_bytes,
                      svg_stream_t stream) {
  if (!x || !centroids || !assign || !counts || !ws) return SVG_ERR_INVALID_ARG;
  if (!sizes_ok(BH, N) || C < 1 || C > N || iters < 1) return SVG_ERR_INVALID_ARG;
  if (C > kMaxClusters) return SVG_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return SVG_ERR_UNSUPPORTED;
  if (!aligned(x, 16) || !aligned(centroids, 16) || !aligned(ws, 256)) return SVG_ERR_INVALID_ARG;
  size_t need = 0;
  KmeansWs w = carve_kmeans(ws, BH, N, D, C, &need);
  if (ws_bytes < need) return SVG_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
  const int Cpad = kmeans_cpad(C);
  CUtensorMap mx, mhi, mlo;
  if (!make_map_2d(&mx, x, static_cast<uint64_t>(BH) * N, D, 128) ||
      !make_map_2d(&mhi, w.hi, static_cast<uint64_t>(BH) * Cpad, D, 128) ||
      !make_map_2d(&mlo, w.lo, static_cast<uint64_t>(BH) * Cpad, D, 128))
    return SVG_ERR_CUDA;
  kmeans_split_kernel<<<dim3((Cpad + 7) / 8, BH), 256, 0, s>>>(centroids, C, Cpad, D, w.hi, w.lo,
                                                              w.norms, w.num_ties, w.counters);
  if (launch_status("kmeans_split_kernel") != SVG_OK) return SVG_ERR_CUDA;
  // ||x||^2 per token (for the near-tie margin) is formed by the first
  // round's assign from the x tiles it loads anyway, and read by later rounds
  const int units = BH * ((N + 127) / 128);
  const int ga = units < num_sms() ? units : num_sms();
  const dim3 gb((N + 1024 * kBucketTokens - 1) / (1024 * kBucketTokens), BH);
  const dim3 gacc((max_accum_chunks(N, C) + kAccumWarps - 1) / kAccumWarps, BH);
  int32_t *sizes = w.sizes(BH, C), *cursor = w.cursor(BH, C), *arrive = w.arrive(BH, C);
  // one centroid chunk (C <= 128): the chunk stays resident per head; more:
  // tiles in pairs sharing every chunk
  const bool single = Cpad == kKmChunk;
  int make_xnorm = 1;
  auto assign_kernel = [&](auto kernel, size_t smem_bytes, int threads) {
    if (!set_smem(kernel, smem_bytes)) return SVG_ERR_CUDA;
    kernel<<<ga, threads, smem_bytes, s>>>(mx, mhi, mlo, BH, N, C, Cpad, w.norms, w.xnorm, assign,
                                          sizes, w.ties, w.num_ties, make_xnorm, g_wait_ns);
    return launch_status("kmeans_assign_tc_kernel");
  };
  for (int it = 0; it < iters; ++it) {
    cudaEvent_t *pe = prof_slot(0);
    if (pe) cudaEventRecord(pe[0], s);
    svg_status st;
    if (D == 128)
      st = single ? assign_kernel(kmeans_assign_tc_kernel<128, true>, KmCfg<128, true>::SMEM_BYTES,
                                  KmCfg<128, true>::THREADS)
                  : assign_kernel(kmeans_assign_tc_kernel<128, false>, KmCfg<128, false>::SMEM_BYTES,
                                  KmCfg<128, false>::THREADS);
    else
      st = single ? assign_kernel(kmeans_assign_tc_kernel<64, true>, KmCfg<64, true>::SMEM_BYTES,
                                  KmCfg<64, true>::THREADS)
                  : assign_kernel(kmeans_assign_tc_kernel<64, false>, KmCfg<64, false>::SMEM_BYTES,
                                  KmCfg<64, false>::THREADS);
    if (st != SVG_OK) return st;
    make_xnorm = 0;
    if (pe) cudaEventRecord(pe[1], s);
    if (D == 128)
      kmeans_refine_kernel<128><<<num_sms() * 4, 256, 0, s>>>(xb, N, C, centroids, w.ties,
                                                              w.num_ties, assign, sizes);
    else
      kmeans_refine_kernel<64><<<num_sms() * 4, 256, 0, s>>>(xb, N, C, centroids, w.ties,
                                                             w.num_ties, assign, sizes);
    if (launch_status("kmeans_refine_kernel") != SVG_OK) return SVG_ERR_CUDA;
    kmeans_bucket_kernel<<<gb, 1024, 0, s>>>(assign, N, C, sizes, cursor, w.bucket, w.offsets,
                                             counts, w.chunks, w.num_chunks);
    if (launch_status("kmeans_bucket_kernel") != SVG_OK) return SVG_ERR_CUDA;
    if (D == 128)
      kmeans_accum_kernel<128><<<gacc, 32 * kAccumWarps, 0, s>>>(xb, N, C, Cpad, w.bucket, w.offsets, w.chunks,
                                                    w.num_chunks, w.partial, arrive, sizes, cursor,
                                                    centroids, w.hi, w.lo, w.norms, w.num_ties);
    else
      kmeans_accum_kernel<64><<<gacc, 32 * kAccumWarps, 0, s>>>(xb, N, C, Cpad, w.bucket, w.offsets, w.chunks,
                                                   w.num_chunks, w.partial, arrive, sizes, cursor,
                                                   centroids, w.hi, w.lo, w.norms, w.num_ties);
    if (launch_status("kmeans_accum_kernel") != SVG_OK) return SVG_ERR_CUDA;
  }
  return launch_status();
}

// ------------------------------------------------------------------ permutation
size_t svg_permute_workspace_size(int BH, int N, int C) {
  if (!sizes_ok(BH, N) || C <= 0) return 0;
  return align256(static_cast<size_t>(BH) * num_chunks(N) * C * sizeof(int32_t));
}

svg_status svg_permute(const int32_t *assign, int BH, int N, int C, int32_t *perm,
                       int32_t *offsets, int ntensors, const void *const *src, void *const *dst,
                       int D, void *ws, size_t ws_bytes, svg_stream_t stream) {
  if (!assign || !perm || !offsets || !ws) return SVG_ERR_INVALID_ARG;
  if (!sizes_ok(BH, N) || C < 1 || ntensors < 0 || ntensors > 3) return SVG_ERR_INVALID_ARG;
  if (C > kMaxClusters) return SVG_ERR_UNSUPPORTED;
  if (ntensors > 0) {
    if (!src || !dst) return SVG_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SVG_ERR_UNSUPPORTED;
    for (int t = 0; t < ntensors; ++t) {
      if (!src[t] || !dst[t] || !aligned(src[t], 16) || !aligned(dst[t], 16))
        return SVG_ERR_INVALID_ARG;
      if (src[t] == dst[t]) return SVG_ERR_INVALID_ARG;
    }
  }
  if (!aligned(ws, 256)) return SVG_ERR_INVALID_ARG;
  if (ws_bytes < svg_permute_workspace_size(BH, N, C)) return SVG_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  svg_status st = run_sort(assign, BH, N, C, perm, offsets, static_cast<int32_t *>(ws), s);
  if (st != SVG_OK || ntensors == 0) return st;
  return run_row_move(true, ntensors, src, dst, perm, BH, N, D, s);
}

svg_status svg_unpermute(const void *xp, const int32_t *perm, int BH, int N, int D, void *x,
                         svg_stream_t stream) {
  if (!xp || !perm || !x || xp == x) return SVG_ERR_INVALID_ARG;
  if (!sizes_ok(BH, N)) return SVG_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SVG_ERR_UNSUPPORTED;
  if (!aligned(xp, 16) || !aligned(x, 16)) return SVG_ERR_INVALID_ARG;
  const void *src[1] = {xp};
  void *dst[1] = {x};
  return run_row_move(false, 1, src, dst, perm, BH, N, D, reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ top-p selection
svg_status svg_select_topp(const float *mu_q, const int32_t *n_q, const float *mu_k,
                           const int32_t *n_k, int BH, int Cq, int Ck, int D, float p, float scale,
                           int32_t *sel_count, int32_t *sel_cols, svg_stream_t stream) {
  if (!mu_q || !n_q || !mu_k || !n_k || !sel_count || !sel_cols) return SVG_ERR_INVALID_ARG;
  if (BH <= 0 || Cq <= 0 || Ck <= 0 || !(p > 0.f) || std::isnan(p)) return SVG_ERR_INVALID_ARG;
  if (Ck > kMaxCk || (D != 64 && D != 128)) return SVG_ERR_UNSUPPORTED;
  if (!aligned(mu_q, 16) || !aligned(mu_k, 16)) return SVG_ERR_INVALID_ARG;
  // the default scale is formed in float64 (1/sqrt(D) correctly rounded), the
  // precision the cut is decided in
  const double scale_d = scale > 0.f ? static_cast<double>(scale) : 1.0 / std::sqrt(static_cast<double>(D));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t smem = select_smem_bytes(D, Ck);
  const dim3 grid((Cq + kSelRows - 1) / kSelRows, BH);
  const int cpl = select_cpl(Ck);
  auto launch = [&](auto kernel) {
    if (!set_smem(kernel, smem)) return SVG_ERR_CUDA;
    kernel<<<grid, kSelRows * 32, smem, s>>>(mu_q, n_q, mu_k, n_k, Cq, Ck, p, scale_d, sel_count, sel_cols);
    return launch_status("select_topp_kernel");
  };
  if (D == 128) {
    switch (cpl) {
      case 4: return launch(select_topp_kernel<128, 4>);
      case 8: return launch(select_topp_kernel<128, 8>);
      case 16: return launch(select_topp_kernel<128, 16>);
      default: return launch(select_topp_kernel<128, 32>);
    }
  }
  switch (cpl) {
    case 4: return launch(select_topp_kernel<64, 4>);
    case 8: return launch(select_topp_kernel<64, 8>);
    case 16: return launch(select_topp_kernel<64, 16>);
    default: return launch(select_topp_kernel<64, 32>);
  }
}

// ------------------------------------------------------------------ sparse attention
size_t svg_sparse_attn_workspace_size(int BH, int N, int Cq) {
  if (!sizes_ok(BH, N) || Cq <= 0) return 0;
  size_t bytes = 0;
  carve_attn(nullptr, BH, N, Cq, &bytes);
  return bytes;
}

}  // extern "C"

namespace {
// Shared body of svg_sparse_attn (perm == nullptr: permuted output rows),
// svg_sparse_attn_unpermuted (row r of a head stored at row perm[r]),
// svg_sparse_attn_gather (perm_k set) and svg_sparse_attn_fp8 (q_scale and
// k_scale set: qp and kp hold E4M3 bytes).
svg_status sparse_attn_impl(const void *qp, const void *kp, const void *vp, const int32_t *perm_k,
                            int BH, int N, int D, const int32_t *q_off, int Cq, const int32_t *k_off,
                            int Ck, const int32_t *sel_count, const int32_t *sel_cols, float scale,
                            const int32_t *perm, void *op, float *lse, void *ws, size_t ws_bytes,
                            svg_stream_t stream, const float *q_scale = nullptr, const float *k_scale = nullptr) {
  if (!qp || !kp || !vp || !q_off || !k_off || !sel_count || !sel_cols || !op || !ws)
    return SVG_ERR_INVALID_ARG;
  const bool gather = perm_k != nullptr;
  const bool fp8 = q_scale != nullptr;
  if (fp8 && (k_scale == nullptr || gather)) return SVG_ERR_INVALID_ARG;
  if (perm != nullptr && (op == qp || op == kp || op == vp)) return SVG_ERR_INVALID_ARG;
  if (!sizes_ok(BH, N) || Cq < 1 || Ck < 1) return SVG_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SVG_ERR_UNSUPPORTED;
  if (fp8 && D != 128) return SVG_ERR_UNSUPPORTED;
  if (Ck > AttnCfg<128>::MAX_SEL) return SVG_ERR_UNSUPPORTED;
  if (!aligned(qp, 16) || !aligned(kp, 16) || !aligned(vp, 16) || !aligned(op, 16) ||
      !aligned(ws, 256))
    return SVG_ERR_INVALID_ARG;
  size_t need = 0;
  AttnWs w = carve_attn(ws, BH, N, Cq, &need);
  if (ws_bytes < need) return SVG_ERR_WORKSPACE;
  if (!(scale > 0.f)) scale = 1.f / std::sqrt(static_cast<float>(D));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  const int pairs = BH * Cq;
  const int max_sel = Ck < AttnCfg<128>::MAX_SEL ? Ck : AttnCfg<128>::MAX_SEL;
  attn_plan_merge_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(q_off, sel_count, sel_cols, BH, Cq, Ck, max_sel,
                                                            w.same_prev);
  attn_plan_count_kernel<<<(pairs + 7) / 8, 256, 0, s>>>(q_off, k_off, sel_count, sel_cols, BH,
                                                            Cq, Ck, max_sel, w.same_prev, w.qtiles, w.ktiles,
                                                            w.q_end);
  attn_plan_emit_kernel<<<1, kAttnBuckets, 0, s>>>(q_off, w.qtiles, w.ktiles, w.q_end, BH, Cq, w.items,
                                                   w.num_items, w.next_item);
  svg_status st = launch_status();
  if (st != SVG_OK) return st;

  AttnMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const uint64_t rows = static_cast<uint64_t>(BH) * N;
  if (!make_map_2d(&maps.q, qp, rows, D, 128, fp8)) return SVG_ERR_CUDA;
  for (int b = 0; b < (gather ? 0 : kNumBoxSizes); ++b)   // gather mode copies rows without tensor maps
    if (!make_map_2d(&maps.k[b], kp, rows, D, 8 << b, fp8) || !make_map_2d(&maps.v[b], vp, rows, D, 8 << b))
      return SVG_ERR_CUDA;
  AttnParams prm;
  prm.q_off = q_off;
  prm.k_off = k_off;
  prm.sel_count = sel_count;
  prm.sel_cols = sel_cols;
  prm.items = w.items;
  prm.num_items = w.num_items;
  prm.next_item = w.next_item;
  prm.op = static_cast<__nv_bfloat16 *>(op);
  prm.lse = lse;
  prm.perm = perm;
  prm.perm_k = perm_k;
  prm.kg = static_cast<const __nv_bfloat16 *>(kp);
  prm.vg = static_cast<const __nv_bfloat16 *>(vp);
  prm.q_scale = q_scale;
  prm.k_scale = k_scale;
  prm.ranges = w.ranges;
  prm.issued = nullptr;
  if (g_prof.on) {
    prm.issued = static_cast<unsigned long long *>(issued_pairs_address());
    if (prm.issued == nullptr) return SVG_ERR_CUDA;
  }
  prm.N = N;
  prm.Cq = Cq;
  prm.Ck = Ck;
  prm.BH = BH;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wait_ns = g_wait_ns;
  prm.fault = g_fault;
  const int grid = num_sms() < kAttnMaxCtas ? num_sms() : kAttnMaxCtas;
  cudaEvent_t *pe = prof_slot(1);
  if (pe) cudaEventRecord(pe[0], s);
  auto launch = [&](auto kernel, int threads, int smem) {
    if (!set_smem(kernel, smem)) return false;
    kernel<<<grid, threads, smem, s>>>(maps, prm);
    return true;
  };
  bool ok;
  if (fp8)
    ok = launch(sparse_attn_kernel<128, false, true>, AttnCfg<128, true>::THREADS, AttnCfg<128, true>::SMEM_BYTES);
  else if (D == 128)
    ok = gather ? launch(sparse_attn_kernel<128, true>, AttnCfg<128>::THREADS, AttnCfg<128>::SMEM_BYTES)
                : launch(sparse_attn_kernel<128, false>, AttnCfg<128>::THREADS, AttnCfg<128>::SMEM_BYTES);
  else
    ok = gather ? launch(sparse_attn_kernel<64, true>, AttnCfg<64>::THREADS, AttnCfg<64>::SMEM_BYTES)
                : launch(sparse_attn_kernel<64, false>, AttnCfg<64>::THREADS, AttnCfg<64>::SMEM_BYTES);
  if (!ok) return SVG_ERR_CUDA;
  if (pe) cudaEventRecord(pe[1], s);
  return launch_status("sparse_attn_kernel");
}
}  // namespace

extern "C" {

svg_status svg_sparse_attn(const void *qp, const void *kp, const void *vp, int BH, int N, int D,
                           const int32_t *q_off, int Cq, const int32_t *k_off, int Ck,
                           const int32_t *sel_count, const int32_t *sel_cols, float scale,
                           void *op, float *lse, void *ws, size_t ws_bytes,
                           svg_stream_t stream) {
  return sparse_attn_impl(qp, kp, vp, nullptr, BH, N, D, q_off, Cq, k_off, Ck, sel_count, sel_cols,
                          scale, nullptr, op, lse, ws, ws_bytes, stream);
}

svg_status svg_sparse_attn_unpermuted(const void *qp, const void *kp, const void *vp, int BH,
                                      int N, int D, const int32_t *q_off, int Cq,
                                      const int32_t *k_off, int Ck, const int32_t *sel_count,
                                      const int32_t *sel_cols, float scale, const int32_t *perm_q,
                                      void *o, float *lse, void *ws, size_t ws_bytes,
                                      svg_stream_t stream) {
  if (!perm_q) return SVG_ERR_INVALID_ARG;
  return sparse_attn_impl(qp, kp, vp, nullptr, BH, N, D, q_off, Cq, k_off, Ck, sel_count, sel_cols,
                          scale, perm_q, o, lse, ws, ws_bytes, stream);
}

int svg_dynrad_num_blocks(int N, int frames, int block) {
  if (N <= 0 || frames <= 0 || block <= 0 || N % frames != 0) return 0;
  const long long cb = static_cast<long long>(frames) * dynrad_blocks_per_frame(N, frames, block);
  return cb > (1ll << 30) ? 0 : static_cast<int>(cb);
}

size_t svg_dynrad_workspace_size(int BH, int N, int D, int frames, int block) {
  const int Cb = svg_dynrad_num_blocks(N, frames, block);
  if (Cb == 0 || BH <= 0 || D <= 0 || !sizes_ok(BH, N)) return 0;
  return align256(2ull * static_cast<size_t>(BH) * Cb * D * sizeof(double));
}

svg_status svg_dynrad_select(const void *q, const void *k, int BH, int N, int D, int frames, int block, int mode,
                             float w0, float gamma, float rho0, float theta, float scale, int32_t *offsets,
                             int32_t *sel_count, int32_t *sel_cols, void *ws, size_t ws_bytes,
                             svg_stream_t stream) {
  if (!offsets || !sel_count || !sel_cols || !sizes_ok(BH, N)) return SVG_ERR_INVALID_ARG;
  const int Cb = svg_dynrad_num_blocks(N, frames, block);
  if (Cb == 0) return SVG_ERR_INVALID_ARG;
  if (Cb > kDynradMaxBlocks) return SVG_ERR_UNSUPPORTED;
  if (mode < SVG_DYNRAD_CANDIDATES || mode > SVG_DYNRAD_DYNAMIC) return SVG_ERR_INVALID_ARG;
  if (!(w0 >= 0.f) || !(gamma >= 0.f) || !(w0 < 1e30f) || !(gamma < 1e30f)) return SVG_ERR_INVALID_ARG;
  if (mode == SVG_DYNRAD_STATIC && !(rho0 > 0.f && rho0 < 1e30f)) return SVG_ERR_INVALID_ARG;
  const bool dynamic = mode == SVG_DYNRAD_DYNAMIC;
  if (dynamic) {
    if (!q || !k || !ws || std::isnan(theta)) return SVG_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SVG_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(ws, 256)) return SVG_ERR_INVALID_ARG;
    if (ws_bytes < svg_dynrad_workspace_size(BH, N, D, frames, block)) return SVG_ERR_WORKSPACE;
  }
  const int nb = dynrad_blocks_per_frame(N, frames, block);
  const double scale_d = scale > 0.f ? static_cast<double>(scale) : 1.0 / std::sqrt(static_cast<double>(D));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int n_off = BH * (Cb + 1);
  dynrad_offsets_kernel<<<(n_off + 255) / 256, 256, 0, s>>>(BH, N, frames, nb, block, offsets);
  if (launch_status("dynrad_offsets_kernel") != SVG_OK) return SVG_ERR_CUDA;
  double *means = static_cast<double *>(ws);
  const dim3 g(Cb, BH);
  if (dynamic) {
    const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(q), *kb = static_cast<const __nv_bfloat16 *>(k);
    if (D == 128)
      dynrad_means_kernel<128><<<dim3(Cb, BH, 2), 128, 0, s>>>(qb, kb, BH, N, frames, nb, block, means);
    else
      dynrad_means_kernel<64><<<dim3(Cb, BH, 2), 64, 0, s>>>(qb, kb, BH, N, frames, nb, block, means);
    if (launch_status("dynrad_means_kernel") != SVG_OK) return SVG_ERR_CUDA;
  }
  const int Dk = dynamic ? D : 64;   // the query-mean buffer is only read in dynamic mode
  const size_t smem = dynrad_select_smem(frames, Dk);
  const double w0d = w0, gd = gamma, rd = rho0, td = theta;
  if (Dk == 128)
    dynrad_select_kernel<128><<<g, 32, smem, s>>>(BH, frames, nb, mode, w0d, gd, rd, td, scale_d, means,
                                                  sel_count, sel_cols);
  else
    dynrad_select_kernel<64><<<g, 32, smem, s>>>(BH, frames, nb, mode, w0d, gd, rd, td, scale_d,
                                                 dynamic ? means : nullptr, sel_count, sel_cols);
  return launch_status("dynrad_select_kernel");
}

svg_status svg_sparse_attn_gather(const void *qp, const void *k, const void *v, const int32_t *perm_k,
                                  int BH, int N, int D, const int32_t *q_off, int Cq,
                                  const int32_t *k_off, int Ck, const int32_t *sel_count,
                                  const int32_t *sel_cols, float scale, const int32_t *perm_q,
                                  void *o, float *lse, void *ws, size_t ws_bytes,
                                  svg_stream_t stream) {
  if (!perm_k) return SVG_ERR_INVALID_ARG;
  if (o == k || o == v) return SVG_ERR_INVALID_ARG;
  return sparse_attn_impl(qp, k, v, perm_k, BH, N, D, q_off, Cq, k_off, Ck, sel_count, sel_cols,
                          scale, perm_q, o, lse, ws, ws_bytes, stream);
}

svg_status svg_quantize_e4m3(const void *x, const int32_t *perm, int BH, int N, int D, int per_row, void *x8,
                             float *scales, svg_stream_t stream) {
  if (!x || !x8 || !scales || !sizes_ok(BH, N) || (per_row != 0 && per_row != 1)) return SVG_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SVG_ERR_UNSUPPORTED;
  if (!aligned(x, 16) || !aligned(x8, 16) || !aligned(scales, 4) || x == x8) return SVG_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
  uint8_t *q = static_cast<uint8_t *>(x8);
  const size_t rows = static_cast<size_t>(BH) * N;
  const size_t per_block = 8 * (256 / D) * 4;   // 8 warps x rows per warp pass x passes per iteration
  const size_t want = (rows + per_block - 1) / per_block;
  const int grid = static_cast<int>(want < static_cast<size_t>(num_sms()) * 8 ? want : num_sms() * 8);
  if (per_row) {
    if (D == 128)
      quant_e4m3_kernel<128, true><<<grid, 256, 0, s>>>(xb, perm, N, rows, nullptr, q, scales);
    else
      quant_e4m3_kernel<64, true><<<grid, 256, 0, s>>>(xb, perm, N, rows, nullptr, q, scales);
    return launch_status("quant_e4m3_kernel");
  }
  // per head: amax (float bits, max-folded into the zeroed scales), quantise, amax -> scale
  const size_t per_head = static_cast<size_t>(N) * D;
  int chunks = static_cast<int>((per_head / 8 + 255) / 256);
  const int cap = (num_sms() * 8 + BH - 1) / BH;
  if (chunks > cap) chunks = cap;
  if (chunks < 1) chunks = 1;
  int32_t *bits = reinterpret_cast<int32_t *>(scales);
  svg_status st = cuda_status(cudaMemsetAsync(bits, 0, static_cast<size_t>(BH) * sizeof(int32_t), s),
                              "cudaMemsetAsync(scales)");
  if (st != SVG_OK) return st;
  head_amax_kernel<<<dim3(chunks, BH), 256, 0, s>>>(xb, per_head, bits);
  if ((st = launch_status("head_amax_kernel")) != SVG_OK) return st;
  if (D == 128)
    quant_e4m3_kernel<128, false><<<grid, 256, 0, s>>>(xb, perm, N, rows, bits, q, nullptr);
  else
    quant_e4m3_kernel<64, false><<<grid, 256, 0, s>>>(xb, perm, N, rows, bits, q, nullptr);
  if ((st = launch_status("quant_e4m3_kernel")) != SVG_OK) return st;
  head_scale_kernel<<<(BH + 255) / 256, 256, 0, s>>>(bits, BH);
  return launch_status("head_scale_kernel");
}

svg_status svg_sparse_attn_fp8(const void *q8, const float *q_scale, const void *k8, const float *k_scale,
                               const void *vp, int BH, int N, int D, const int32_t *q_off, int Cq,
                               const int32_t *k_off, int Ck, const int32_t *sel_count, const int32_t *sel_cols,
                               float scale, const int32_t *perm_q, void *o, float *lse, void *ws,
                               size_t ws_bytes, svg_stream_t stream) {
  if (!q_scale || !k_scale) return SVG_ERR_INVALID_ARG;
  return sparse_attn_impl(q8, k8, vp, nullptr, BH, N, D, q_off, Cq, k_off, Ck, sel_count, sel_cols, scale,
                          perm_q, o, lse, ws, ws_bytes, stream, q_scale, k_scale);
}

}  // extern "C"

// ------------------------------------------------------------------ sparse attention without allocation
// Scratch for callers that cannot pass a workspace (see svg.h): a fixed array
// in this module, one per device that loads the library.  Host code must not
// hand the symbol itself to a kernel (in host code it only names a host-side
// stand-in); its device address is looked up once per device.
namespace {
static __device__ __align__(256) uint8_t g_noalloc_scratch[SVG_NOALLOC_SCRATCH_BYTES];

void *g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Device address of g_noalloc_scratch on the current device (nullptr on failure).
void *noalloc_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) {
      cuda_status(e, "cudaGetSymbolAddress(no-allocation scratch)");   // recorded for svg_last_cuda_error
      cudaGetLastError();                                              // and not left pending
      return nullptr;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  return g_noalloc_ptr[dev];
}
}  // namespace

extern "C" svg_status svg_sparse_attn_noalloc(const void *qp, const void *kp, const void *vp, int BH,
                                              int N, int D, const int32_t *q_off, int Cq,
                                              const int32_t *k_off, int Ck,
                                              const int32_t *sel_count, const int32_t *sel_cols,
                                              float scale, void *op, float *lse,
                                              svg_stream_t stream) {
  if (!sizes_ok(BH, N) || Cq < 1) return SVG_ERR_INVALID_ARG;
  const size_t need = svg_sparse_attn_workspace_size(BH, N, Cq);
  if (need == 0 || need > SVG_NOALLOC_SCRATCH_BYTES) return SVG_ERR_WORKSPACE;
  void *ws = noalloc_scratch_address();
  if (ws == nullptr) return SVG_ERR_CUDA;
  // Every scratch entry the attention path reads is written earlier in the
  // same call (planning kernels), so leftovers of a previous call are harmless.
  return svg_sparse_attn(qp, kp, vp, BH, N, D, q_off, Cq, k_off, Ck, sel_count, sel_cols, scale, op,
                         lse, ws, SVG_NOALLOC_SCRATCH_BYTES, stream);
}
