// DynamicRad block masks (the page "DynamicRad: Content-Adaptive Sparse
// Attention for Long Video Diffusion", section 2(a) "Unified candidate set and
// dual-mode selection"), produced in the block-list format of the top-p
// selection so the same attention kernel consumes them.
//
// Tokens are frame-major (token n = t S + s, S = N / frames); a block is B
// consecutive tokens of one frame, so frame t holds nb = ceil(S / B) blocks
// and block id c = t nb + b covers tokens [t S + b B, t S + min((b+1) B, S)).
// Radial candidate set: key block (t2, b2) is a candidate of query block
// (t1, b1) iff |b1 - b2| <= w(|t1 - t2|), w(d) = floor(w0 gamma^d), where
// gamma^d is formed by d successive float64 multiplications.
//   mode 0: every candidate;
//   mode 1 (static ratio): per key frame the k = max(1, ceil(rho(d) m))
//     candidates nearest to b1 (ties to the lower b2), m = candidates in that
//     frame, rho(d) = min(1, rho0 gamma^d);
//   mode 2 (dynamic threshold): candidates whose proxy
//     scale * mean(q block) . mean(k block) (float64) is >= theta; a row that
//     keeps none keeps its highest-proxy candidate (ties to the lower id).
// Kept ids are written in ascending order.
#pragma once
#include "common.cuh"

namespace svg {

constexpr int kDynradMaxBlocks = 1024;   // the attention kernel's limit on key blocks

__host__ __device__ inline int dynrad_blocks_per_frame(int N, int frames, int block) {
  const int S = N / frames;
  return (S + block - 1) / block;
}

// offsets [BH, Cb + 1]: first token of every block, then N.
__global__ void dynrad_offsets_kernel(int BH, int N, int frames, int nb, int block, int32_t *__restrict__ offsets) {
  const int Cb = frames * nb;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= BH * (Cb + 1)) return;
  const int c = idx % (Cb + 1);
  const int S = N / frames;
  offsets[idx] = c == Cb ? N : (c / nb) * S + min((c % nb) * block, S);
}

// grid (Cb, BH, 2), D threads: z = 0 averages q, z = 1 averages k; thread d
// sums channel d of the block's rows in float64 (exact for bf16 inputs) and
// divides once.  means [2][BH][Cb][D].
template <int D>
__global__ void __launch_bounds__(D) dynrad_means_kernel(const __nv_bfloat16 *__restrict__ q,
                                                         const __nv_bfloat16 *__restrict__ k, int BH, int N,
                                                         int frames, int nb, int block,
                                                         double *__restrict__ means) {
  const int c = blockIdx.x, h = blockIdx.y, z = blockIdx.z;
  const int S = N / frames;
  const int r0 = (c / nb) * S + min((c % nb) * block, S);
  const int r1 = (c / nb) * S + min((c % nb + 1) * block, S);
  const __nv_bfloat16 *x = (z == 0 ? q : k) + static_cast<size_t>(h) * N * D;
  double s = 0.0;
  for (int r = r0; r < r1; ++r) s += static_cast<double>(__bfloat162float(x[static_cast<size_t>(r) * D + threadIdx.x]));
  const int Cb = frames * nb;
  means[((static_cast<size_t>(z) * BH + h) * Cb + c) * D + threadIdx.x] = r1 > r0 ? s / (r1 - r0) : 0.0;
}

// One warp per (query block, head): grid (Cb, BH), 32 threads; dynamic shared
// memory: frames ints (windows) + frames doubles (ratios) + D doubles (the
// query block's mean).
template <int D>
__global__ void __launch_bounds__(32) dynrad_select_kernel(int BH, int frames, int nb, int mode, double w0,
                                                           double gamma, double rho0, double theta, double scale,
                                                           const double *__restrict__ means,
                                                           int32_t *__restrict__ sel_count,
                                                           int32_t *__restrict__ sel_cols) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  double *rtab = reinterpret_cast<double *>(smem_raw);   // [frames]
  double *qm = rtab + frames;                              // [D]
  int *wtab = reinterpret_cast<int *>(qm + D);             // [frames]
  const int lane = threadIdx.x;
  const int i = blockIdx.x, h = blockIdx.y;
  const int Cb = frames * nb;
  const int t1 = i / nb, b1 = i % nb;
  if (lane == 0) {   // w0 gamma^d and rho0 gamma^d by successive multiplications
    double w = w0, r = rho0;
    for (int d = 0; d < frames; ++d) {
      wtab[d] = static_cast<int>(floor(fmin(w, static_cast<double>(nb))));
      rtab[d] = fmin(1.0, r);
      w *= gamma;
      r *= gamma;
    }
  }
  const double *mk = nullptr;   // dynamic mode: the key block means of this head
  if (mode == 2) {
    const double *mq = means + (static_cast<size_t>(h) * Cb + i) * D;
    mk = means + (static_cast<size_t>(BH + h) * Cb) * D;
    for (int d = lane; d < D; d += 32) qm[d] = mq[d];
  }
  __syncwarp();
  int32_t *out = sel_cols + (static_cast<size_t>(h) * Cb + i) * Cb;
  int pos = 0;
  double best = -INFINITY;   // mode 2: this lane's best proxy and its id (the fallback)
  int best_id = 0x7fffffff;
  for (int t2 = 0; t2 < frames; ++t2) {
    const int d = t1 > t2 ? t1 - t2 : t2 - t1;
    const int w = wtab[d];
    const int lo = max(0, b1 - w), hi = min(nb - 1, b1 + w);
    const int m = hi - lo + 1;
    const int kkeep = max(1, static_cast<int>(ceil(rtab[d] * static_cast<double>(m))));
    for (int base = lo; base <= hi; base += 32) {
      const int b2 = base + lane;
      const bool cand = b2 <= hi;
      const int id = t2 * nb + b2;
      bool keep = cand;
      if (cand && mode == 1) {   // rank in the nearest-first order (distance, then lower b2)
        const int delta = b2 > b1 ? b2 - b1 : b1 - b2;
        int rank = 0;
        if (delta > 0) {
          rank = min(hi, b1 + delta - 1) - max(lo, b1 - delta + 1) + 1;
          if (b2 > b1 && b1 - delta >= lo) ++rank;
        }
        keep = rank < kkeep;
      } else if (cand && mode == 2) {
        const double *kr = mk + static_cast<size_t>(id) * D;
        double acc = 0.0;
#pragma unroll 8
        for (int e = 0; e < D; e += 2) {
          const double2 kv = __ldg(reinterpret_cast<const double2 *>(kr + e));
          acc = fma(qm[e], kv.x, acc);
          acc = fma(qm[e + 1], kv.y, acc);
        }
        const double proxy = acc * scale;
        keep = proxy >= theta;
        if (proxy > best || (proxy == best && id < best_id)) {
          best = proxy;
          best_id = id;
        }
      }
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      if (keep) out[pos + __popc(bal & ((1u << lane) - 1u))] = id;
      pos += __popc(bal);
    }
  }
  if (mode == 2 && pos == 0) {   // nothing reached theta: keep the top candidate
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, best_id, o);
      if (ob > best || (ob == best && oi < best_id)) {
        best = ob;
        best_id = oi;
      }
    }
    if (lane == 0) out[0] = best_id;
    pos = 1;
  }
  if (lane == 0) sel_count[static_cast<size_t>(h) * Cb + i] = pos;
}

inline size_t dynrad_select_smem(int frames, int D) {
  return static_cast<size_t>(frames) * sizeof(double) + static_cast<size_t>(D) * sizeof(double) +
         static_cast<size_t>(frames) * sizeof(int);
}

}  // namespace svg
