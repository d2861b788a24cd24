// Step a1: per-head second moments M_Q = E[q q^T], M_K = E[k k^T] and the
// anchor qbar = E[q] ("MiniMax H3 Spark Attention (SM89)", "What it's doing
// under the hood"; "Spark-H3" news post, Spark-Reweight bullet).
//
// The moment a partition whitens with decides, through its Cholesky factor,
// every bf16 rounding of the normalised whitened tokens, and one rounding that
// lands on the other side of a bf16 midpoint moves a token across a cut. So
// the Gram sums are float64 sums of exact products, as the plain definition
// (1/N) sum_t x_t x_t^T evaluates them: bf16 inputs widened to float64 and
// multiplied on the float64 tensor cores (dmma.cuh), never float32 partials.
//
// Kernel 1 (moments_gram64): grid (splits, B*H). Each CTA takes a contiguous
// range of 64-token tiles of one head, widens each tile to float64 in shared
// memory (double-buffered, the next tile's global loads in flight during the
// current tile's MMAs) and accumulates the upper-triangle tiles of X^T X in
// registers (72 of the 128 16x8 tiles for d = 128: five for warps 0-7 and
// four for warps 8-15, 18 per scheduler);
// with COLSUM also the exact float64 column sums. Kernel 1b
// (moments_colsum): the column sums alone, for the anchor when the query
// moment is not needed. Kernel 2
// (moments_reduce) adds a head's partials in a fixed order, mirrors the
// triangle and divides by N. The number of token chunks depends on N only, so
// a head's sums are the same whatever else shares the call.
#include "dmma.cuh"
#include "plan.h"

namespace spark {

constexpr int MOM_THREADS = 512;                      // 16 warps: four per scheduler keep the MMA pipe fed

template <int D>
struct MomSmem {
  static constexpr int TT = BLK;                      // tokens per tile
  static constexpr int LD = D + 4;                    // float64 row stride (conflict-free fragments)
  static constexpr int TILE = TT * LD;                // doubles per tile buffer
  static constexpr size_t bytes = sizeof(double) * 2 * TILE;
  static constexpr int CPT = TT * (D / 8) / MOM_THREADS;   // 16-byte chunks per thread and tile
};

template <int D, bool COLSUM>
__global__ void __launch_bounds__(MOM_THREADS, 1)
moments_gram64_kernel(const uint16_t* __restrict__ X, int N, int blocks_per_split, double* __restrict__ part) {
  using SM = MomSmem<D>;
  using TRI = TriTiles<D>;
  constexpr int LD = SM::LD;
  // PAIRS = NW * base + extra tiles: warps below `extra` take base + 1, the
  // rest base, so that every scheduler (warps w, w + 4, ...) gets the same
  // share (extra is a multiple of 4 for d = 64 and d = 128)
  constexpr int NW = MOM_THREADS / 32;
  constexpr int BASE = TRI::PAIRS / NW, EXTRA = TRI::PAIRS - BASE * NW;
  constexpr int SLOTS = BASE + (EXTRA > 0 ? 1 : 0);  // tiles per warp, at most
  static_assert(EXTRA % 4 == 0, "equal shares per scheduler");
  extern __shared__ __align__(16) double msm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int split = blockIdx.x, bh = blockIdx.y, splits = gridDim.x;
  const int nb = N / BLK;
  const int b0 = split * blocks_per_split, b1 = min(nb, b0 + blocks_per_split);
  const int ntiles = max(0, b1 - b0);
  const uint16_t* Xh = X + ((size_t)bh * N + (size_t)b0 * BLK) * D;

  int pr[SLOTS], pc[SLOTS];
  bool pv[SLOTS];
  const int first = warp * BASE + min(warp, EXTRA), count = BASE + (warp < EXTRA ? 1 : 0);
#pragma unroll
  for (int s = 0; s < SLOTS; ++s) {
    const int p = first + s;
    pv[s] = s < count;
    pr[s] = 0;
    pc[s] = 0;
    if (pv[s]) TRI::decode(p, pr[s], pc[s]);
  }
  double acc[SLOTS][4];
#pragma unroll
  for (int s = 0; s < SLOTS; ++s)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[s][e] = 0.0;
  double csum = 0.0;

  uint4 pre[SM::CPT];
  auto fetch = [&](int t) {
#pragma unroll
    for (int i = 0; i < SM::CPT; ++i) {
      const int c = tid + MOM_THREADS * i, r = c / (D / 8), ch = c % (D / 8);
      pre[i] = __ldg(reinterpret_cast<const uint4*>(Xh + ((size_t)t * BLK + r) * D + ch * 8));
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int i = 0; i < SM::CPT; ++i) {
      const int c = tid + MOM_THREADS * i, r = c / (D / 8), ch = c % (D / 8);
      bf8_to_f64(pre[i], msm + buf * SM::TILE + r * LD + ch * 8, lane);
    }
  };

  if (ntiles > 0) {
    fetch(0);
    stash(0);
  }
  __syncthreads();
  for (int it = 0; it < ntiles; ++it) {
    const double* xs = msm + (it & 1) * SM::TILE;
    if (it + 1 < ntiles) fetch(it + 1);
    if (COLSUM && tid < D) {
      double s = 0.0;
      for (int r = 0; r < BLK; ++r) s += xs[r * LD + tid];
      csum += s;
    }
#pragma unroll
    for (int ks = 0; ks < BLK / 16; ++ks) {
      const double* xk = xs + ks * 16 * LD;
      double a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = 0.0;
#pragma unroll
      for (int s = 0; s < SLOTS; ++s) {
        if (!pv[s]) continue;                          // warp-uniform
        if (s == 0 || pr[s] != pr[s - 1]) {
          // A = X^T on this row tile: a[i] = x[token t + 4 (i / 2)][dim 16 r + g + 8 (i % 2)]
#pragma unroll
          for (int i = 0; i < 8; ++i) a[i] = xk[(t4 + 4 * (i / 2)) * LD + 16 * pr[s] + g + 8 * (i % 2)];
        }
        double b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) b[i] = xk[(t4 + 4 * i) * LD + 8 * pc[s] + g];
        dmma16816(acc[s], a, b);
      }
    }
    if (it + 1 < ntiles) stash((it + 1) & 1);
    __syncthreads();
  }

  // upper triangle (row <= col) of this chunk's sums; the reduce mirrors it
  double* out = part + ((size_t)bh * splits + split) * (size_t)(D * D + D);
#pragma unroll
  for (int s = 0; s < SLOTS; ++s) {
    if (!pv[s]) continue;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int row = 16 * pr[s] + g + 8 * (e >> 1), col = 8 * pc[s] + 2 * t4 + (e & 1);
      if (row <= col) out[row * D + col] = acc[s][e];
    }
  }
  if (COLSUM && tid < D) out[D * D + tid] = csum;
}

// Column sums alone (same tiles, same order of additions as the COLSUM path
// of moments_gram64, so both give bit-identical anchors).
template <int D>
__global__ void __launch_bounds__(256)
moments_colsum_kernel(const uint16_t* __restrict__ X, int N, int blocks_per_split, double* __restrict__ part) {
  constexpr int CPT = BLK * (D / 8) / 256;
  __shared__ __align__(16) uint16_t ts[2][BLK * D];
  const int tid = threadIdx.x;
  const int split = blockIdx.x, bh = blockIdx.y, splits = gridDim.x;
  const int nb = N / BLK;
  const int b0 = split * blocks_per_split, b1 = min(nb, b0 + blocks_per_split);
  const int ntiles = max(0, b1 - b0);
  const uint16_t* Xh = X + ((size_t)bh * N + (size_t)b0 * BLK) * D;
  uint4 pre[CPT];
  auto fetch = [&](int t) {
#pragma unroll
    for (int i = 0; i < CPT; ++i)
      pre[i] = __ldg(reinterpret_cast<const uint4*>(Xh + (size_t)t * BLK * D) + tid + 256 * i);
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int i = 0; i < CPT; ++i) reinterpret_cast<uint4*>(ts[buf])[tid + 256 * i] = pre[i];
  };
  double csum = 0.0;
  if (ntiles > 0) {
    fetch(0);
    stash(0);
  }
  __syncthreads();
  for (int it = 0; it < ntiles; ++it) {
    if (it + 1 < ntiles) fetch(it + 1);
    if (tid < D) {
      const uint16_t* xs = ts[it & 1];
      double s = 0.0;
      for (int r = 0; r < BLK; ++r) s += (double)bf2f(xs[r * D + tid]);
      csum += s;
    }
    if (it + 1 < ntiles) stash((it + 1) & 1);
    __syncthreads();
  }
  if (tid < D) part[((size_t)bh * splits + split) * (size_t)(D * D + D) + D * D + tid] = csum;
}

// grid (B*H, 2 tensors, entry slices): tensor 0 = q (its moment if gram_mask
// bit 0, and the anchor), tensor 1 = k (its moment if gram_mask bit 1).
template <int D>
__global__ void moments_reduce_kernel(const double* __restrict__ part, int splits, int N, double* __restrict__ MQ,
                                      double* __restrict__ MK, double* __restrict__ qmean, int gram_mask) {
  const int bh = blockIdx.x, t = blockIdx.y, BH = gridDim.x;
  const bool gram = (gram_mask >> t) & 1;
  const double* src = part + (size_t)(t * BH + bh) * splits * (size_t)(D * D + D);
  double* M = (t == 0 ? MQ : MK) + (size_t)bh * D * D;
  const double dN = (double)N;
  const int e0 = gram ? 0 : D * D;                    // without the moment only the column sums
  for (int e = e0 + blockIdx.z * blockDim.x + threadIdx.x; e < D * D + D; e += gridDim.z * blockDim.x) {
    if (e < D * D) {
      if (!gram) continue;
      const int i = e / D, j = e % D;
      const int se = i <= j ? e : j * D + i;
      double s = 0.0;
      for (int c = 0; c < splits; ++c) s += src[(size_t)c * (D * D + D) + se];
      M[e] = s / dN;
    } else if (t == 0) {
      double s = 0.0;
      for (int c = 0; c < splits; ++c) s += src[(size_t)c * (D * D + D) + e];
      qmean[(size_t)bh * D + (e - D * D)] = s / dN;
    }
  }
}

template <int D>
static cudaError_t run_moments(const Plan& pl, const uint16_t* q, const uint16_t* k, double* MQ, double* MK,
                               double* qmean, double* part, int splits, bool gram_q, bool gram_k,
                               cudaStream_t s) {
  using SM = MomSmem<D>;
  const int bps = (pl.nb + splits - 1) / splits;
  const size_t tstride = (size_t)pl.BH * splits * (D * D + D);
  cudaError_t e;
  if (gram_q) {
    e = cudaFuncSetAttribute(moments_gram64_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SM::bytes);
    if (e != cudaSuccess) return e;
    moments_gram64_kernel<D, true><<<dim3(splits, pl.BH), MOM_THREADS, SM::bytes, s>>>(q, pl.N, bps, part);
  } else {
    moments_colsum_kernel<D><<<dim3(splits, pl.BH), 256, 0, s>>>(q, pl.N, bps, part);
  }
  if (gram_k) {
    e = cudaFuncSetAttribute(moments_gram64_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SM::bytes);
    if (e != cudaSuccess) return e;
    moments_gram64_kernel<D, false><<<dim3(splits, pl.BH), MOM_THREADS, SM::bytes, s>>>(k, pl.N, bps, part + tstride);
  }
  moments_reduce_kernel<D><<<dim3(pl.BH, 2, D / 8), 256, 0, s>>>(part, splits, pl.N, MQ, MK, qmean,
                                                                 (gram_q ? 1 : 0) | (gram_k ? 2 : 0));
  return cudaGetLastError();
}

cudaError_t launch_moments(const Plan& pl, const uint16_t* q, const uint16_t* k, double* MQ, double* MK,
                           double* qmean, void* ws, bool gram_q, bool gram_k, cudaStream_t s) {
  double* part = ws_at<double>(ws, pl.off_mpart);
  if (pl.d == 128) return run_moments<128>(pl, q, k, MQ, MK, qmean, part, pl.moment_splits, gram_q, gram_k, s);
  return run_moments<64>(pl, q, k, MQ, MK, qmean, part, pl.moment_splits, gram_q, gram_k, s);
}

}  // namespace spark

// ------------------------------------------------------------------ allocation-free variant
// spark_moments_noalloc: the same kernels as spark_moments, with the per-chunk
// partial sums kept in a fixed file-scope device array instead of the
// caller's workspace, for callers that cannot hand over or allocate device
// memory. The token range of a head may be cut into fewer chunks than
// spark_moments uses (so that every partial fits the array): the float64
// sums are then added in another order and can differ from spark_moments'
// in the last bits.
#include <mutex>

namespace spark {

constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)SPARK_NOALLOC_SCRATCH_BYTES;

// One copy per device that loads the library, alive until the process exits.
// Host code must not pass this name to a kernel: on the host it is only a
// stand-in symbol; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) double g_moment_scratch[NOALLOC_SCRATCH_BYTES / sizeof(double)];

static std::mutex g_scratch_mutex;

// Device address of g_moment_scratch on the current device, looked up on
// every call with that device current (cheap, and still right after a
// device reset has loaded the module again at another address).
static cudaError_t moment_scratch_address(double** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_moment_scratch);
  if (e != cudaSuccess) return e;
  *out = static_cast<double*>(p);
  return cudaSuccess;
}

}  // namespace spark

extern "C" spark_status spark_moments_noalloc(const spark_params* p, const void* q, const void* k,
                                              double* MQ, double* MK, double* qmean,
                                              cudaStream_t stream) {
  using namespace spark;
  const spark_status v = spark_validate(p);
  if (v != SPARK_OK) return v;
  Plan pl;
  make_plan(p, &pl);
  if (!q || !k || !MQ || !MK || !qmean) return SPARK_ERR_INVALID_ARG;
  if (((uintptr_t)q & 15u) != 0 || ((uintptr_t)k & 15u) != 0) return SPARK_ERR_INVALID_ARG;
  // every (head, tensor) needs at least one partial of d*d + d doubles
  const size_t per_partial = ((size_t)pl.d * pl.d + pl.d) * sizeof(double);
  const size_t fit = NOALLOC_SCRATCH_BYTES / per_partial;
  const size_t min_need = 2 * (size_t)pl.BH;
  if (min_need > fit) return SPARK_ERR_UNSUPPORTED;
  const int splits = (int)std::max<size_t>(1, std::min<size_t>((size_t)pl.moment_splits, fit / min_need));
  double* scratch = nullptr;
  if (moment_scratch_address(&scratch) != cudaSuccess) return SPARK_ERR_CUDA;
  const cudaError_t e =
      pl.d == 128 ? run_moments<128>(pl, (const uint16_t*)q, (const uint16_t*)k, MQ, MK, qmean, scratch, splits,
                                     true, true, stream)
                  : run_moments<64>(pl, (const uint16_t*)q, (const uint16_t*)k, MQ, MK, qmean, scratch, splits,
                                    true, true, stream);
  return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}
