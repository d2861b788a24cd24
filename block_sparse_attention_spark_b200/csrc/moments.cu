// Step a1: per-head second moments M_Q = E[q q^T], M_K = E[k k^T] and the
// anchor qbar = E[q] ("MiniMax H3 Spark Attention (SM89)", "What it's doing
// under the hood"; "Spark-H3" news post, Spark-Reweight bullet).
//
// Kernel 1 (moments_partial): grid (splits, B*H, 2 tensors). Each CTA streams
// a contiguous token range of one head through shared memory and forms the
// partial Gram X^T X plus the column sums, float64-accumulated: for d = 128
// on the tcgen05 tensor cores (gram_tc.cuh, exact float64 column sums), for
// d = 64 with mma.sync (3-stage cp.async pipeline, 16-byte loads). Kernel 2
// (moments_reduce) adds the partials of a head in a fixed order
// (deterministic) and divides by N.
#include "gram.cuh"
#include "gram_tc.cuh"
#include "plan.h"

namespace spark {

template <int D, int STAGES>
__global__ void __launch_bounds__(256, 1)
moments_partial_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, int N,
                       int blocks_per_split, double* __restrict__ part) {
  using G = Gram<D>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  double* acc64 = reinterpret_cast<double*>(smem_raw);
  uint16_t* tiles = reinterpret_cast<uint16_t*>(smem_raw + sizeof(double) * G::ACC * G::THREADS);
  __shared__ double colsum_sh[D];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, bh = blockIdx.y, t = blockIdx.z;
  const int BH = gridDim.y, splits = gridDim.x;
  const uint16_t* X = (t == 0 ? q : k) + (size_t)bh * N * D;
  const int nb = N / BLK;
  const int b0 = split * blocks_per_split;
  const int b1 = min(nb, b0 + blocks_per_split);
  const int ntiles = max(0, b1 - b0);

  for (int j = tid; j < G::ACC * G::THREADS; j += G::THREADS) acc64[j] = 0.0;
  float acc[G::ACC];
#pragma unroll
  for (int j = 0; j < G::ACC; ++j) acc[j] = 0.f;
  double csum = 0.0;

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < ntiles) G::load_tile(tiles + s * G::TILE, X, nullptr, (long)(b0 + s) * BLK, tid);
    cp_async_commit();
  }
  for (int it = 0; it < ntiles; ++it) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    const int nxt = it + STAGES - 1;
    if (nxt < ntiles) G::load_tile(tiles + (nxt % STAGES) * G::TILE, X, nullptr, (long)(b0 + nxt) * BLK, tid);
    cp_async_commit();
    const uint16_t* sm = tiles + (it % STAGES) * G::TILE;
    G::tile_mma(sm, acc, warp, lane);
    if (tid < D) {
      double s = 0.0;
#pragma unroll 8
      for (int r = 0; r < BLK; ++r) s += (double)bf2f(sm[r * G::RS + tid]);
      csum += s;
    }
    if ((it + 1) % G::FLUSH == 0 || it == ntiles - 1) G::flush(acc, acc64, tid);
  }
  cp_async_wait<0>();
  __syncthreads();

  double* out = part + ((size_t)(t * BH + bh) * splits + split) * (size_t)(D * D + D);
#pragma unroll 4
  for (int j = 0; j < G::ACC; ++j) {
    int row, col;
    G::coord(j, warp, lane, row, col);
    out[row * D + col] = acc64[j * G::THREADS + tid];
  }
  if (tid < D) out[D * D + tid] = csum;
  (void)colsum_sh;
}

template <int D>
__global__ void moments_reduce_kernel(const double* __restrict__ part, int splits, int N,
                                      double* __restrict__ MQ, double* __restrict__ MK,
                                      double* __restrict__ qmean) {
  const int bh = blockIdx.x, t = blockIdx.y, BH = gridDim.x;
  const double* src = part + (size_t)(t * BH + bh) * splits * (size_t)(D * D + D);
  double* M = (t == 0 ? MQ : MK) + (size_t)bh * D * D;
  const double invN = 1.0 / (double)N;
  for (int e = threadIdx.x; e < D * D + D; e += blockDim.x) {
    double s = 0.0;
    for (int i = 0; i < splits; ++i) s += src[(size_t)i * (D * D + D) + e];
    if (e < D * D) {
      M[e] = s * invN;
    } else if (t == 0) {
      qmean[(size_t)bh * D + (e - D * D)] = s * invN;
    }
  }
}

// d = 128: the same partial sums on the tcgen05 tensor cores (gram_tc.cuh).
__global__ void __launch_bounds__(tc::GT_THREADS, 1)
moments_partial_tc_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, int N,
                          int blocks_per_split, double* __restrict__ part, int* status) {
  constexpr int D = tc::GramTcLayout::D;
  const int split = blockIdx.x, bh = blockIdx.y, t = blockIdx.z;
  const int BH = gridDim.y, splits = gridDim.x;
  const uint16_t* X = (t == 0 ? q : k) + (size_t)bh * N * D;
  const int nb = N / BLK;
  const int b0 = split * blocks_per_split;
  const int b1 = min(nb, b0 + blocks_per_split);
  double* out = part + ((size_t)(t * BH + bh) * splits + split) * (size_t)(D * D + D);
  tc::gram_tc_body<true>(X, [=](int tt, int r) { return (b0 + tt) * BLK + r; }, max(0, b1 - b0), out, status);
}

template <int D>
static cudaError_t run_moments(const Plan& pl, const uint16_t* q, const uint16_t* k, double* MQ,
                               double* MK, double* qmean, void* ws, int* status, cudaStream_t s) {
  if constexpr (D == 128) {
    const int splits = pl.moment_splits;
    const int bps = (pl.nb + splits - 1) / splits;
    double* part = ws_at<double>(ws, pl.off_mpart);
    cudaError_t e = cudaFuncSetAttribute(moments_partial_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         tc::GramTcLayout::SMEM);
    if (e != cudaSuccess) return e;
    moments_partial_tc_kernel<<<dim3(splits, pl.BH, 2), tc::GT_THREADS, tc::GramTcLayout::SMEM, s>>>(q, k, pl.N, bps,
                                                                                                       part, status);
    moments_reduce_kernel<D><<<dim3(pl.BH, 2), 256, 0, s>>>(part, splits, pl.N, MQ, MK, qmean);
    return cudaGetLastError();
  }
  constexpr int STAGES = 3;
  using G = Gram<D>;
  const size_t smem = sizeof(double) * G::ACC * G::THREADS + sizeof(uint16_t) * G::TILE * STAGES;
  auto kern = moments_partial_kernel<D, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int splits = pl.moment_splits;
  const int bps = (pl.nb + splits - 1) / splits;
  double* part = ws_at<double>(ws, pl.off_mpart);
  kern<<<dim3(splits, pl.BH, 2), G::THREADS, smem, s>>>(q, k, pl.N, bps, part);
  moments_reduce_kernel<D><<<dim3(pl.BH, 2), 256, 0, s>>>(part, splits, pl.N, MQ, MK, qmean);
  return cudaGetLastError();
}

cudaError_t launch_moments(const Plan& pl, const uint16_t* q, const uint16_t* k, double* MQ,
                           double* MK, double* qmean, void* ws, int* status, cudaStream_t s) {
  if (pl.d == 128) return run_moments<128>(pl, q, k, MQ, MK, qmean, ws, status, s);
  return run_moments<64>(pl, q, k, MQ, MK, qmean, ws, status, s);
}

}  // namespace spark

// ------------------------------------------------------------------ allocation-free variant
// spark_moments_noalloc: the same two kernels, with the per-chunk partial
// sums kept in a fixed file-scope device array instead of the caller's
// workspace, for callers that cannot hand over or allocate device memory.
#include <mutex>

namespace spark {

constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)SPARK_NOALLOC_SCRATCH_BYTES;

// One copy per device that loads the library, alive until the process exits.
// Host code must not pass this name to a kernel: on the host it is only a
// stand-in symbol; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) double g_moment_scratch[NOALLOC_SCRATCH_BYTES / sizeof(double)];

constexpr int NOALLOC_MAX_DEVICES = 128;
static std::mutex g_scratch_mutex;
static double* g_scratch_addr[NOALLOC_MAX_DEVICES] = {};

// Device address of g_moment_scratch on the current device. Looked up once
// per device (on that device's first call) and cached.
static cudaError_t moment_scratch_address(double** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_moment_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<double*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

template <int D>
static cudaError_t run_moments_static(const Plan& pl, const uint16_t* q, const uint16_t* k, double* MQ,
                                      double* MK, double* qmean, double* part, int splits,
                                      cudaStream_t s) {
  constexpr int STAGES = 3;
  using G = Gram<D>;
  const size_t smem = sizeof(double) * G::ACC * G::THREADS + sizeof(uint16_t) * G::TILE * STAGES;
  auto kern = moments_partial_kernel<D, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int bps = (pl.nb + splits - 1) / splits;
  kern<<<dim3(splits, pl.BH, 2), G::THREADS, smem, s>>>(q, k, pl.N, bps, part);
  moments_reduce_kernel<D><<<dim3(pl.BH, 2), 256, 0, s>>>(part, splits, pl.N, MQ, MK, qmean);
  return cudaGetLastError();
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
      pl.d == 128 ? run_moments_static<128>(pl, (const uint16_t*)q, (const uint16_t*)k, MQ, MK, qmean,
                                            scratch, splits, stream)
                  : run_moments_static<64>(pl, (const uint16_t*)q, (const uint16_t*)k, MQ, MK, qmean,
                                           scratch, splits, stream);
  return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}
