// Step a2: Spark-Reblock ("Spark-H3" news post, Spark-Reblock bullet;
// "MiniMax H3 Spark Attention (SM89)", "What it's doing under the hood").
//
// Queries are similar when their score patterns over the keys are similar;
// the metric is the Mahalanobis cosine under the opposite side's second
// moment. With M + eps*tr(M)/d*I = L L^T (Cholesky), u = L^T x turns that
// cosine into the plain cosine of u. The partitioner splits each group of g
// blocks along the top principal direction of its normalised whitened
// vectors (fixed 16 power iterations from the all-ones direction), ranking
// tokens by (projection, index) and sending the first 64*floor(g/2) left,
// until every leaf holds exactly 64 tokens (O(N log N) levels).
//
// Kernels, in launch order:
//   whiten_prep  : one CTA per head - regularise M, float64 Cholesky -> L (f32)
//   normalize    : one thread per token - u = L^T x (f32), u_hat = bf16(u/|u|)
//   tree_build   : node table (first block, g) per level; depends on nb only
//   init_idx     : identity token order
//   split_level  : one CTA per (node, head) per level - Gram of the group
//                  (mma.sync, float64 flush), covariance, float64 power
//                  iteration in registers, float64 projections, orientation,
//                  radix select of the cut, stable in-place partition
//   leaf_sort    : ascending original index inside every 64-token leaf -> perm
#include <math.h>

#include "gram.cuh"
#include "plan.h"

namespace spark {

constexpr double REG_EPS = 1e-6;   // relative diagonal jitter before the Cholesky factor
constexpr int POWER_ITERS = 16;

// ------------------------------------------------------------------ whitening factor
template <int D>
__global__ void __launch_bounds__(256)
whiten_prep_kernel(const double* __restrict__ M, float* __restrict__ Lout, int* status) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  double* A = reinterpret_cast<double*>(smem_raw);
  __shared__ double tr_sh;
  const int tid = threadIdx.x, bh = blockIdx.x;
  const double* Mb = M + (size_t)bh * D * D;
  for (int e = tid; e < D * D; e += blockDim.x) A[e] = Mb[e];
  __syncthreads();
  if (tid == 0) {
    double tr = 0.0;
    for (int i = 0; i < D; ++i) tr += A[i * D + i];
    tr_sh = tr;
  }
  __syncthreads();
  const double tr = tr_sh;
  float* L = Lout + (size_t)bh * D * D;
  if (tr == 0.0) {   // all-zero moment: whiten with the identity
    for (int e = tid; e < D * D; e += blockDim.x) L[e] = (e / D == e % D) ? 1.f : 0.f;
    return;
  }
  if (tid < D) A[tid * D + tid] += REG_EPS * (tr / D);
  __syncthreads();
  for (int j = 0; j < D; ++j) {
    if (tid == 0) {
      const double piv = A[j * D + j];
      if (!(piv > 0.0)) set_status(status, STATUS_BAD_PIVOT);
      A[j * D + j] = piv > 0.0 ? sqrt(piv) : 0.0;
    }
    __syncthreads();
    const double dj = A[j * D + j];
    for (int i = j + 1 + tid; i < D; i += blockDim.x) A[i * D + j] = dj > 0.0 ? A[i * D + j] / dj : 0.0;
    __syncthreads();
    const int m = D - j - 1;
    for (int e = tid; e < m * m; e += blockDim.x) {
      const int i = j + 1 + e / m, kk = j + 1 + e % m;
      if (kk <= i) A[i * D + kk] -= A[i * D + j] * A[kk * D + j];
    }
    __syncthreads();
  }
  for (int e = tid; e < D * D; e += blockDim.x) {
    const int i = e / D, j = e % D;
    L[e] = (j <= i) ? (float)A[e] : 0.f;
  }
}

// Output dims [Q*D/4, (Q+1)*D/4) of u = L^T x; L is lower triangular, so
// only inputs i >= Q*D/4 contribute. The inner loop is fully unrolled so the
// token's x stays in registers.
template <int D, int Q>
__device__ __forceinline__ void normalize_quarter(const uint32_t (&xr)[D / 2], const float* Ls, float* us,
                                                  int tid, double& nrm2) {
  for (int j4 = Q * (D / 16); j4 < (Q + 1) * (D / 16); ++j4) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int i = Q * (D / 4); i < D; ++i) {
      const float4 l = *reinterpret_cast<const float4*>(Ls + i * D + 4 * j4);
      const float xi = (i & 1) ? bf_hi(xr[i >> 1]) : bf_lo(xr[i >> 1]);
      a0 = fmaf(l.x, xi, a0); a1 = fmaf(l.y, xi, a1);
      a2 = fmaf(l.z, xi, a2); a3 = fmaf(l.w, xi, a3);
    }
    us[(4 * j4 + 0) * 256 + tid] = a0; us[(4 * j4 + 1) * 256 + tid] = a1;
    us[(4 * j4 + 2) * 256 + tid] = a2; us[(4 * j4 + 3) * 256 + tid] = a3;
    nrm2 += (double)a0 * a0 + (double)a1 * a1 + (double)a2 * a2 + (double)a3 * a3;
  }
}

// ------------------------------------------------------------------ normalised whitened tokens
// u_j = sum_{i >= j} L[i][j] x_i, u_hat = bf16(u / |u|). Thread = token.
template <int D>
__global__ void __launch_bounds__(256)
normalize_kernel(const uint16_t* __restrict__ X, const float* __restrict__ Lall, int N,
                 uint16_t* __restrict__ uhat) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* Ls = reinterpret_cast<float*>(smem_raw);       // [D][D]
  float* us = Ls + D * D;                                // [D][256]
  const int tid = threadIdx.x, bh = blockIdx.y;
  const float* L = Lall + (size_t)bh * D * D;
  for (int e = tid * 4; e < D * D; e += blockDim.x * 4)
    *reinterpret_cast<float4*>(Ls + e) = *reinterpret_cast<const float4*>(L + e);
  const long tok = (long)blockIdx.x * blockDim.x + tid;
  uint32_t xr[D / 2];
  if (tok < N) {
    const uint4* src = reinterpret_cast<const uint4*>(X + ((size_t)bh * N + tok) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      uint4 w = src[c];
      xr[4 * c + 0] = w.x; xr[4 * c + 1] = w.y; xr[4 * c + 2] = w.z; xr[4 * c + 3] = w.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < D / 2; ++c) xr[c] = 0u;
  }
  __syncthreads();
  double nrm2 = 0.0;
  normalize_quarter<D, 0>(xr, Ls, us, tid, nrm2);
  normalize_quarter<D, 1>(xr, Ls, us, tid, nrm2);
  normalize_quarter<D, 2>(xr, Ls, us, tid, nrm2);
  normalize_quarter<D, 3>(xr, Ls, us, tid, nrm2);
  if (tok >= N) return;
  const double nrm = sqrt(nrm2);
  const double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
  uint4* dst = reinterpret_cast<uint4*>(uhat + ((size_t)bh * N + tok) * D);
#pragma unroll 4
  for (int c = 0; c < D / 8; ++c) {
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int j = 8 * c + 2 * h;
      const uint16_t lo = __bfloat16_as_ushort(__double2bfloat16((double)us[j * 256 + tid] * inv));
      const uint16_t hi = __bfloat16_as_ushort(__double2bfloat16((double)us[(j + 1) * 256 + tid] * inv));
      w[h] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ------------------------------------------------------------------ tree table
// Nodes that split, level by level: (first block, g blocks). Same recursion
// as the host side make_plan() uses for the counts.
__global__ void tree_build_kernel(int nb, int2* nodes) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int count = 1, off = 0;
  nodes[0] = make_int2(0, nb);
  while (count > 0) {
    int nxt = 0;
    const int base = off + count;
    for (int i = 0; i < count; ++i) {
      const int2 nd = nodes[off + i];
      const int gl = nd.y / 2, gr = nd.y - nd.y / 2;
      if (gl >= 2) nodes[base + nxt++] = make_int2(nd.x, gl);
      if (gr >= 2) nodes[base + nxt++] = make_int2(nd.x + gl, gr);
    }
    off = base;
    count = nxt;
  }
}

__global__ void init_idx_kernel(int32_t* idx, int N, long total) {
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x)
    idx[i] = (int32_t)(i % N);
}

// ------------------------------------------------------------------ block-wide helpers
__device__ __forceinline__ int block_excl_scan_256(int flag, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  const int within = __popc(m & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(m);
  __syncthreads();
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int c = warp_tot[w];
    before += (w < warp) ? c : 0;
    tot += c;
  }
  __syncthreads();
  total = tot;
  return before + within;
}

// Radix select over 8-bit digits: finds the key of rank `rank` (1-based)
// among the n keys produced by getkey(i) whose high bits match. Keys are
// uint64 (digits from bit 56 down). All 256 threads must call it.
template <class GetKey>
__device__ uint64_t radix_select_u64(int n, int rank, int nbits, GetKey getkey, int* hist,
                                     int* sh_sel) {
  uint64_t prefix = 0, mask = 0;
  const int tid = threadIdx.x;
  for (int shift = nbits - 8; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) {
      const uint64_t k = getkey(i);
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255], 1);
    }
    __syncthreads();
    if (tid < 32) {
      int loc[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { loc[j] = hist[tid * 8 + j]; s += loc[j]; }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += t;
      }
      const int excl = incl - s;
      if (excl < rank && rank <= incl) {
        int c = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (c < rank && rank <= c + loc[j]) { sh_sel[0] = tid * 8 + j; sh_sel[1] = rank - c; }
          c += loc[j];
        }
      }
    }
    __syncthreads();
    prefix |= ((uint64_t)sh_sel[0]) << shift;
    mask |= ((uint64_t)255) << shift;
    rank = sh_sel[1];
    __syncthreads();
  }
  return prefix;
}

// ------------------------------------------------------------------ one split level
template <int D>
struct SplitSmem {
  using G = Gram<D>;
  static constexpr int STAGES = 3;
  static constexpr size_t acc_bytes = sizeof(double) * G::ACC * G::THREADS;   // also holds S
  static constexpr size_t tile_bytes = sizeof(uint16_t) * G::TILE * STAGES;
  static constexpr size_t bytes = acc_bytes + tile_bytes;
};

template <int D>
__global__ void __launch_bounds__(256, 1)
split_level_kernel(const uint16_t* __restrict__ uhat, int N, const int2* __restrict__ nodes,
                   int32_t* __restrict__ idx, double* __restrict__ pval, int32_t* __restrict__ pidx,
                   int* status) {
  using G = Gram<D>;
  using SM = SplitSmem<D>;
  constexpr int STAGES = SM::STAGES;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  double* acc64 = reinterpret_cast<double*>(smem_raw);
  uint16_t* tiles = reinterpret_cast<uint16_t*>(smem_raw + SM::acc_bytes);
  __shared__ double mus[D], vs[D], zs[D];
  __shared__ double red_d[8];
  __shared__ int red_i[8];
  __shared__ int hist[256];
  __shared__ int sh_sel[2];
  __shared__ int warp_tot[8];
  __shared__ double sh_scalar;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int2 node = nodes[blockIdx.x];
  const int bh = blockIdx.y;
  const int n = node.y * BLK, pos0 = node.x * BLK, nL = BLK * (node.y / 2);
  const int ntiles = node.y;
  const uint16_t* X = uhat + (size_t)bh * N * D;
  int32_t* ids = idx + (size_t)bh * N + pos0;
  double* pv = pval + (size_t)bh * N + pos0;
  int32_t* pi = pidx + (size_t)bh * N + pos0;

  // ---- phase 1: Gram matrix and column sums of the group
  for (int j = tid; j < G::ACC * G::THREADS; j += G::THREADS) acc64[j] = 0.0;
  float acc[G::ACC];
#pragma unroll
  for (int j = 0; j < G::ACC; ++j) acc[j] = 0.f;
  double csum = 0.0;
#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < ntiles) G::load_tile(tiles + s * G::TILE, X, ids + s * BLK, 0, tid);
    cp_async_commit();
  }
  for (int it = 0; it < ntiles; ++it) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    const int nxt = it + STAGES - 1;
    if (nxt < ntiles) G::load_tile(tiles + (nxt % STAGES) * G::TILE, X, ids + nxt * BLK, 0, tid);
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
  const double invn = 1.0 / (double)n;
  if (tid < D) mus[tid] = csum * invn;
  __syncthreads();

  // ---- phase 2: S = G/n - mu mu^T, written over the accumulators as a D x D matrix
  {
    double g[G::ACC];
#pragma unroll
    for (int j = 0; j < G::ACC; ++j) g[j] = acc64[j * G::THREADS + tid];
    __syncthreads();
#pragma unroll
    for (int j = 0; j < G::ACC; ++j) {
      int row, col;
      G::coord(j, warp, lane, row, col);
      acc64[row * D + col] = g[j] * invn - mus[row] * mus[col];
    }
  }
  __syncthreads();

  // ---- phase 3: power iteration v <- S v / |S v| (float64, S in registers)
  constexpr int RPT = D / 32, CPT = D / 8;
  const int rg = tid >> 3, cg = tid & 7;
  double Sr[RPT][CPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i)
#pragma unroll
    for (int j = 0; j < CPT; ++j) Sr[i][j] = acc64[(rg * RPT + i) * D + cg * CPT + j];
  if (tid < D) vs[tid] = 1.0 / sqrt((double)D);
  __syncthreads();
  for (int iter = 0; iter < POWER_ITERS; ++iter) {
    double z[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      double s = 0.0;
#pragma unroll
      for (int j = 0; j < CPT; ++j) s = fma(Sr[i][j], vs[cg * CPT + j], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      z[i] = s;
    }
    if (cg == 0) {
#pragma unroll
      for (int i = 0; i < RPT; ++i) zs[rg * RPT + i] = z[i];
    }
    __syncthreads();
    if (warp == 0) {
      double s = 0.0;
      for (int c = lane; c < D; c += 32) s = fma(zs[c], zs[c], s);
      s = warp_sum(s);
      if (lane == 0) sh_scalar = s;
    }
    __syncthreads();
    const double nrm = sqrt(sh_scalar);
    if (nrm == 0.0) {
      if (tid < D) vs[tid] = 0.0;
      __syncthreads();
      break;
    }
    if (tid < D) vs[tid] = zs[tid] / nrm;
    __syncthreads();
  }

  // ---- phase 4: projections p_i = v . (u_i - mu) (float64); best |p|, lowest index
  double best_abs = -1.0, best_p = 0.0;
  int best_id = 0x7fffffff;
  {
    constexpr int QD = D / 4;
    const int tok = tid >> 2, qd = tid & 3;
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
      if (s < ntiles) G::load_tile(tiles + s * G::TILE, X, ids + s * BLK, 0, tid);
      cp_async_commit();
    }
    for (int it = 0; it < ntiles; ++it) {
      cp_async_wait<STAGES - 2>();
      __syncthreads();
      const int nxt = it + STAGES - 1;
      if (nxt < ntiles) G::load_tile(tiles + (nxt % STAGES) * G::TILE, X, ids + nxt * BLK, 0, tid);
      cp_async_commit();
      const uint16_t* sm = tiles + (it % STAGES) * G::TILE;
      double s = 0.0;
#pragma unroll 8
      for (int j = qd * QD; j < (qd + 1) * QD; ++j)
        s = fma(vs[j], (double)bf2f(sm[tok * G::RS + j]) - mus[j], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (qd == 0) {
        const int pos = it * BLK + tok;
        const int id = ids[pos];
        pv[pos] = s;
        pi[pos] = id;
        const double a = fabs(s);
        if (a > best_abs || (a == best_abs && id < best_id)) { best_abs = a; best_p = s; best_id = id; }
      }
    }
    cp_async_wait<0>();
  }
  // block argmax of (|p|, -index)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double oa = __shfl_xor_sync(0xffffffffu, best_abs, o);
    const double op = __shfl_xor_sync(0xffffffffu, best_p, o);
    const int oi = __shfl_xor_sync(0xffffffffu, best_id, o);
    if (oa > best_abs || (oa == best_abs && oi < best_id)) { best_abs = oa; best_p = op; best_id = oi; }
  }
  if (lane == 0) { red_d[warp] = best_p; red_i[warp] = best_id; zs[warp] = best_abs; }
  __syncthreads();
  if (tid == 0) {
    double ba = zs[0], bp = red_d[0];
    int bi = red_i[0];
    for (int w = 1; w < 8; ++w) {
      if (zs[w] > ba || (zs[w] == ba && red_i[w] < bi)) { ba = zs[w]; bp = red_d[w]; bi = red_i[w]; }
    }
    sh_scalar = (bp < 0.0) ? -1.0 : 1.0;
  }
  __syncthreads();
  const double sgn = sh_scalar;

  // ---- phase 5: the cut - key of rank nL among (sgn * p) keys, then index ties
  auto pkey = [&](int i) -> uint64_t { return ordered_key(sgn * pv[i]); };
  const uint64_t kstar = radix_select_u64(n, nL, 64, pkey, hist, sh_sel);
  int c_less = 0, c_eq = 0;
  for (int i = tid; i < n; i += blockDim.x) {
    const uint64_t k = pkey(i);
    c_less += (k < kstar);
    c_eq += (k == kstar);
  }
  for (int o = 16; o > 0; o >>= 1) {
    c_less += __shfl_xor_sync(0xffffffffu, c_less, o);
    c_eq += __shfl_xor_sync(0xffffffffu, c_eq, o);
  }
  if (lane == 0) { red_i[warp] = c_less; warp_tot[warp] = c_eq; }
  __syncthreads();
  if (tid == 0) {
    int a = 0, b = 0;
    for (int w = 0; w < 8; ++w) { a += red_i[w]; b += warp_tot[w]; }
    sh_sel[0] = a;
    sh_sel[1] = b;
  }
  __syncthreads();
  const int need = nL - sh_sel[0];
  const int ties = sh_sel[1];
  __syncthreads();
  int32_t istar = 0x7fffffff;
  if (need < ties) {   // several tokens share the cut value: lowest indices go left
    auto ikey = [&](int i) -> uint64_t {
      return (pkey(i) == kstar) ? (uint64_t)(uint32_t)pi[i] : 0xffffffffull;
    };
    istar = (int32_t)radix_select_u64(n, need, 32, ikey, hist, sh_sel);
  }

  // ---- phase 6: stable partition, written in place over the group's indices
  int left_done = 0, right_done = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + tid;
    int goleft = 0;
    int32_t id = 0;
    if (i < n) {
      const uint64_t k = pkey(i);
      id = pi[i];
      goleft = (k < kstar) || (k == kstar && id <= istar);
    }
    int tot;
    const int lpos = block_excl_scan_256(goleft, warp_tot, tot);
    if (i < n) {
      const int dst = goleft ? left_done + lpos : nL + right_done + (tid - lpos);
      const bool in_side = goleft ? (dst < nL) : (dst < n);
      if (in_side) ids[dst] = id;
      else set_status(status, STATUS_BAD_INPUT);
    }
    left_done += tot;
    right_done += min((int)blockDim.x, n - base) - tot;
  }
}

// ------------------------------------------------------------------ leaves -> perm
__global__ void leaf_sort_kernel(const int32_t* __restrict__ idx, int32_t* __restrict__ perm,
                                 long nblocks_total) {
  __shared__ int32_t v[8][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long blk = (long)blockIdx.x * 8 + warp;
  if (blk >= nblocks_total) return;
  const int32_t* src = idx + blk * BLK;
  v[warp][lane] = src[lane];
  v[warp][lane + 32] = src[lane + 32];
  __syncwarp();
  const int32_t a = v[warp][lane], b = v[warp][lane + 32];
  int ra = 0, rb = 0;
  for (int j = 0; j < 64; ++j) {
    const int32_t w = v[warp][j];
    ra += (w < a);
    rb += (w < b);
  }
  perm[blk * BLK + ra] = a;
  perm[blk * BLK + rb] = b;
}

// ------------------------------------------------------------------ positional tiles
__global__ void positional_perm_kernel(int32_t* perm, int N, int Hl, int Wl, long total) {
  for (long g = (long)blockIdx.x * blockDim.x + threadIdx.x; g < total; g += (long)gridDim.x * blockDim.x) {
    const int pi = (int)(g % N);
    const int tile = pi / BLK, r = pi % BLK;
    const int nyt = Hl / 8, nxt = Wl / 4;
    const int xt = tile % nxt, yt = (tile / nxt) % nyt, ft = tile / (nxt * nyt);
    const int a = r / 32, b = (r / 4) % 8, c = r % 4;
    perm[g] = ((2 * ft + a) * Hl + 8 * yt + b) * Wl + 4 * xt + c;
  }
}

// ------------------------------------------------------------------ launcher
template <int D>
static cudaError_t run_reblock(const Plan& pl, const uint16_t* x, const double* M, int32_t* perm,
                               void* ws, int* status, cudaStream_t s) {
  float* L = ws_at<float>(ws, pl.off_L);
  uint16_t* uhat = ws_at<uint16_t>(ws, pl.off_uhat);
  int32_t* idx = ws_at<int32_t>(ws, pl.off_idx);
  double* pval = ws_at<double>(ws, pl.off_pval);
  int32_t* pidx = ws_at<int32_t>(ws, pl.off_pidx);
  int2* nodes = ws_at<int2>(ws, pl.off_nodes);
  cudaError_t e;

  const size_t smem_w = sizeof(double) * D * D;
  e = cudaFuncSetAttribute(whiten_prep_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_w);
  if (e != cudaSuccess) return e;
  whiten_prep_kernel<D><<<pl.BH, 256, smem_w, s>>>(M, L, status);

  const size_t smem_n = sizeof(float) * (D * D + D * 256);
  e = cudaFuncSetAttribute(normalize_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_n);
  if (e != cudaSuccess) return e;
  normalize_kernel<D><<<dim3((pl.N + 255) / 256, pl.BH), 256, smem_n, s>>>(x, L, pl.N, uhat);

  tree_build_kernel<<<1, 1, 0, s>>>(pl.nb, nodes);
  const long total = (long)pl.BH * pl.N;
  init_idx_kernel<<<(int)std::min<long>((total + 255) / 256, 4096), 256, 0, s>>>(idx, pl.N, total);

  const size_t smem_s = SplitSmem<D>::bytes;
  e = cudaFuncSetAttribute(split_level_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s);
  if (e != cudaSuccess) return e;
  for (int lv = 0; lv < pl.nlevels; ++lv) {
    split_level_kernel<D><<<dim3(pl.level_count[lv], pl.BH), 256, smem_s, s>>>(
        uhat, pl.N, nodes + pl.level_off[lv], idx, pval, pidx, status);
  }
  const long nbt = (long)pl.BH * pl.nb;
  leaf_sort_kernel<<<(int)((nbt + 7) / 8), 256, 0, s>>>(idx, perm, nbt);
  return cudaGetLastError();
}

cudaError_t launch_reblock(const Plan& pl, const uint16_t* x, const double* M, int32_t* perm,
                           void* ws, int* status, cudaStream_t s) {
  if (pl.d == 128) return run_reblock<128>(pl, x, M, perm, ws, status, s);
  return run_reblock<64>(pl, x, M, perm, ws, status, s);
}

cudaError_t launch_positional(const Plan& pl, int F, int Hl, int Wl, int32_t* perm, cudaStream_t s) {
  (void)F;
  const long total = (long)pl.BH * pl.N;
  positional_perm_kernel<<<(int)std::min<long>((total + 255) / 256, 4096), 256, 0, s>>>(perm, pl.N, Hl, Wl, total);
  return cudaGetLastError();
}

}  // namespace spark
