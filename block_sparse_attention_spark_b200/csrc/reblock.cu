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
//   whiten_prep  : one CTA per head - regularise M, float64 Cholesky -> L (f64)
//   normalize64  : persistent CTAs over 16-token tiles - U = X L in float64 on
//                  the float64 tensor cores, u_hat = bf16(u/|u|) from the
//                  float64 quotient (the plain definition's value)
//   tree_build   : node table (first block, g) per level; depends on nb only
//   init_idx     : identity token order
//   big_gram / big_reduce / big_solve / big_project / big_select, per level above the
//                  subtree level - chunked Gram sums of the groups (tcgen05
//                  for d = 128, mma.sync for d = 64; float64 flush; right
//                  halves derived from the parent level),
//                  covariance and float64 power iteration in registers,
//                  float64 projections, orientation, radix select of the cut,
//                  stable partition of the group's index slice
//   subtree      : one CTA per group of at most SUB_BLOCKS blocks - all
//                  remaining splits of its subtree in shared memory
//   leaf_sort    : ascending original index inside every 64-token leaf -> perm
#include <math.h>

#include "dmma.cuh"
#include "gram.cuh"
#include "gram_tc.cuh"
#include "plan.h"

namespace spark {

constexpr double REG_EPS = 1e-6;   // relative diagonal jitter before the Cholesky factor
constexpr int NORM_EVERY = 4;      // power-iteration steps between rescalings of v

// ------------------------------------------------------------------ whitening factor
template <int D>
__global__ void __launch_bounds__(256)
whiten_prep_kernel(const double* __restrict__ M, double* __restrict__ Lout, int* status) {
  // A row-major with an odd row stride (D + 1 doubles): walking a column
  // then touches a different bank pair on every row
  constexpr int LDA = D + 1;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  double* A = reinterpret_cast<double*>(smem_raw);
  __shared__ double tr_sh;
  __shared__ double colj[D];                 // column j of the factor (conflict-free reads)
  const int tid = threadIdx.x, bh = blockIdx.x;
  const int warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
  const double* Mb = M + (size_t)bh * D * D;
  for (int e = tid; e < D * D; e += blockDim.x) A[(e / D) * LDA + e % D] = Mb[e];
  __syncthreads();
  if (tid == 0) {
    double tr = 0.0;
    for (int i = 0; i < D; ++i) tr += A[i * LDA + i];
    tr_sh = tr;
  }
  __syncthreads();
  const double tr = tr_sh;
  double* L = Lout + (size_t)bh * D * D;
  if (tr == 0.0) {   // all-zero moment: whiten with the identity
    for (int e = tid; e < D * D; e += blockDim.x) L[e] = (e / D == e % D) ? 1.0 : 0.0;
    return;
  }
  if (tid < D) A[tid * LDA + tid] += REG_EPS * (tr / D);
  __syncthreads();
  for (int j = 0; j < D; ++j) {
    if (tid == 0) {
      const double piv = A[j * LDA + j];
      if (!(piv > 0.0)) set_status(status, STATUS_BAD_PIVOT);
      A[j * LDA + j] = piv > 0.0 ? sqrt(piv) : 0.0;
    }
    __syncthreads();
    const double dj = A[j * LDA + j];
    for (int i = j + 1 + tid; i < D; i += blockDim.x) {
      const double l = dj > 0.0 ? A[i * LDA + j] / dj : 0.0;
      A[i * LDA + j] = l;
      colj[i] = l;
    }
    __syncthreads();
    // trailing update of the lower triangle: warp per row, lanes along it
    for (int i = j + 1 + warp; i < D; i += nwarps) {
      const double li = colj[i];
      for (int kk = j + 1 + lane; kk <= i; kk += 32) A[i * LDA + kk] -= li * colj[kk];
    }
    __syncthreads();
  }
  for (int e = tid; e < D * D; e += blockDim.x) {
    const int i = e / D, j = e % D;
    L[e] = (j <= i) ? A[i * LDA + j] : 0.0;
  }
}

// ------------------------------------------------------------------ normalised whitened tokens
// u_j = sum_{i >= j} L[i][j] x_i, u_hat = bf16(u / |u|), evaluated as the
// plain definition does: u in float64 (bf16 x widened, float64 factor,
// float64 tensor cores, dmma.cuh), |u| = sqrt of the float64 sum of squares,
// and each u_j / |u| rounded once to bf16 (nearest, ties to even). Up to
// float64 summation order this is the oracle's value, so u_hat, the vectors
// every later split reads, agrees bit for bit except where a quotient sits
// within a float64 rounding of a bf16 midpoint.
//
// The quotient: q = u_j * (1 / |u|) is within 3 float64 ulps of the IEEE
// quotient u_j / |u|. q is rounded to nearest float32, f, and f to nearest
// bf16. Rounding twice differs from rounding q once only when f lands
// exactly on a bf16 halfway point (low 16 bits 0x8000), and f lands there
// whenever q (or the IEEE quotient) is within half a float32 ulp of a
// halfway point, far more than 3 float64 ulps; so when f's low half is not
// 0x8000, bf16(f) is the bf16 of the IEEE quotient, and otherwise
// (practically never) the division is carried out and rounded once.
//
// Persistent CTAs, one per SM, each take a balanced contiguous range of the
// layer's (head, 16-token tile) items, in segments of one head: per segment
// the CTA loads that head's factor L into shared memory (float64), then its
// sixteen warps work in pairs, each pair on its own 16-token tiles: rows
// staged as bf16 through a pair-private cp.async double buffer, widened to
// float64 as the A fragments are read; each warp of the pair takes half of
// the tile's 8-column output tiles ({0, 3, 4, 7, ...} and {1, 2, 5, 6, ...}:
// 36 of the 72 16x8x16 products each, the k-chunks above the diagonal of L
// being skipped); the two halves of each row norm meet in shared memory
// behind a 64-thread named barrier, and the bf16 rows go back through the
// staging buffer just consumed. Four warps per scheduler keep the float64
// MMA pipe fed; CTA-wide barriers only around the loads of L.
template <int D>
struct NormSmem {
  static constexpr int LD = D + 4;                    // float64 row stride of L (conflict-free fragments)
  static constexpr int RS = D + 8;                    // bf16 row stride of a staged tile
  static constexpr int TOK = 16;                      // tokens per pair tile
  static constexpr int THREADS = 512;
  static constexpr int NP = THREADS / 64;             // warp pairs
  static constexpr int WTILE = TOK * RS;              // bf16 elements per staged tile
  static constexpr size_t off_x = sizeof(double) * D * LD;
  static constexpr size_t off_n = off_x + sizeof(uint16_t) * NP * 2 * WTILE;
  static constexpr size_t bytes = off_n + sizeof(double) * NP * 2 * TOK;   // row-norm halves [pair][half][token]
  static constexpr int CT = D / 8, KC = D / 16;
  static constexpr int CPW = CT / 2;                  // 8-column output tiles per warp
  static constexpr int CH = TOK * (D / 8) / 64;       // 16-byte chunks per thread of a pair and tile
};

// bf16 bits of u / r for a pair (u0, u1), low half u0; rinv = 1 / r.
__device__ __forceinline__ uint32_t bf16x2_of_quotients(double u0, double u1, double r, double rinv) {
  const float f0 = __double2float_rn(u0 * rinv), f1 = __double2float_rn(u1 * rinv);
  if (((__float_as_uint(f0) & 0xffffu) == 0x8000u) | ((__float_as_uint(f1) & 0xffffu) == 0x8000u)) {
    return (uint32_t)__bfloat16_as_ushort(__double2bfloat16(u0 / r)) |
           ((uint32_t)__bfloat16_as_ushort(__double2bfloat16(u1 / r)) << 16);
  }
  uint32_t w;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(f1), "f"(f0));
  return w;
}

template <int D>
__global__ void __launch_bounds__(NormSmem<D>::THREADS, 1)
normalize64_kernel(const uint16_t* __restrict__ X, const double* __restrict__ Lall, int N, int BH,
                   uint16_t* __restrict__ uhat) {
  using SM = NormSmem<D>;
  constexpr int LD = SM::LD, RS = SM::RS, TOK = SM::TOK, KC = SM::KC, CPW = SM::CPW, NP = SM::NP;
  extern __shared__ __align__(16) unsigned char nsm_raw[];
  double* Ls = reinterpret_cast<double*>(nsm_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int pw = warp >> 1, hh = warp & 1, ptid = tid & 63;
  uint16_t* Xw = reinterpret_cast<uint16_t*>(nsm_raw + SM::off_x) + pw * 2 * SM::WTILE;
  double* nsq = reinterpret_cast<double*>(nsm_raw + SM::off_n) + pw * 2 * TOK;
  auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(1 + pw) : "memory"); };
  // this warp's output tiles: (c % 4) in {0, 3} for the first warp of a pair, {1, 2} for the second
  int cs[CPW];
#pragma unroll
  for (int j = 0; j < CPW; ++j) cs[j] = 4 * (j >> 1) + ((j & 1) ? (hh ? 2 : 3) : (hh ? 1 : 0));
  const int ntile = N / TOK;
  const long items = (long)BH * ntile;
  const long i0 = items * blockIdx.x / gridDim.x, i1 = items * (blockIdx.x + 1) / gridDim.x;
  for (long seg = i0; seg < i1;) {
    const int bh = (int)(seg / ntile);
    const int c0 = (int)(seg - (long)bh * ntile);
    const int c1 = (int)min((long)ntile, (long)c0 + (i1 - seg));
    seg += c1 - c0;
    __syncthreads();                                   // every warp is done with the previous head's L
    {
      const double2* Lg = reinterpret_cast<const double2*>(Lall + (size_t)bh * D * D);
      for (int e = tid; e < D * D / 2; e += SM::THREADS) {
        const int i = (2 * e) / D, j = (2 * e) % D;
        *reinterpret_cast<double2*>(Ls + i * LD + j) = Lg[e];
      }
    }
    __syncthreads();
    const uint16_t* Xh = X + (size_t)bh * N * D;
    uint16_t* Uh = uhat + (size_t)bh * N * D;
    auto load = [&](int t, int buf) {
#pragma unroll
      for (int i = 0; i < SM::CH; ++i) {
        const int c = ptid + 64 * i, r = c / (D / 8), ch = c % (D / 8);
        cp_async16(Xw + buf * SM::WTILE + r * RS + ch * 8, Xh + ((size_t)t * TOK + r) * D + ch * 8);
      }
    };
    int t = c0 + pw, buf = 0;
    if (t < c1) load(t, 0);
    cp_async_commit();
    for (; t < c1; t += NP, buf ^= 1) {
      if (t + NP < c1) load(t + NP, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
      pair_sync();                                     // both warps' copies of this tile have landed
      uint16_t* xs = Xw + buf * SM::WTILE;
      double acc[CPW][4];
#pragma unroll
      for (int j = 0; j < CPW; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.0;
#pragma unroll
      for (int kc = 0; kc < KC; ++kc) {
        // A = the tile's tokens x dims 16 kc..: a[i] = x[g + 8 (i % 2)][16 kc + t + 4 (i / 2)]
        double a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = (double)bf2f(xs[(g + 8 * (i % 2)) * RS + 16 * kc + t4 + 4 * (i / 2)]);
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          if (kc < (cs[j] >> 1)) continue;             // L is zero above its diagonal (warp-uniform)
          double b[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) b[i] = Ls[(16 * kc + t4 + 4 * i) * LD + 8 * cs[j] + g];
          dmma16816(acc[j], a, b);
        }
      }
      // |u|^2 of tokens g and g + 8: this warp's columns, then the other half of the pair
      double s0 = 0.0, s1 = 0.0;
#pragma unroll
      for (int j = 0; j < CPW; ++j) {
        s0 = fma(acc[j][0], acc[j][0], s0);
        s0 = fma(acc[j][1], acc[j][1], s0);
        s1 = fma(acc[j][2], acc[j][2], s1);
        s1 = fma(acc[j][3], acc[j][3], s1);
      }
      s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
      s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
      if (t4 == 0) {
        nsq[hh * TOK + g] = s0;
        nsq[hh * TOK + g + 8] = s1;
      }
      pair_sync();                                     // both halves in place; both warps done with xs
      const double n0 = nsq[g] + nsq[TOK + g], n1 = nsq[g + 8] + nsq[TOK + g + 8];
      const double r0 = sqrt(n0), r1 = sqrt(n1);
      const double inv0 = r0 > 0.0 ? 1.0 / r0 : 0.0, inv1 = r1 > 0.0 ? 1.0 / r1 : 0.0;
      uint16_t* os = xs;
#pragma unroll
      for (int j = 0; j < CPW; ++j) {
        const int col = 8 * cs[j] + 2 * t4;
        const uint32_t w0 = r0 > 0.0 ? bf16x2_of_quotients(acc[j][0], acc[j][1], r0, inv0) : 0u;
        const uint32_t w1 = r1 > 0.0 ? bf16x2_of_quotients(acc[j][2], acc[j][3], r1, inv1) : 0u;
        *reinterpret_cast<uint32_t*>(os + g * RS + col) = w0;
        *reinterpret_cast<uint32_t*>(os + (g + 8) * RS + col) = w1;
      }
      pair_sync();                                     // the staged bf16 rows are complete
#pragma unroll
      for (int i = 0; i < SM::CH; ++i) {
        const int c = ptid + 64 * i, r = c / (D / 8), ch = c % (D / 8);
        *reinterpret_cast<uint4*>(Uh + ((size_t)t * TOK + r) * D + ch * 8) =
            *reinterpret_cast<const uint4*>(os + r * RS + ch * 8);
      }
      pair_sync();                                     // staging read and norms used: both may be reused
    }
    cp_async_wait<0>();
  }
}

// ------------------------------------------------------------------ tree table
// Nodes that split, level by level: (first block, g blocks). Same recursion
// as the host side make_plan() uses for the counts.
__global__ void tree_build_kernel(int nb, int2* nodes) {
  // one warp: each level's nodes in rounds of 32, every lane emitting the
  // children (0, 1 or 2) of one node, placed in node order by ballot counts
  if (blockIdx.x != 0 || threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  if (lane == 0) nodes[0] = make_int2(0, nb);
  __syncwarp();
  int count = 1, off = 0;
  while (count > 0) {
    const int base = off + count;
    int nxt = 0;
    for (int i0 = 0; i0 < count; i0 += 32) {
      const int i = i0 + lane;
      int2 nd = make_int2(0, 0);
      if (i < count) nd = nodes[off + i];
      const int gl = nd.y / 2, gr = nd.y - nd.y / 2;
      const bool el = i < count && gl >= 2, er = i < count && gr >= 2;
      const unsigned bl = __ballot_sync(0xffffffffu, el), br = __ballot_sync(0xffffffffu, er);
      const unsigned below = (1u << lane) - 1u;
      int pos = base + nxt + __popc(bl & below) + __popc(br & below);
      if (el) nodes[pos++] = make_int2(nd.x, gl);
      if (er) nodes[pos] = make_int2(nd.x + gl, gr);
      nxt += __popc(bl) + __popc(br);
    }
    __syncwarp();
    off = base;
    count = nxt;
  }
}

__global__ void init_idx_kernel(int32_t* idx, int N, long total) {
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x)
    idx[i] = (int32_t)(i % N);
}

// ------------------------------------------------------------------ block-wide helpers
// Exclusive prefix count of 0/1 flags over a block of NW warps (and the total).
template <int NW>
__device__ __forceinline__ int block_excl_scan(int flag, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  const int within = __popc(m & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(m);
  __syncthreads();
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int c = warp_tot[w];
    before += (w < warp) ? c : 0;
    tot += c;
  }
  __syncthreads();
  total = tot;
  return before + within;
}

// Exclusive prefix sum of per-thread counts over a block of NW warps (and the total).
template <int NW>
__device__ __forceinline__ int block_excl_sum(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int c = warp_tot[w];
    before += (w < warp) ? c : 0;
    tot += c;
  }
  __syncthreads();
  total = tot;
  return before + incl - v;
}

// Radix select over 8-bit digits: finds the key of rank `rank` (1-based)
// among the n keys produced by getkey(i) whose high bits match. Keys are
// uint64 (digits from bit 56 down). All 256 threads must call it. UNR keys
// per thread and pass are loaded before they are counted (several loads in
// flight for keys in global memory; 1 for keys in shared memory).
template <int UNR, class GetKey>
__device__ uint64_t radix_select_u64(int n, int rank, int nbits, GetKey getkey, int* hist,
                                     int* sh_sel, unsigned long long* sh_key) {
  uint64_t prefix = 0, mask = 0;
  const int tid = threadIdx.x;
  for (int shift = nbits - 8; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    // uniform trip count, UNR independent key loads per thread, then
    // warp-aggregated adds
    for (int i0 = 0; i0 < n; i0 += blockDim.x * UNR) {
      uint64_t kk[UNR];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int i = i0 + u * blockDim.x + tid;
        kk[u] = i < n ? getkey(i) : 0ull;
      }
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int i = i0 + u * blockDim.x + tid;
        const int bkt = (i < n && (kk[u] & mask) == prefix) ? (int)((kk[u] >> shift) & 255) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, bkt);
        if (bkt >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bkt], __popc(peers));
      }
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
          if (c < rank && rank <= c + loc[j]) { sh_sel[0] = tid * 8 + j; sh_sel[1] = rank - c; sh_sel[2] = loc[j]; }
          c += loc[j];
        }
      }
    }
    __syncthreads();
    prefix |= ((uint64_t)sh_sel[0]) << shift;
    mask |= ((uint64_t)255) << shift;
    rank = sh_sel[1];
    const int in_bucket = sh_sel[2];
    __syncthreads();
    if (in_bucket == 1 && shift > 0) {
      // a single key carries this prefix: it is the answer
#pragma unroll 4
      for (int i = tid; i < n; i += blockDim.x) {
        const uint64_t k = getkey(i);
        if ((k & mask) == prefix) *sh_key = k;
      }
      __syncthreads();
      const uint64_t r = *sh_key;
      __syncthreads();
      return r;
    }
  }
  return prefix;
}

// Power iteration v <- S v / |S v| (float64), iters steps (16 by default) from the
// all-ones direction; S is a D x D row-major matrix in shared memory (the
// buffer is reused as scratch afterwards). Thread (rg, cg) holds rows
// rg*RPT.. and columns cg*CPT.. of S in registers and its own copy of v on
// those columns; z goes through a padded, double-buffered shared array (one
// slot of padding per column group: conflict-free reads) and |z|^2 through
// per-warp partials, so a step needs one barrier. v is rescaled to unit
// length every NORM_EVERY steps and after the last one (the direction after
// iters steps is the same as with a rescale at every step). Writes v
// to vs.
template <int D>
__device__ void power_iterate_regs(const double (&Sr)[D / 32][D / 8], double* zb, double* vs, int iters);

template <int D>
__device__ void power_iterate(double* acc64, double* vs, int iters) {
  const int tid = threadIdx.x;
  constexpr int RPT = D / 32, CPT = D / 8;
  const int rg = tid >> 3, cg = tid & 7;
  double Sr[RPT][CPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i)
#pragma unroll
    for (int j = 0; j < CPT; ++j) Sr[i][j] = acc64[(rg * RPT + i) * D + cg * CPT + j];
  __syncthreads();                           // S has been copied to registers: acc64 becomes the z buffers
  power_iterate_regs<D>(Sr, acc64, vs, iters);
}

// The power iteration proper. Thread (rg, cg) = (tid / 8, tid % 8) holds rows
// rg*RPT.. and columns cg*CPT.. of S in Sr; zb: shared scratch of at least
// 2 * (D + D / CPT) + 16 doubles.
template <int D>
__device__ void power_iterate_regs(const double (&Sr)[D / 32][D / 8], double* zb, double* vs, int iters) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int RPT = D / 32, CPT = D / 8, ZP = D + D / CPT;
  const int rg = tid >> 3, cg = tid & 7;
  double vloc[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) vloc[j] = 1.0 / sqrt((double)D);
  auto zpad = [](int c) { return c + c / CPT; };
  bool zero_dir = false;
  double* nparts = zb + 2 * ZP;               // [2][8] per-warp partial |z|^2
  // v <- S v, scaled to unit length every NORM_EVERY steps and at the end:
  // scaling does not change the direction, and with |S| <= 1 (a covariance
  // of unit vectors) NORM_EVERY unscaled steps stay far from underflow
  for (int iter = 0; iter < iters; ++iter) {
    double* z = zb + (iter & 1) * ZP;
    const bool norm_step = (iter % NORM_EVERY) == NORM_EVERY - 1 || iter == iters - 1;
    double sq = 0.0;
    double zr[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) zr[i] = 0.0;
#pragma unroll
    for (int j = 0; j < CPT; ++j)
#pragma unroll
      for (int i = 0; i < RPT; ++i) zr[i] = fma(Sr[i][j], vloc[j], zr[i]);
#pragma unroll
    for (int o = 1; o <= 4; o <<= 1)
#pragma unroll
      for (int i = 0; i < RPT; ++i) zr[i] += __shfl_xor_sync(0xffffffffu, zr[i], o);
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      if (cg == 0) z[zpad(rg * RPT + i)] = zr[i];
      sq = fma(zr[i], zr[i], sq);
    }
    if (norm_step) {
      // lanes 0, 8, 16, 24 of each warp hold the warp's four row groups
      sq += __shfl_xor_sync(0xffffffffu, sq, 8);
      sq += __shfl_xor_sync(0xffffffffu, sq, 16);
      if (lane == 0) nparts[(iter & 1) * 8 + warp] = sq;
    }
    __syncthreads();
    double inv = 1.0;
    if (norm_step) {
      double pw[8];
#pragma unroll
      for (int w = 0; w < 8; ++w) pw[w] = nparts[(iter & 1) * 8 + w];
      const double nn = ((pw[0] + pw[1]) + (pw[2] + pw[3])) + ((pw[4] + pw[5]) + (pw[6] + pw[7]));
      if (nn == 0.0) { zero_dir = true; break; }   // uniform: every thread saw the same partials
      inv = rsqrt(nn);
    }
#pragma unroll
    for (int j = 0; j < CPT; ++j) vloc[j] = z[zpad(cg * CPT + j)] * inv;
  }
  if (zero_dir) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) vloc[j] = 0.0;
  }
  if (rg == 0) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) vs[cg * CPT + j] = vloc[j];
  }
  __syncthreads();

}

// The cut of one group: the key of rank nL among the (sgn * p, index) keys
// (block radix select on the ordered float64 projection, then index ties),
// then a stable partition: the nL smallest keys to positions 0..nL-1, the
// rest after them. pkey(i) / pid(i): ordered key and token index of member
// i; put(dst, i) moves member i to position dst. UNR: members per thread and
// pass (8 for keys in global memory, 1 for keys in shared memory).
template <int UNR, int NW, class KeyF, class IdF, class PutF>
__device__ void cut_partition(int n, int nL, KeyF pkey, IdF pid, PutF put, int* hist, int* sh_sel,
                              unsigned long long* sh_key, int* warp_tot, int* red_i, int* status) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint64_t kstar = radix_select_u64<UNR>(n, nL, 64, pkey, hist, sh_sel, sh_key);
  int c_less = 0, c_eq = 0;
#pragma unroll 8
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
    for (int w = 0; w < NW; ++w) { a += red_i[w]; b += warp_tot[w]; }
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
      return (pkey(i) == kstar) ? (uint64_t)(uint32_t)pid(i) : 0xffffffffull;
    };
    istar = (int32_t)radix_select_u64<UNR>(n, need, 32, ikey, hist, sh_sel, sh_key);
  }
  // stable partition: thread t takes UNR consecutive members per pass, one
  // block scan of the per-thread left counts places them
  int left_done = 0, right_done = 0;
  for (int base = 0; base < n; base += blockDim.x * UNR) {
    const int i0 = base + tid * UNR;
    bool gl[UNR];
    int cnt = 0;
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int i = i0 + u;
      gl[u] = false;
      if (i < n) {
        const uint64_t k = pkey(i);
        gl[u] = (k < kstar) || (k == kstar && pid(i) <= istar);
      }
      cnt += gl[u];
    }
    int tot;
    int l = UNR == 1 ? block_excl_scan<NW>(cnt, warp_tot, tot) : block_excl_sum<NW>(cnt, warp_tot, tot);
    int r = max(0, min(tid * UNR, n - base)) - l;              // members before this thread going right
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int i = i0 + u;
      if (i < n) {
        const int dst = gl[u] ? left_done + l++ : nL + right_done + r++;
        const bool in_side = gl[u] ? (dst < nL) : (dst < n);
        if (in_side) put(dst, i);
        else set_status(status, STATUS_BAD_INPUT);
      }
    }
    left_done += tot;
    right_done += min((int)blockDim.x * UNR, n - base) - tot;
  }
}

// The cut over a group's projections in global scratch (pv, pi), written
// over the group's index slice ids, by a block of NW warps.
template <int NW>
__device__ void cut_and_partition(int n, int nL, double sgn, const double* pv, const int32_t* pi,
                                  int32_t* ids, int* hist, int* sh_sel, unsigned long long* sh_key,
                                  int* warp_tot, int* red_i, int* status) {
  cut_partition<8, NW>(
      n, nL, [&](int i) -> uint64_t { return ordered_key(sgn * pv[i]); }, [&](int i) { return pi[i]; },
      [&](int dst, int i) { ids[dst] = pi[i]; }, hist, sh_sel, sh_key, warp_tot, red_i, status);
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

// ------------------------------------------------------------------ large groups over many CTAs
// Every level above the subtree level spreads a group over a grid of chunk
// CTAs (32 tiles each): partial Gram matrices (float64 sums of float32 tile
// sums), one CTA per group to reduce them and run the power iteration,
// chunk CTAs for the projections (with each chunk's best |p| candidate), and
// one CTA per group for orientation, cut and partition. When a level's
// groups are the two halves of each group one level up, only left halves
// get chunk Gram partials: a right half's Gram sum is its parent's (kept
// from the level above) minus its sibling's.
constexpr int BIG_CHUNK_TILES = 32;
constexpr int BIG_SELECT_WIDE_TOKENS = 8192;   // groups this large: 1024-thread select blocks

template <int D>
__global__ void __launch_bounds__(256, 1)
big_gram_kernel(const uint16_t* __restrict__ uhat, int N, const int2* __restrict__ nodes, int nnodes,
                int chunks, int kstep, const int32_t* __restrict__ idx, double* __restrict__ part) {
  using G = Gram<D>;
  using SM = SplitSmem<D>;
  constexpr int STAGES = SM::STAGES;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  double* acc64 = reinterpret_cast<double*>(smem_raw);
  uint16_t* tiles = reinterpret_cast<uint16_t*>(smem_raw + SM::acc_bytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, k = blockIdx.y * kstep, bh = blockIdx.z;
  const int2 node = nodes[k];
  const int t0 = c * BIG_CHUNK_TILES, t1 = min(node.y, t0 + BIG_CHUNK_TILES);
  const int ntiles = max(0, t1 - t0);
  const uint16_t* X = uhat + (size_t)bh * N * D;
  const int32_t* ids = idx + (size_t)bh * N + (size_t)node.x * BLK + (size_t)t0 * BLK;

  for (int j = tid; j < G::ACC * G::THREADS; j += G::THREADS) acc64[j] = 0.0;
  float acc[G::ACC];
#pragma unroll
  for (int j = 0; j < G::ACC; ++j) acc[j] = 0.f;
  double csum = 0.0;
#pragma unroll
  for (int st = 0; st < STAGES - 1; ++st) {
    if (st < ntiles) G::load_tile(tiles + st * G::TILE, X, ids + st * BLK, 0, tid);
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
    {
      constexpr int RSTEP = 256 / D;
      float c4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int r = tid / D, kk = 0; r < BLK; r += RSTEP, ++kk) c4[kk & 3] += bf2f(sm[r * G::RS + (tid % D)]);
      csum += (double)((c4[0] + c4[1]) + (c4[2] + c4[3]));
    }
    if ((it + 1) % G::FLUSH == 0 || it == ntiles - 1) G::flush(acc, acc64, tid);
  }
  cp_async_wait<0>();
  __syncthreads();
  double* out = part + ((size_t)(bh * nnodes + k) * chunks + c) * (size_t)(D * D + D);
#pragma unroll 4
  for (int j = 0; j < G::ACC; ++j) {
    int row, col;
    G::coord(j, warp, lane, row, col);
    out[row * D + col] = acc64[j * G::THREADS + tid];
  }
  double* cs = reinterpret_cast<double*>(tiles);
  cs[tid] = csum;
  __syncthreads();
  if (tid < D) {
    double t = 0.0;
    for (int kk = 0; kk < 256 / D; ++kk) t += cs[tid + kk * D];
    out[D * D + tid] = t;
  }
}

// d = 128: the chunk's Gram sums on the tcgen05 tensor cores (gram_tc.cuh);
// same output as big_gram_kernel.
__global__ void __launch_bounds__(tc::GT_THREADS, 1)
big_gram_tc_kernel(const uint16_t* __restrict__ uhat, int N, const int2* __restrict__ nodes, int nnodes,
                   int chunks, int kstep, const int32_t* __restrict__ idx, double* __restrict__ part, int* status) {
  constexpr int D = tc::GramTcLayout::D;
  const int c = blockIdx.x, k = blockIdx.y * kstep, bh = blockIdx.z;
  const int2 node = nodes[k];
  const int t0 = c * BIG_CHUNK_TILES, t1 = min(node.y, t0 + BIG_CHUNK_TILES);
  const uint16_t* X = uhat + (size_t)bh * N * D;
  const int32_t* ids = idx + (size_t)bh * N + (size_t)node.x * BLK + (size_t)t0 * BLK;
  double* out = part + ((size_t)(bh * nnodes + k) * chunks + c) * (size_t)(D * D + D);
  tc::gram_tc_body<false>(X, [=](int tt, int r) { return ids[tt * BLK + r]; }, max(0, t1 - t0), out, status);
}

// The chunk partials of each group that has them, summed in chunk order
// (c = 0, 1, ...) into chunk 0's slot: grid (entry slices, groups, heads),
// every entry owned by one thread, so the reads and the in-place write do
// not meet. big_solve then reads one Gram sum per group.
template <int D>
__global__ void __launch_bounds__(256)
big_reduce_kernel(const int2* __restrict__ nodes, int nnodes, int chunks, int kstep, double* __restrict__ part) {
  const int k = blockIdx.y * kstep, bh = blockIdx.z;
  const int used = (nodes[k].y + BIG_CHUNK_TILES - 1) / BIG_CHUNK_TILES;
  if (used <= 1) return;
  double* src = part + (size_t)(bh * nnodes + k) * chunks * (size_t)(D * D + D);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < D * D + D; e += gridDim.x * blockDim.x) {
    double t = 0.0;
    for (int c = 0; c < used; ++c) t += src[(size_t)c * (D * D + D) + e];
    src[e] = t;
  }
}

template <int D>
__global__ void __launch_bounds__(256, 1)
big_solve_kernel(const int2* __restrict__ nodes, int nnodes, int chunks, const double* __restrict__ part,
                 double* __restrict__ info, int derive, const double* __restrict__ gpar, int npar,
                 double* __restrict__ gout, int iters) {
  // The group's Gram sum G = sum u u^T and column sums: from its own chunk
  // partials, or (derive) a right child's as its parent's minus its left
  // sibling's, the parent's having been stored one level up. Stored again
  // (gout) when the next level derives from this one.
  constexpr int RPT = D / 32, CPT = D / 8;
  __shared__ double mus[D], vs[D];
  __shared__ double zbuf[2 * (D + D / CPT) + 16];
  const int tid = threadIdx.x, k = blockIdx.x, bh = blockIdx.y;
  const int2 node = nodes[k];
  const int n = node.y * BLK;
  const int ks = derive ? (k & ~1) : k;                    // node whose partials exist
  const bool right = derive && (k & 1);
  const int used = 1;                                      // big_reduce left the sum in chunk 0
  const double* src = part + (size_t)(bh * nnodes + ks) * chunks * (size_t)(D * D + D);
  const double* par = right ? gpar + (size_t)(bh * npar + (k >> 1)) * (size_t)(D * D + D) : nullptr;
  double* gsave = gout ? gout + (size_t)(bh * nnodes + k) * (size_t)(D * D + D) : nullptr;
  const double invn = 1.0 / (double)n;
  if (tid < D) {
    double t = 0.0;
    for (int c = 0; c < used; ++c) t += src[(size_t)c * (D * D + D) + D * D + tid];
    if (right) t = par[D * D + tid] - t;
    if (gsave) gsave[D * D + tid] = t;
    mus[tid] = t * invn;
  }
  __syncthreads();
  // each thread reads its own RPT x CPT block of G straight into the
  // power iteration's register layout (all loads in flight together)
  const int rg = tid >> 3, cg = tid & 7;
  double Sr[RPT][CPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i)
#pragma unroll
    for (int j = 0; j < CPT; ++j) Sr[i][j] = 0.0;
  for (int c = 0; c < used; ++c) {
    const double* pc = src + (size_t)c * (D * D + D);
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
      for (int j = 0; j < CPT; ++j) Sr[i][j] += pc[(rg * RPT + i) * D + cg * CPT + j];
  }
#pragma unroll
  for (int i = 0; i < RPT; ++i)
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int row = rg * RPT + i, col = cg * CPT + j;
      const double g = right ? par[row * D + col] - Sr[i][j] : Sr[i][j];
      if (gsave) gsave[row * D + col] = g;
      Sr[i][j] = g * invn - mus[row] * mus[col];
    }
  power_iterate_regs<D>(Sr, zbuf, vs, iters);
  double* out = info + (size_t)(bh * nnodes + k) * (D + 1);
  if (tid < D) out[tid] = vs[tid];
  if (tid < 32) {
    double vmu = 0.0;
    for (int j = tid; j < D; j += 32) vmu = fma(vs[j], mus[j], vmu);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmu += __shfl_xor_sync(0xffffffffu, vmu, o);
    if (tid == 0) out[D] = vmu;
  }
}

template <int D>
__global__ void __launch_bounds__(256)
big_project_kernel(const uint16_t* __restrict__ uhat, int N, const int2* __restrict__ nodes, int nnodes,
                   int chunks, const int32_t* __restrict__ idx, const double* __restrict__ info,
                   double* __restrict__ pval, int32_t* __restrict__ pidx, double* __restrict__ cand) {
  using G = Gram<D>;
  constexpr int STAGES = 3;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  uint16_t* tiles = reinterpret_cast<uint16_t*>(smem_raw);
  __shared__ double red_a[8], red_p[8];
  __shared__ int red_id[8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, k = blockIdx.y, bh = blockIdx.z;
  const int2 node = nodes[k];
  const int t0 = c * BIG_CHUNK_TILES, t1 = min(node.y, t0 + BIG_CHUNK_TILES);
  const int ntiles = max(0, t1 - t0);
  const uint16_t* X = uhat + (size_t)bh * N * D;
  const size_t gpos = (size_t)bh * N + (size_t)node.x * BLK + (size_t)t0 * BLK;
  const int32_t* ids = idx + gpos;
  const double* v = info + (size_t)(bh * nnodes + k) * (D + 1);
  constexpr int QD = D / 4;
  const int tok = tid >> 2, qd = tid & 3;
  double vr[QD];
#pragma unroll
  for (int j = 0; j < QD; ++j) vr[j] = v[qd * QD + j];
  const double vmu = v[D];
  double best_abs = -1.0, best_p = 0.0;
  int best_id = 0x7fffffff;
#pragma unroll
  for (int st = 0; st < STAGES - 1; ++st) {
    if (st < ntiles) G::load_tile(tiles + st * G::TILE, X, ids + st * BLK, 0, tid);
    cp_async_commit();
  }
  for (int it = 0; it < ntiles; ++it) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    const int nxt = it + STAGES - 1;
    if (nxt < ntiles) G::load_tile(tiles + (nxt % STAGES) * G::TILE, X, ids + nxt * BLK, 0, tid);
    cp_async_commit();
    const uint16_t* sm = tiles + (it % STAGES) * G::TILE;
    const uint4* rr = reinterpret_cast<const uint4*>(sm + tok * G::RS + qd * QD);
    double s4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int cc = 0; cc < QD / 8; ++cc) {
      const uint4 w = rr[cc];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s4[e] = fma(vr[8 * cc + 2 * e], (double)bf_lo(ws[e]), s4[e]);
        s4[e] = fma(vr[8 * cc + 2 * e + 1], (double)bf_hi(ws[e]), s4[e]);
      }
    }
    double sv = (s4[0] + s4[1]) + (s4[2] + s4[3]);
    sv += __shfl_xor_sync(0xffffffffu, sv, 1);
    sv += __shfl_xor_sync(0xffffffffu, sv, 2);
    sv -= vmu;
    if (qd == 0) {
      const int pos = it * BLK + tok;
      const int id = ids[pos];
      pval[gpos + pos] = sv;
      pidx[gpos + pos] = id;
      const double a = fabs(sv);
      if (a > best_abs || (a == best_abs && id < best_id)) { best_abs = a; best_p = sv; best_id = id; }
    }
  }
  cp_async_wait<0>();
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double oa = __shfl_xor_sync(0xffffffffu, best_abs, o);
    const double op = __shfl_xor_sync(0xffffffffu, best_p, o);
    const int oi = __shfl_xor_sync(0xffffffffu, best_id, o);
    if (oa > best_abs || (oa == best_abs && oi < best_id)) { best_abs = oa; best_p = op; best_id = oi; }
  }
  if (lane == 0) { red_a[warp] = best_abs; red_p[warp] = best_p; red_id[warp] = best_id; }
  __syncthreads();
  if (tid == 0) {
    double ba = red_a[0], bp = red_p[0];
    int bi = red_id[0];
    for (int w = 1; w < 8; ++w)
      if (red_a[w] > ba || (red_a[w] == ba && red_id[w] < bi)) { ba = red_a[w]; bp = red_p[w]; bi = red_id[w]; }
    double* o = cand + ((size_t)(bh * nnodes + k) * chunks + c) * 3;
    o[0] = ba;
    o[1] = bp;
    o[2] = (double)bi;
  }
}

// THREADS = 1024 for the levels with large groups (the select and partition
// passes are latency-bound loops over the group's keys), 256 below; the cut
// and the stable order do not depend on it.
template <int THREADS>
__global__ void __launch_bounds__(THREADS)
big_select_kernel(int N, const int2* __restrict__ nodes, int nnodes, int chunks, const double* __restrict__ cand,
                  int32_t* __restrict__ idx, const double* __restrict__ pval, const int32_t* __restrict__ pidx,
                  int* status) {
  constexpr int NW = THREADS / 32;
  __shared__ int hist[256];
  __shared__ int sh_sel[3];
  __shared__ unsigned long long sh_key;
  __shared__ int warp_tot[NW];
  __shared__ int red_i[NW];
  __shared__ double sh_sgn;
  const int tid = threadIdx.x, k = blockIdx.x, bh = blockIdx.y;
  const int2 node = nodes[k];
  const int n = node.y * BLK, nL = BLK * (node.y / 2);
  const int used = (node.y + BIG_CHUNK_TILES - 1) / BIG_CHUNK_TILES;
  if (tid == 0) {
    const double* cd = cand + (size_t)(bh * nnodes + k) * chunks * 3;
    double ba = -1.0, bp = 0.0;
    double bi = 4.0e9;
    for (int c = 0; c < used; ++c) {
      const double a = cd[3 * c], pp = cd[3 * c + 1], id = cd[3 * c + 2];
      if (a > ba || (a == ba && id < bi)) { ba = a; bp = pp; bi = id; }
    }
    sh_sgn = (bp < 0.0) ? -1.0 : 1.0;
  }
  __syncthreads();
  const size_t gpos = (size_t)bh * N + (size_t)node.x * BLK;
  cut_and_partition<NW>(n, nL, sh_sgn, pval + gpos, pidx + gpos, idx + gpos, hist, sh_sel, &sh_key, warp_tot,
                        red_i, status);
}

// ------------------------------------------------------------------ whole small subtrees
// One CTA per node of at most SUB_BLOCKS blocks at the first level where all
// nodes are that small: the node's normalised whitened rows are staged in
// shared memory once and every remaining split of its subtree is done
// on-chip (same split rule as the chunked levels): Gram by mma.sync with
// per-lane gathered ldmatrix rows, float64 covariance and power iteration in
// the MMA fragment layout, float64 projections, orientation, and the cut by
// exact ranks of (projection, index) - the node's slice of the local order
// is rewritten in ascending rank, so children are contiguous slices.
constexpr int SUB_BLOCKS = 9;
constexpr bool SUB_PAIR = true;   // two groups of a level share one power iteration

template <int D>
struct SubSmem {
  static constexpr int RS = D + 8;                       // padded row (elements): conflict-free ldmatrix
  static constexpr int TMAX = SUB_BLOCKS * BLK;
  static constexpr size_t off_rows = 0;
  static constexpr size_t off_pv = off_rows + sizeof(uint16_t) * TMAX * RS;
  static constexpr size_t off_ids = off_pv + sizeof(double) * TMAX;
  static constexpr size_t off_loc = off_ids + sizeof(int32_t) * TMAX;
  static constexpr size_t off_stok = off_loc + sizeof(uint16_t) * TMAX;   // partition target
  static constexpr size_t off_zp = (off_stok + sizeof(uint16_t) * TMAX + 15) & ~(size_t)15;
  static constexpr size_t zp_bytes = sizeof(double) * 2 * 2 * D > sizeof(int32_t) * TMAX ? sizeof(double) * 2 * 2 * D : sizeof(int32_t) * TMAX;
  static constexpr size_t bytes = off_zp + (zp_bytes > sizeof(double) * 256 ? zp_bytes : sizeof(double) * 256);
};

// One split of a subtree group, in three phases so that two groups of the
// same level can share the latency-bound power iteration:
//   sub_cov    : Gram of the group (float32 over at most SUB_BLOCKS tiles),
//                column means (float64, into mus), covariance S in this
//                thread's fragment entries (formed in float64, kept in float32)
//   sub_power  : float32 power iteration of one or two groups' S, one barrier
//                per step for both; v into vs (float64)
//   sub_finish : float64 projections, orientation, the cut, the group's slice
//                of the local order rewritten left child first
template <int D>
__device__ void sub_cov(const uint16_t* rows, const uint16_t* loc, double* zp, double* mus, int s0, int nn,
                        float (&S)[Gram<D>::ACC]) {
  using G = Gram<D>;
  using SM = SubSmem<D>;
  constexpr int RS = SM::RS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp % 4, wn = warp / 4;
  const int m0 = wm * G::WM, n0 = wn * G::WN;
  const int ntiles = nn / BLK;
  const uint16_t* lo = loc + s0;

  // Gram of the node (float32 over at most SUB_BLOCKS tiles) and column sums
  float acc[G::ACC];
#pragma unroll
  for (int j = 0; j < G::ACC; ++j) acc[j] = 0.f;
  for (int t = 0; t < ntiles; ++t) {
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const int t0 = t * BLK + ks * 16;
      uint32_t a[G::MT][4];
      const uint16_t* ra = rows + (size_t)lo[t0 + (lane & 7) + (lane >> 4) * 8] * RS;
#pragma unroll
      for (int mt = 0; mt < G::MT; ++mt)
        ldsm_x4_t(a[mt][0], a[mt][1], a[mt][2], a[mt][3], ra + m0 + mt * 16 + ((lane >> 3) & 1) * 8);
      const uint16_t* rb = rows + (size_t)lo[t0 + (lane & 7) + ((lane >> 3) & 1) * 8] * RS;
#pragma unroll
      for (int np = 0; np < G::NT / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, rb + n0 + np * 16 + (lane >> 4) * 8);
#pragma unroll
        for (int mt = 0; mt < G::MT; ++mt) {
          mma_bf16(&acc[(mt * G::NT + 2 * np) * 4], a[mt], b0, b1);
          mma_bf16(&acc[(mt * G::NT + 2 * np + 1) * 4], a[mt], b2, b3);
        }
      }
    }
  }
  {
    // column sums: thread = 8 columns (one 16-byte load per row) x every
    // RG-th token; the row groups of a warp are folded by shuffles, the
    // warps' float partials by one float64 pass
    constexpr int CG = D / 8, RG = 256 / CG;
    const int cg = tid % CG, rg = tid / CG;
    float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int t = rg; t < nn; t += RG) {
      const uint4 w = *reinterpret_cast<const uint4*>(rows + (size_t)lo[t] * RS + cg * 8);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        a8[2 * e] += bf_lo(ws[e]);
        a8[2 * e + 1] += bf_hi(ws[e]);
      }
    }
#pragma unroll
    for (int o = CG; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) a8[e] += __shfl_xor_sync(0xffffffffu, a8[e], o);
    float* cs = reinterpret_cast<float*>(zp);   // [8 warps][D] scratch before the power iteration uses it
    if (lane < CG) {
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[warp * D + cg * 8 + e] = a8[e];
    }
    __syncthreads();
    if (tid < D) {
      double t = 0.0;
      for (int w = 0; w < 8; ++w) t += (double)cs[w * D + tid];
      mus[tid] = t / (double)nn;
    }
  }
  __syncthreads();
  // S = G / n - mu mu^T on this thread's fragment entries, formed in float64
  // and kept in float32: a subtree's groups are small and its Gram sums are
  // float32 already, and float32 steps halve the latency-bound iteration
  const double invn = 1.0 / (double)nn;
#pragma unroll
  for (int j = 0; j < G::ACC; ++j) {
    int row, col;
    G::coord(j, warp, lane, row, col);
    S[j] = (float)((double)acc[j] * invn - mus[row] * mus[col]);
  }
}

template <int D, bool PAIR>
__device__ void sub_power(const float (&SA)[Gram<D>::ACC], const float (&SB)[Gram<D>::ACC], double* zp, double* vsA,
                          double* vsB, int iters) {
  // the direction is scale-free, so rescaling v by an approximate norm every
  // NORM_EVERY_F32 steps changes nothing; two unscaled float32 steps stay far
  // from underflow for any nonzero covariance of distinct bf16 unit vectors.
  // A group whose S v vanishes keeps v = 0 (its norm step sets the scale to 0).
  using G = Gram<D>;
  constexpr int NORM_EVERY_F32 = 2;
  constexpr int NG = PAIR ? 2 : 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp % 4, wn = warp / 4;
  const int m0 = wm * G::WM, n0 = wn * G::WN;
  (void)tid;
  // rows m0 + mt*16 + lane/4 + 8h, columns n0 + nt*8 + 2 (lane % 4) + e
  float vl[NG][G::NT * 2];
#pragma unroll
  for (int q = 0; q < NG; ++q)
#pragma unroll
    for (int j = 0; j < G::NT * 2; ++j) vl[q][j] = 1.0f;
  bool zero_dir[NG];
#pragma unroll
  for (int q = 0; q < NG; ++q) zero_dir[q] = false;
  float* zpf = reinterpret_cast<float*>(zp);
  for (int iter = 0; iter < iters; ++iter) {
    float* zb = zpf + (iter & 1) * 2 * NG * D;        // [group][wn][row]: the two column halves' partial sums
    const bool norm_step = (iter % NORM_EVERY_F32) == NORM_EVERY_F32 - 1 || iter == iters - 1;
    float zr[NG][G::MT][2];
#pragma unroll
    for (int q = 0; q < NG; ++q)
#pragma unroll
      for (int mt = 0; mt < G::MT; ++mt) { zr[q][mt][0] = 0.f; zr[q][mt][1] = 0.f; }
#pragma unroll
    for (int nt = 0; nt < G::NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int mt = 0; mt < G::MT; ++mt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            zr[0][mt][h] = fmaf(SA[(mt * G::NT + nt) * 4 + 2 * h + e], vl[0][nt * 2 + e], zr[0][mt][h]);
            if (PAIR) zr[NG - 1][mt][h] = fmaf(SB[(mt * G::NT + nt) * 4 + 2 * h + e], vl[NG - 1][nt * 2 + e], zr[NG - 1][mt][h]);
          }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1)
#pragma unroll
      for (int q = 0; q < NG; ++q)
#pragma unroll
        for (int mt = 0; mt < G::MT; ++mt)
#pragma unroll
          for (int h = 0; h < 2; ++h) zr[q][mt][h] += __shfl_xor_sync(0xffffffffu, zr[q][mt][h], o);
    if ((lane & 3) == 0) {
#pragma unroll
      for (int q = 0; q < NG; ++q)
#pragma unroll
        for (int mt = 0; mt < G::MT; ++mt)
#pragma unroll
          for (int h = 0; h < 2; ++h) zb[(q * 2 + wn) * D + m0 + mt * 16 + (lane >> 2) + 8 * h] = zr[q][mt][h];
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      const float* z = zb + q * 2 * D;
      float inv = 1.f;
      if (norm_step) {
        // every warp forms |z|^2 itself, in the same order: no second barrier
        float sq = 0.f;
#pragma unroll
        for (int k = 0; k < D / 32; ++k) {
          const float zz = z[lane + 32 * k] + z[D + lane + 32 * k];
          sq = fmaf(zz, zz, sq);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (sq == 0.f) zero_dir[q] = true;
        inv = zero_dir[q] ? 0.f : rsqrtf(sq);
      }
#pragma unroll
      for (int nt = 0; nt < G::NT; ++nt) {
        const float2 za = *reinterpret_cast<const float2*>(z + n0 + nt * 8 + 2 * (lane & 3));
        const float2 zc = *reinterpret_cast<const float2*>(z + D + n0 + nt * 8 + 2 * (lane & 3));
        vl[q][nt * 2] = (za.x + zc.x) * inv;
        vl[q][nt * 2 + 1] = (za.y + zc.y) * inv;
      }
    }
  }
  if (wm == 0 && lane < 4) {
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      double* vs = q == 0 ? vsA : vsB;
#pragma unroll
      for (int nt = 0; nt < G::NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) vs[n0 + nt * 8 + 2 * lane + e] = zero_dir[q] ? 0.0 : (double)vl[q][nt * 2 + e];
    }
  }
  __syncthreads();
}

template <int D>
__device__ void sub_finish(const uint16_t* rows, double* pv, const int32_t* ids, uint16_t* loc, uint16_t* stok,
                           double* zp, const double* mus, const double* vs, double* red_d, int* red_i,
                           double* sh_sgn, int* hist, int* sh_sel, unsigned long long* sh_key, int* warp_tot,
                           int* status, int s0, int nn) {
  using SM = SubSmem<D>;
  constexpr int RS = SM::RS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint16_t* lo = loc + s0;
  // projections p_t = v . (u_t - mu), float64; best |p| (lowest index on ties)
  double best_abs = -1.0, best_p = 0.0;
  int best_id = 0x7fffffff;
  {
    constexpr int QD = D / 4;
    const int tk = tid >> 2, qd = tid & 3;
    double vr[QD];
#pragma unroll
    for (int j = 0; j < QD; ++j) vr[j] = vs[qd * QD + j];
    double vmu = 0.0;                                   // v . mu, the same order in every warp
    for (int j = lane; j < D; j += 32) vmu = fma(vs[j], mus[j], vmu);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmu += __shfl_xor_sync(0xffffffffu, vmu, o);
    // two tokens per thread and pass (independent float64 chains)
    for (int b0 = 0; b0 < nn; b0 += 128) {
      const bool two = b0 + 64 < nn;                  // nn is a multiple of 64: uniform
      double sacc[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int t = b0 + 64 * u + tk;
        double s4[4] = {0.0, 0.0, 0.0, 0.0};
        if (u == 0 || two) {
          const uint4* rr = reinterpret_cast<const uint4*>(rows + (size_t)lo[t] * RS + qd * QD);
#pragma unroll
          for (int c = 0; c < QD / 8; ++c) {
            const uint4 w = rr[c];
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              s4[e] = fma(vr[8 * c + 2 * e], (double)bf_lo(ws[e]), s4[e]);
              s4[e] = fma(vr[8 * c + 2 * e + 1], (double)bf_hi(ws[e]), s4[e]);
            }
          }
        }
        sacc[u] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        sacc[u] += __shfl_xor_sync(0xffffffffu, sacc[u], 1);
        sacc[u] += __shfl_xor_sync(0xffffffffu, sacc[u], 2);
        sacc[u] -= vmu;
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int t = b0 + 64 * u + tk;
        if (qd == 0 && (u == 0 || two)) {
          pv[t] = sacc[u];
          const int id = ids[lo[t]];
          const double a = fabs(sacc[u]);
          if (a > best_abs || (a == best_abs && id < best_id)) { best_abs = a; best_p = sacc[u]; best_id = id; }
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double oa = __shfl_xor_sync(0xffffffffu, best_abs, o);
    const double op = __shfl_xor_sync(0xffffffffu, best_p, o);
    const int oi = __shfl_xor_sync(0xffffffffu, best_id, o);
    if (oa > best_abs || (oa == best_abs && oi < best_id)) { best_abs = oa; best_p = op; best_id = oi; }
  }
  if (lane == 0) { red_d[warp] = best_abs; red_d[8 + warp] = best_p; red_i[warp] = best_id; }
  __syncthreads();
  if (tid == 0) {
    double ba = red_d[0], bp = red_d[8];
    int bi = red_i[0];
    for (int w = 1; w < 8; ++w) {
      if (red_d[w] > ba || (red_d[w] == ba && red_i[w] < bi)) { ba = red_d[w]; bp = red_d[8 + w]; bi = red_i[w]; }
    }
    *sh_sgn = (bp < 0.0) ? -1.0 : 1.0;
  }
  __syncthreads();
  const double sgn = *sh_sgn;
  // the cut: the nL smallest (sgn * p, index) keys become the left child's
  // slice, the rest the right child's (order inside a child is irrelevant:
  // it is cut again, and leaves are sorted by index at the end)
  const int nL = BLK * ((nn / BLK) / 2);
  if (nn <= 256) {
    // at most one member per thread: its rank among the unique (key, index)
    // pairs is its position, so the nL smallest come first (no select passes)
    uint64_t* kv = reinterpret_cast<uint64_t*>(pv);
    int* kid = reinterpret_cast<int*>(zp);
    uint64_t mykey = 0;
    int myid = 0;
    if (tid < nn) {
      mykey = ordered_key(sgn * pv[tid]);
      myid = ids[lo[tid]];
    }
    __syncthreads();                                   // pv is read as doubles above
    if (tid < nn) {
      kv[tid] = mykey;
      kid[tid] = myid;
    }
    __syncthreads();
    if (tid < nn) {
      int rank = 0;
      for (int u = 0; u < nn; ++u) {
        const uint64_t k = kv[u];
        rank += (k < mykey) | ((k == mykey) & (kid[u] < myid));
      }
      stok[rank] = lo[tid];
    }
  } else {
    cut_partition<1, 8>(
        nn, nL, [&](int t) -> uint64_t { return ordered_key(sgn * pv[t]); }, [&](int t) { return ids[lo[t]]; },
        [&](int dst, int t) { stok[dst] = lo[t]; }, hist, sh_sel, sh_key, warp_tot, red_i, status);
  }
  __syncthreads();
  for (int t = tid; t < nn; t += blockDim.x) loc[s0 + t] = stok[t];
  __syncthreads();
}

template <int D>
__global__ void __launch_bounds__(256, 1)
subtree_kernel(const uint16_t* __restrict__ uhat, int N, const int2* __restrict__ nodes,
               int32_t* __restrict__ idx, int* status, int iters) {
  using SM = SubSmem<D>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  uint16_t* rows = reinterpret_cast<uint16_t*>(smem_raw + SM::off_rows);
  double* pv = reinterpret_cast<double*>(smem_raw + SM::off_pv);
  int32_t* ids = reinterpret_cast<int32_t*>(smem_raw + SM::off_ids);
  uint16_t* loc = reinterpret_cast<uint16_t*>(smem_raw + SM::off_loc);
  uint16_t* stok = reinterpret_cast<uint16_t*>(smem_raw + SM::off_stok);
  double* zp = reinterpret_cast<double*>(smem_raw + SM::off_zp);
  __shared__ double mus[D], vs[D], mus2[D], vs2[D], red_d[16];
  __shared__ int red_i[8], hist[256], sh_sel[3], warp_tot[8];
  __shared__ unsigned long long sh_key;
  __shared__ double sh_sgn;
  __shared__ int2 lvl[2][SUB_BLOCKS];
  __shared__ int lvl_n[2];

  const int tid = threadIdx.x;
  const int2 node = nodes[blockIdx.x];
  const int bh = blockIdx.y;
  const int g0 = node.y, n = g0 * BLK, pos0 = node.x * BLK;
  if (g0 > SUB_BLOCKS) {   // never launched that way; keep the shared arrays in bounds regardless
    if (tid == 0) set_status(status, STATUS_BAD_INPUT);
    return;
  }
  int32_t* gidx = idx + (size_t)bh * N + pos0;
  const uint16_t* X = uhat + (size_t)bh * N * D;
  for (int t = tid; t < n; t += blockDim.x) {
    ids[t] = gidx[t];
    loc[t] = (uint16_t)t;
  }
  __syncthreads();
  constexpr int CH = D / 8;
  for (int c = tid; c < n * CH; c += blockDim.x) {
    const int t = c / CH, ch = c % CH;
    cp_async16(rows + (size_t)t * SM::RS + ch * 8, X + (size_t)ids[t] * D + ch * 8);
  }
  cp_async_commit();
  cp_async_wait<0>();
  if (tid == 0) { lvl[0][0] = make_int2(0, g0); lvl_n[0] = 1; }
  __syncthreads();
  int cur = 0;
  while (lvl_n[cur] > 0) {
    const int cnt = lvl_n[cur];
    // the level's groups two at a time (every listed group has at least 2 blocks)
    for (int i = 0; i < cnt; i += SUB_PAIR ? 2 : 1) {
      const int2 na = lvl[cur][i];
      const bool two = SUB_PAIR && i + 1 < cnt;
      const int2 nbn = two ? lvl[cur][i + 1] : na;
      float SA[Gram<D>::ACC], SB[Gram<D>::ACC];
      sub_cov<D>(rows, loc, zp, mus, na.x * BLK, na.y * BLK, SA);
      if (two) {
        sub_cov<D>(rows, loc, zp, mus2, nbn.x * BLK, nbn.y * BLK, SB);
        sub_power<D, true>(SA, SB, zp, vs, vs2, iters);
      } else {
        sub_power<D, false>(SA, SA, zp, vs, vs, iters);
      }
      sub_finish<D>(rows, pv, ids, loc, stok, zp, mus, vs, red_d, red_i, &sh_sgn, hist, sh_sel, &sh_key, warp_tot,
                    status, na.x * BLK, na.y * BLK);
      if (two)
        sub_finish<D>(rows, pv, ids, loc, stok, zp, mus2, vs2, red_d, red_i, &sh_sgn, hist, sh_sel, &sh_key,
                      warp_tot, status, nbn.x * BLK, nbn.y * BLK);
    }
    if (tid == 0) {
      int m = 0;
      for (int i = 0; i < cnt; ++i) {
        const int2 nd = lvl[cur][i];
        if (nd.y < 2) continue;
        const int gl = nd.y / 2, gr = nd.y - gl;
        if (gl >= 2) lvl[cur ^ 1][m++] = make_int2(nd.x, gl);
        if (gr >= 2) lvl[cur ^ 1][m++] = make_int2(nd.x + gl, gr);
      }
      lvl_n[cur ^ 1] = m;
    }
    __syncthreads();
    cur ^= 1;
  }
  for (int t = tid; t < n; t += blockDim.x) gidx[t] = ids[loc[t]];
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
  double* L = ws_at<double>(ws, pl.off_L);
  uint16_t* uhat = ws_at<uint16_t>(ws, pl.off_uhat);
  int32_t* idx = ws_at<int32_t>(ws, pl.off_idx);
  double* pval = ws_at<double>(ws, pl.off_pval);
  int32_t* pidx = ws_at<int32_t>(ws, pl.off_pidx);
  int2* nodes = ws_at<int2>(ws, pl.off_nodes);
  cudaError_t e;

  const size_t smem_w = sizeof(double) * D * (D + 1);
  e = cudaFuncSetAttribute(whiten_prep_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_w);
  if (e != cudaSuccess) return e;
  whiten_prep_kernel<D><<<pl.BH, 256, smem_w, s>>>(M, L, status);

  {
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long items = (long)pl.BH * (pl.N / NormSmem<D>::TOK);
    e = cudaFuncSetAttribute(normalize64_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)NormSmem<D>::bytes);
    if (e != cudaSuccess) return e;
    normalize64_kernel<D><<<(int)std::min<long>(items, sms), NormSmem<D>::THREADS, NormSmem<D>::bytes, s>>>(
        x, L, pl.N, pl.BH, uhat);
  }

  tree_build_kernel<<<1, 32, 0, s>>>(pl.nb, nodes);
  const long total = (long)pl.BH * pl.N;
  init_idx_kernel<<<(int)std::min<long>((total + 255) / 256, 4096), 256, 0, s>>>(idx, pl.N, total);

  const size_t smem_s = SplitSmem<D>::bytes;
  const size_t smem_t = SubSmem<D>::bytes;
  e = cudaFuncSetAttribute(subtree_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_t);
  if (e != cudaSuccess) return e;
  if constexpr (D == 128) {
    e = cudaFuncSetAttribute(big_gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::GramTcLayout::SMEM);
  } else {
    e = cudaFuncSetAttribute(big_gram_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s);
  }
  if (e != cudaSuccess) return e;
  const size_t smem_solve = 0;                     // S goes straight to registers
  const size_t smem_proj = sizeof(uint16_t) * Gram<D>::TILE * 3;
  e = cudaFuncSetAttribute(big_project_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_proj);
  if (e != cudaSuccess) return e;
  double* bpart = ws_at<double>(ws, pl.off_bigpart);
  double* binfo = ws_at<double>(ws, pl.off_biginfo);
  double* bcand = ws_at<double>(ws, pl.off_bigcand);
  double* gstore[2] = {ws_at<double>(ws, pl.off_gstore[0]), ws_at<double>(ws, pl.off_gstore[1])};
  for (int lv = 0; lv < pl.nlevels; ++lv) {
    if (pl.level_maxg[lv] <= SUB_BLOCKS) {   // this level and everything below it, in shared memory
      subtree_kernel<D><<<dim3(pl.level_count[lv], pl.BH), 256, smem_t, s>>>(uhat, pl.N, nodes + pl.level_off[lv],
                                                                            idx, status, pl.power_iters);
      break;
    }
    // each group spread over chunk CTAs; a right child's Gram derived from its parent's
    const int cnt = pl.level_count[lv], ch = pl.level_chunks[lv];
    const int2* nd = nodes + pl.level_off[lv];
    const int derive = pl.level_derive[lv];
    const int kstep = derive ? 2 : 1;
    double* gpar = derive ? gstore[(lv - 1) & 1] : nullptr;
    double* gout = pl.level_store[lv] ? gstore[lv & 1] : nullptr;
    if constexpr (D == 128)
      big_gram_tc_kernel<<<dim3(ch, cnt / kstep, pl.BH), tc::GT_THREADS, tc::GramTcLayout::SMEM, s>>>(
          uhat, pl.N, nd, cnt, ch, kstep, idx, bpart, status);
    else
      big_gram_kernel<D><<<dim3(ch, cnt / kstep, pl.BH), 256, smem_s, s>>>(uhat, pl.N, nd, cnt, ch, kstep, idx, bpart);
    if (ch > 1)
      big_reduce_kernel<D><<<dim3(std::min(16, (D * D + D + 255) / 256), cnt / kstep, pl.BH), 256, 0, s>>>(
          nd, cnt, ch, kstep, bpart);
    big_solve_kernel<D><<<dim3(cnt, pl.BH), 256, smem_solve, s>>>(nd, cnt, ch, bpart, binfo, derive, gpar,
                                                                   derive ? pl.level_count[lv - 1] : 0, gout,
                                                                   pl.power_iters);
    big_project_kernel<D><<<dim3(ch, cnt, pl.BH), 256, smem_proj, s>>>(uhat, pl.N, nd, cnt, ch, idx, binfo, pval,
                                                                      pidx, bcand);
    if (pl.level_maxg[lv] * BLK >= BIG_SELECT_WIDE_TOKENS)
      big_select_kernel<1024><<<dim3(cnt, pl.BH), 1024, 0, s>>>(pl.N, nd, cnt, ch, bcand, idx, pval, pidx, status);
    else
      big_select_kernel<256><<<dim3(cnt, pl.BH), 256, 0, s>>>(pl.N, nd, cnt, ch, bcand, idx, pval, pidx, status);
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
