// Step a3 (block statistics, summaries) and a4 (top-K block selection).
//
// blockstats: one CTA per (key block, head). Gathers the block's 64 q, k, v
//   rows by the permutation, writes the permuted copies the attention
//   kernel streams, the float64 block means of q and k, and the block's
//   summary ("Spark-H3" news post, Spark-Reweight bullet and figure caption;
//   "MiniMax H3 Spark Attention (SM89)", under the hood): anchor logits
//   x_j = qbar . k_j / sqrt(d), w = softmax(x), k~ = sum w k, v~ = sum w v,
//   beta = ln sum e^x - qbar . k~ / sqrt(d) (k~ as stored in bf16), or the
//   mean-pooling ablation (mean k, mean v, beta = ln 64).
// score + topk: block scores s_ab = Qbar_a . Kbar_b / sqrt(d) in float64
//   ("Spark-H3" news post: the exact branch computes the top-ranked
//   key/value blocks) for a chunk of heads at a time, then per row a
//   warp-level radix select of the Ksel largest, ties to the lower b,
//   written in ascending b order.
#include <math.h>

#include "common.cuh"
#include "dmma.cuh"
#include "plan.h"

namespace spark {

template <int D>
__global__ void __launch_bounds__(256)
blockstats_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                  const uint16_t* __restrict__ v, const int32_t* __restrict__ perm,
                  const int32_t* __restrict__ perm_k,
                  const double* __restrict__ qmean, int N, int nb, int nb_pad, int summary,
                  uint16_t* __restrict__ Qp, uint16_t* __restrict__ Kp, uint16_t* __restrict__ Vp,
                  double* __restrict__ qm, double* __restrict__ km, uint16_t* __restrict__ kt,
                  uint16_t* __restrict__ vt, float* __restrict__ beta, int* status) {
  constexpr int CH = D / 8;   // 16-byte chunks per row
  __shared__ __align__(16) uint16_t ks[BLK * D];
  __shared__ __align__(16) uint16_t vsm[BLK * D];
  __shared__ float qb[D];
  __shared__ float w[BLK];
  __shared__ float red[8];
  __shared__ float sh_m, sh_lz;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x, bh = blockIdx.y;
  const size_t hb = (size_t)bh * N * D;

  if (b >= nb) {   // zero padding rows of the summary tables
    for (int j = tid; j < D; j += blockDim.x) {
      kt[((size_t)bh * nb_pad + b) * D + j] = 0;
      vt[((size_t)bh * nb_pad + b) * D + j] = 0;
    }
    if (tid == 0) beta[(size_t)bh * nb_pad + b] = 0.f;
    return;
  }

  // gather + permuted copies (q through the query permutation, k and v
  // through the key permutation, the same array unless the layout is separate)
  const int32_t* pr = perm + (size_t)bh * N + (size_t)b * BLK;
  const int32_t* pk = perm_k + (size_t)bh * N + (size_t)b * BLK;
  for (int c = tid; c < BLK * CH; c += blockDim.x) {
    const int r = c / CH, ch = c % CH;
    int row = pr[r], rowk = pk[r];
    if ((unsigned)row >= (unsigned)N) { set_status(status, STATUS_BAD_INPUT); row = 0; }
    if ((unsigned)rowk >= (unsigned)N) { set_status(status, STATUS_BAD_INPUT); rowk = 0; }
    const size_t src = hb + (size_t)row * D + ch * 8, srck = hb + (size_t)rowk * D + ch * 8;
    const size_t dst = hb + ((size_t)b * BLK + r) * D + ch * 8;
    const uint4 kk = *reinterpret_cast<const uint4*>(k + srck);
    const uint4 vv = *reinterpret_cast<const uint4*>(v + srck);
    const uint4 qq = *reinterpret_cast<const uint4*>(q + src);
    *reinterpret_cast<uint4*>(Kp + dst) = kk;
    *reinterpret_cast<uint4*>(Vp + dst) = vv;
    *reinterpret_cast<uint4*>(Qp + dst) = qq;
    *reinterpret_cast<uint4*>(ks + r * D + ch * 8) = kk;
    *reinterpret_cast<uint4*>(vsm + r * D + ch * 8) = vv;
  }
  if (tid < D) qb[tid] = (float)qmean[(size_t)bh * D + tid];
  __syncthreads();

  // float64 block means (exact sums of 64 bf16 values). q is re-read from the
  // permuted copy this CTA just wrote (same thread block, after the barrier).
  if (tid < D) {
    double s = 0.0;
    for (int r = 0; r < BLK; ++r) s += (double)bf2f(Qp[hb + ((size_t)b * BLK + r) * D + tid]);
    qm[((size_t)bh * nb + b) * D + tid] = s * (1.0 / BLK);
  } else if (tid < 2 * D) {
    const int j = tid - D;
    double s = 0.0;
    for (int r = 0; r < BLK; ++r) s += (double)bf2f(ks[r * D + j]);
    km[((size_t)bh * nb + b) * D + j] = s * (1.0 / BLK);
  }

  const float scale = 1.0f / sqrtf((float)D);
  if (summary == SPARK_SUMMARY_MEANPOOL) {
    __syncthreads();
    if (tid < D) {
      float sk = 0.f, sv = 0.f;
      for (int r = 0; r < BLK; ++r) { sk += bf2f(ks[r * D + tid]); sv += bf2f(vsm[r * D + tid]); }
      kt[((size_t)bh * nb_pad + b) * D + tid] = f2bf(sk * (1.f / BLK));
      vt[((size_t)bh * nb_pad + b) * D + tid] = f2bf(sv * (1.f / BLK));
    }
    if (tid == 0) beta[(size_t)bh * nb_pad + b] = logf((float)BLK);
    return;
  }

  // anchor logits: warp w handles rows 8w..8w+7
  for (int r = warp * 8; r < warp * 8 + 8; ++r) {
    float s = 0.f;
    for (int j = lane; j < D; j += 32) s = fmaf(qb[j], bf2f(ks[r * D + j]), s);
    s = warp_sumf(s);
    if (lane == 0) w[r] = s * scale;
  }
  __syncthreads();
  if (warp == 0) {
    const float x0 = w[lane], x1 = w[lane + 32];
    const float m = warp_maxf(fmaxf(x0, x1));
    const float e0 = expf(x0 - m), e1 = expf(x1 - m);
    const float z = warp_sumf(e0 + e1);
    w[lane] = e0 / z;
    w[lane + 32] = e1 / z;
    if (lane == 0) { sh_m = m; sh_lz = logf(z); }
  }
  __syncthreads();
  float dotpart = 0.f;
  if (tid < D) {
    float sk = 0.f, sv = 0.f;
    for (int r = 0; r < BLK; ++r) {
      sk = fmaf(w[r], bf2f(ks[r * D + tid]), sk);
      sv = fmaf(w[r], bf2f(vsm[r * D + tid]), sv);
    }
    const uint16_t kb = f2bf(sk);
    kt[((size_t)bh * nb_pad + b) * D + tid] = kb;
    vt[((size_t)bh * nb_pad + b) * D + tid] = f2bf(sv);
    dotpart = qb[tid] * bf2f(kb);
  }
  dotpart = warp_sumf(dotpart);
  if (lane == 0) red[warp] = dotpart;
  __syncthreads();
  if (tid == 0) {
    float dsum = 0.f;
    for (int i = 0; i < 8; ++i) dsum += red[i];
    beta[(size_t)bh * nb_pad + b] = (sh_m + sh_lz) - dsum * scale;
  }
}

// ------------------------------------------------------------------ selection
// score_kernel: the block-score matrix of one chunk of heads,
//   sc[h][a][b] = (Qbar_a . Kbar_b) / sqrt(d) in float64, on the float64
//   tensor cores (mma.sync m16n8k16, dmma.cuh): a CTA computes a 128 x 128
//   tile; warp w owns rows 32 (w % 4).. and columns 64 (w / 4)..: two 16-row
//   by eight 8-column MMA tiles. The d dimension is staged 16 at a time
//   through a cp.async double buffer of float64 rows (stride 20 doubles: the
//   fragments' half-warps hit distinct bank pairs); rows past nb are zero.
constexpr int SC_TILE = 128, SC_KSTEP = 16, SC_LD = SC_KSTEP + 4;
constexpr int SC_SMEM = (int)sizeof(double) * 4 * SC_TILE * SC_LD;   // two buffers of each operand

template <int D>
__global__ void __launch_bounds__(256)
score_kernel(const double* __restrict__ qm, const double* __restrict__ km, int nb, int h0,
             double* __restrict__ sc) {
  extern __shared__ __align__(16) double scs[];       // qs [2][a][k], then ks [2][b][k]
  auto qs = [&](int buf) { return scs + buf * (SC_TILE * SC_LD); };
  auto ks = [&](int buf) { return scs + (2 + buf) * (SC_TILE * SC_LD); };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int b0 = blockIdx.x * SC_TILE, a0 = blockIdx.y * SC_TILE, h = blockIdx.z;
  const size_t bh = (size_t)(h0 + h);
  const double* Q = qm + bh * nb * D;
  const double* K = km + bh * nb * D;
  const int wr = (warp & 3) * 32, wc = (warp >> 2) * 64;
  // loader: 128 rows x 16 doubles = 1024 16-byte chunks per operand, 4 per thread
  auto load = [&](int buf, int kc) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = tid + 256 * i, r = c >> 3, ch = c & 7;
      double* dq = qs(buf) + r * SC_LD + 2 * ch;
      double* dk = ks(buf) + r * SC_LD + 2 * ch;
      if (a0 + r < nb) cp_async16(dq, Q + (size_t)(a0 + r) * D + kc + 2 * ch);
      else *reinterpret_cast<double2*>(dq) = make_double2(0.0, 0.0);
      if (b0 + r < nb) cp_async16(dk, K + (size_t)(b0 + r) * D + kc + 2 * ch);
      else *reinterpret_cast<double2*>(dk) = make_double2(0.0, 0.0);
    }
  };
  double acc[2][8][4];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[m][j][e] = 0.0;
  load(0, 0);
  cp_async_commit();
  for (int kc = 0; kc < D; kc += SC_KSTEP) {
    const int buf = (kc / SC_KSTEP) & 1;
    if (kc + SC_KSTEP < D) load(buf ^ 1, kc + SC_KSTEP);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const double* qb = qs(buf);
    const double* kb = ks(buf);
    double a[2][8];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int i = 0; i < 8; ++i) a[m][i] = qb[(wr + 16 * m + g + 8 * (i % 2)) * SC_LD + t4 + 4 * (i / 2)];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      double bf[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) bf[i] = kb[(wc + 8 * j + g) * SC_LD + t4 + 4 * i];
#pragma unroll
      for (int m = 0; m < 2; ++m) dmma16816(acc[m][j], a[m], bf);
    }
    __syncthreads();                                   // the buffer is refilled next step
  }
  cp_async_wait<0>();
  const double sd = sqrt((double)D);
  double* out = sc + (size_t)h * nb * nb;
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int a = a0 + wr + 16 * m + g + 8 * (e >> 1), b = b0 + wc + 8 * j + 2 * t4 + (e & 1);
        if (a < nb && b < nb) out[(size_t)a * nb + b] = acc[m][j][e] / sd;
      }
}

// topk_kernel: one warp per query block a of the chunk: the ksel largest
//   scores of row a, ties to the lower block index, written in ascending
//   block order. Radix select over the ordered keys of -score, 8 bits per
//   pass from the top, stopping as soon as the target key is isolated.
__global__ void __launch_bounds__(256)
topk_kernel(const double* __restrict__ sc, int nb, int ksel, int h0, int heads, int32_t* __restrict__ sel) {
  __shared__ int hist[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long row = (long)blockIdx.x * 8 + warp;     // (head in chunk, query block)
  if (row >= (long)heads * nb) return;
  const int h = (int)(row / nb), a = (int)(row % nb);
  const double* srow = sc + ((size_t)h * nb + a) * nb;
  int* hs = hist[warp];
  auto key = [&](int bb) -> uint64_t { return ordered_key(-srow[bb]); };
  uint64_t prefix = 0, mask = 0;
  int rank = ksel;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += 32) hs[i] = 0;
    __syncwarp();
    for (int bb = lane; bb < nb; bb += 32) {
      const uint64_t kk = key(bb);
      if ((kk & mask) == prefix) atomicAdd(&hs[(kk >> shift) & 255], 1);
    }
    __syncwarp();
    int loc[8], s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) { loc[j] = hs[lane * 8 + j]; s += loc[j]; }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const int excl = incl - s;
    int bucket = 0, newrank = 0, bcount = 0;
    const bool mine = (excl < rank && rank <= incl);
    if (mine) {
      int c = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (c < rank && rank <= c + loc[j]) { bucket = lane * 8 + j; newrank = rank - c; bcount = loc[j]; }
        c += loc[j];
      }
    }
    const unsigned owner = __ballot_sync(0xffffffffu, mine);
    const int src = __ffs(owner) - 1;
    bucket = __shfl_sync(0xffffffffu, bucket, src);
    newrank = __shfl_sync(0xffffffffu, newrank, src);
    bcount = __shfl_sync(0xffffffffu, bcount, src);
    prefix |= ((uint64_t)bucket) << shift;
    mask |= ((uint64_t)255) << shift;
    rank = newrank;
    __syncwarp();
    if (bcount == 1) break;    // a single key has this prefix: it is the target
  }
  // the target key: the unique key with this prefix, or (all 64 bits fixed) the prefix itself
  uint64_t kstar = prefix;
  if (mask != ~0ull) {
    uint64_t mine = ~0ull;
    for (int bb = lane; bb < nb; bb += 32) {
      const uint64_t kk = key(bb);
      if ((kk & mask) == prefix) mine = kk;
    }
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t other = __shfl_xor_sync(0xffffffffu, mine, o);
      mine = other < mine ? other : mine;
    }
    kstar = mine;
    rank = 1;
  }
  // members with key < kstar, plus the first `rank` members with key == kstar
  int out = 0, ties = 0;
  int32_t* dst = sel + ((size_t)(h0 + h) * nb + a) * ksel;
  for (int c0 = 0; c0 < nb; c0 += 32) {
    const int bb = c0 + lane;
    uint64_t kk = ~0ull;
    if (bb < nb) kk = key(bb);
    const bool less = bb < nb && kk < kstar;
    const bool eq = bb < nb && kk == kstar;
    const unsigned em = __ballot_sync(0xffffffffu, eq);
    const int eq_before = ties + __popc(em & ((1u << lane) - 1u));
    const bool take = less || (eq && eq_before < rank);
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    const int at = out + __popc(tm & ((1u << lane) - 1u));
    if (take && at < ksel) dst[at] = bb;
    out += __popc(tm);
    ties += __popc(em);
  }
}

// tail_logits_kernel: the compressed-branch logits of the block tail
//   granularity, x_ab = (Qbar_a . k~_b / sqrt(d) + beta_b) * log2(e), for 8
//   query blocks a per CTA and every summary b (log2 units, as the attention
//   kernel works in; columns nb .. nb_pad-1 are -inf). float32 dot products of
//   the float64 block means (rounded to float32) and the bf16 summaries.
constexpr int TAIL_ROWS = 8;

template <int D>
__global__ void __launch_bounds__(256)
tail_logits_kernel(const double* __restrict__ qm, const uint16_t* __restrict__ kt, const float* __restrict__ beta,
                   int nb, int nb_pad, float* __restrict__ tab) {
  __shared__ float qa[TAIL_ROWS][D];
  const int tid = threadIdx.x, a0 = blockIdx.x * TAIL_ROWS, bh = blockIdx.y;
  for (int e = tid; e < TAIL_ROWS * D; e += blockDim.x) {
    const int r = e / D, j = e % D;
    qa[r][j] = a0 + r < nb ? (float)qm[((size_t)bh * nb + a0 + r) * D + j] : 0.f;
  }
  __syncthreads();
  const float scale = 1.0f / sqrtf((float)D), log2e = 1.4426950408889634f;
  for (int b = tid; b < nb_pad; b += blockDim.x) {
    float acc[TAIL_ROWS];
#pragma unroll
    for (int r = 0; r < TAIL_ROWS; ++r) acc[r] = 0.f;
    if (b < nb) {
      const uint4* row = reinterpret_cast<const uint4*>(kt + ((size_t)bh * nb_pad + b) * D);
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
        const uint4 w = row[c];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = bf_lo(ws[e]), hi = bf_hi(ws[e]);
#pragma unroll
          for (int r = 0; r < TAIL_ROWS; ++r) acc[r] = fmaf(qa[r][8 * c + 2 * e + 1], hi, fmaf(qa[r][8 * c + 2 * e], lo, acc[r]));
        }
      }
    }
    const float bb = b < nb ? beta[(size_t)bh * nb_pad + b] : 0.f;
#pragma unroll
    for (int r = 0; r < TAIL_ROWS; ++r) {
      if (a0 + r >= nb) break;
      tab[((size_t)bh * nb + a0 + r) * nb_pad + b] = b < nb ? (acc[r] * scale + bb) * log2e : -INFINITY;
    }
  }
}

template <int D>
static cudaError_t run_select(const Plan& pl, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                              const int32_t* perm, const double* qmean, int32_t* sel, int summary,
                              void* ws, int* status, cudaStream_t s) {
  uint16_t* Qp = ws_at<uint16_t>(ws, pl.off_Qp);
  uint16_t* Kp = ws_at<uint16_t>(ws, pl.off_Kp);
  uint16_t* Vp = ws_at<uint16_t>(ws, pl.off_Vp);
  double* qm = ws_at<double>(ws, pl.off_qm);
  double* km = ws_at<double>(ws, pl.off_km);
  uint16_t* kt = ws_at<uint16_t>(ws, pl.off_kt);
  uint16_t* vt = ws_at<uint16_t>(ws, pl.off_vt);
  float* beta = ws_at<float>(ws, pl.off_beta);
  const int32_t* perm_k = perm + (pl.nperm == 2 ? (size_t)pl.BH * pl.N : 0);
  blockstats_kernel<D><<<dim3(pl.nb_pad, pl.BH), 256, 0, s>>>(q, k, v, perm, perm_k, qmean, pl.N, pl.nb,
                                                              pl.nb_pad, summary, Qp, Kp, Vp, qm, km,
                                                              kt, vt, beta, status);
  if (pl.tail == SPARK_TAIL_BLOCK)
    tail_logits_kernel<D><<<dim3((pl.nb + TAIL_ROWS - 1) / TAIL_ROWS, pl.BH), 256, 0, s>>>(
        qm, kt, beta, pl.nb, pl.nb_pad, ws_at<float>(ws, pl.off_tail));
  double* sc = ws_at<double>(ws, pl.off_scores);
  const int tiles = (pl.nb + SC_TILE - 1) / SC_TILE;
  cudaError_t e = cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SC_SMEM);
  if (e != cudaSuccess) return e;
  for (int h0 = 0; h0 < pl.BH; h0 += pl.score_heads) {
    const int heads = std::min(pl.score_heads, pl.BH - h0);
    score_kernel<D><<<dim3(tiles, tiles, heads), 256, SC_SMEM, s>>>(qm, km, pl.nb, h0, sc);
    const long rows = (long)heads * pl.nb;
    topk_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(sc, pl.nb, pl.ksel, h0, heads, sel);
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const Plan& pl, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          const int32_t* perm, const double* qmean, int32_t* sel, int summary,
                          void* ws, int* status, cudaStream_t s) {
  if (pl.d == 128) return run_select<128>(pl, q, k, v, perm, qmean, sel, summary, ws, status, s);
  return run_select<64>(pl, q, k, v, perm, qmean, sel, summary, ws, status, s);
}

}  // namespace spark
