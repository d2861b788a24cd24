// Steps a5-a7 on the legacy tensor-core path (mma.sync m16n8k16, bf16 in,
// f32 accumulate): exact branch, compressed branch, merge and un-permute.
//
// One CTA per (query block a, head): 64 queries, 4 warps of 16 rows each.
// Exact branch ("Spark-H3" news post, "What Spark-Attn changed": the exact
// branch fully computes the top-ranked key/value blocks): for every block b
// in sel[a], S = Q K_b^T / sqrt(d) and an online softmax accumulates P V_b.
// Compressed branch ("MiniMax H3 Spark Attention (SM89)", under the hood: a
// real Q per query, only K/V downsampled): the same online softmax continues
// over the summaries k~_b, v~_b of every block b not in sel[a], with logit
// q . k~_b / sqrt(d) + beta_b. A single running (max, sum, output) over both
// term sets is the log-sum-exp merge of the two branch softmaxes. The
// epilogue divides by the sum and writes each row at its original token
// index perm[64a + r]; lse (natural log) likewise.
#include <math.h>

#include "common.cuh"
#include "plan.h"

namespace spark {

template <int D>
struct AttnCfg {
  static constexpr int THREADS = 128;
  static constexpr int RS = D + 8;               // padded smem row stride (elements)
  static constexpr int TILE = BLK * RS;
  static constexpr int KT = D / 16;              // k-steps over the head dim
  static constexpr int NT_O = D / 8;             // n8 tiles of the output
  static constexpr size_t smem = sizeof(uint16_t) * TILE * 5;   // Q + 2 x (K, V)
};

template <int D>
__device__ __forceinline__ void load_rows(uint16_t* sm, const uint16_t* src, int tid) {
  constexpr int CH = D / 8;
#pragma unroll
  for (int c = tid; c < BLK * CH; c += AttnCfg<D>::THREADS) {
    const int r = c / CH, ch = c % CH;
    cp_async16(sm + r * AttnCfg<D>::RS + ch * 8, src + (size_t)r * D + ch * 8);
  }
}

// One 64-key tile of the online softmax. bias/mask apply to the compressed
// tiles only (mask bit set = column excluded).
template <int D, bool COMP>
__device__ __forceinline__ void attend_tile(const uint32_t (&qf)[AttnCfg<D>::KT][4], const uint16_t* ks,
                                            const uint16_t* vs, float (&o)[AttnCfg<D>::NT_O][4],
                                            float (&m)[2], float (&l)[2], float sl2,
                                            const float* bias_l2, uint64_t colmask, int lane) {
  using C = AttnCfg<D>;
  float s[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int r = 0; r < 4; ++r) s[nt][r] = 0.f;
#pragma unroll
  for (int kt = 0; kt < C::KT; ++kt) {
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(b0, b1, b2, b3,
              ks + (np * 16 + (lane & 7) + (lane >> 4) * 8) * C::RS + kt * 16 + ((lane >> 3) & 1) * 8);
      mma_bf16(s[2 * np], qf[kt], b0, b1);
      mma_bf16(s[2 * np + 1], qf[kt], b2, b3);
    }
  }
  // scale to log2 domain, bias, mask
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int col = nt * 8 + 2 * (lane & 3) + (r & 1);
      float x = s[nt][r] * sl2;
      if (COMP) {
        x += bias_l2[col];
        if ((colmask >> col) & 1ull) x = -INFINITY;
      }
      s[nt][r] = x;
      mx[r >> 1] = fmaxf(mx[r >> 1], x);
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
  }
  float mnew[2], corr[2], msafe[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mnew[h] = fmaxf(m[h], mx[h]);
    msafe[h] = (mnew[h] == -INFINITY) ? 0.f : mnew[h];
    corr[h] = exp2f(m[h] - msafe[h]);
    m[h] = mnew[h];
  }
  float rs[2] = {0.f, 0.f};
  uint32_t pf[4][4];   // P as A fragments, 4 k-steps of 16 keys
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const float p0 = exp2f(s[nt][0] - msafe[0]);
    const float p1 = exp2f(s[nt][1] - msafe[0]);
    const float p2 = exp2f(s[nt][2] - msafe[1]);
    const float p3 = exp2f(s[nt][3] - msafe[1]);
    rs[0] += p0 + p1;
    rs[1] += p2 + p3;
    const int kk = nt >> 1, hi = nt & 1;
    pf[kk][hi * 2 + 0] = pack_bf2(p0, p1);
    pf[kk][hi * 2 + 1] = pack_bf2(p2, p3);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 1);
    rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 2);
    l[h] = l[h] * corr[h] + rs[h];
  }
#pragma unroll
  for (int nt = 0; nt < C::NT_O; ++nt) {
    o[nt][0] *= corr[0]; o[nt][1] *= corr[0];
    o[nt][2] *= corr[1]; o[nt][3] *= corr[1];
  }
  // O += P V : A = P (16 x 64 keys), B = V (64 keys x D)
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint32_t a[4] = {pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3]};
#pragma unroll
    for (int np = 0; np < C::NT_O / 2; ++np) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(b0, b1, b2, b3,
                vs + (kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * C::RS + np * 16 + (lane >> 4) * 8);
      mma_bf16(o[2 * np], a, b0, b1);
      mma_bf16(o[2 * np + 1], a, b2, b3);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(128)
attn_mma_kernel(const uint16_t* __restrict__ Qp, const uint16_t* __restrict__ Kp,
                const uint16_t* __restrict__ Vp, const uint16_t* __restrict__ kt,
                const uint16_t* __restrict__ vt, const float* __restrict__ beta,
                const int32_t* __restrict__ perm, const int32_t* __restrict__ sel, int N, int nb,
                int nb_pad, int ksel, uint16_t* __restrict__ out, float* __restrict__ lse,
                int* status) {
  using C = AttnCfg<D>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem_raw);
  uint16_t* kbuf = qs + C::TILE;          // [2][TILE]
  uint16_t* vbuf = kbuf + 2 * C::TILE;    // [2][TILE]
  __shared__ uint32_t selmask[SPARK_MAX_BLOCKS / 32];
  __shared__ float bias_sh[2][BLK];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int a = blockIdx.x, bh = blockIdx.y;
  const size_t hb = (size_t)bh * N * D;
  const int32_t* srow = sel + ((size_t)bh * nb + a) * ksel;
  const int nwords = (nb + 31) / 32;
  for (int i = tid; i < SPARK_MAX_BLOCKS / 32; i += C::THREADS) selmask[i] = 0u;

  load_rows<D>(qs, Qp + hb + (size_t)a * BLK * D, tid);
  cp_async_commit();
  // first exact tile
  {
    int b0 = srow[0];
    if ((unsigned)b0 >= (unsigned)nb) b0 = 0;
    load_rows<D>(kbuf, Kp + hb + (size_t)b0 * BLK * D, tid);
    load_rows<D>(vbuf, Vp + hb + (size_t)b0 * BLK * D, tid);
    cp_async_commit();
  }
  __syncthreads();
  for (int i = tid; i < ksel; i += C::THREADS) {
    const int b = srow[i];
    if ((unsigned)b < (unsigned)nb) atomicOr(&selmask[b >> 5], 1u << (b & 31));
    else set_status(status, STATUS_BAD_INPUT);
  }
  cp_async_wait<0>();
  __syncthreads();

  // Q fragments for this warp's 16 rows
  uint32_t qf[C::KT][4];
#pragma unroll
  for (int kt2 = 0; kt2 < C::KT; ++kt2)
    ldsm_x4(qf[kt2][0], qf[kt2][1], qf[kt2][2], qf[kt2][3],
            qs + (warp * 16 + (lane & 15)) * C::RS + kt2 * 16 + (lane >> 4) * 8);

  float o[C::NT_O][4];
#pragma unroll
  for (int nt = 0; nt < C::NT_O; ++nt)
#pragma unroll
    for (int r = 0; r < 4; ++r) o[nt][r] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  const float LOG2E = 1.4426950408889634f;
  const float sl2 = (1.0f / sqrtf((float)D)) * LOG2E;

  const int ncomp = (nb + BLK - 1) / BLK;
  const int total = ksel + ncomp;
  for (int it = 0; it < total; ++it) {
    const int nxt = it + 1;
    if (nxt < total) {
      uint16_t* kd = kbuf + (nxt & 1) * C::TILE;
      uint16_t* vd = vbuf + (nxt & 1) * C::TILE;
      if (nxt < ksel) {
        int b = srow[nxt];
        if ((unsigned)b >= (unsigned)nb) b = 0;
        load_rows<D>(kd, Kp + hb + (size_t)b * BLK * D, tid);
        load_rows<D>(vd, Vp + hb + (size_t)b * BLK * D, tid);
      } else {
        const int t = nxt - ksel;
        load_rows<D>(kd, kt + ((size_t)bh * nb_pad + (size_t)t * BLK) * D, tid);
        load_rows<D>(vd, vt + ((size_t)bh * nb_pad + (size_t)t * BLK) * D, tid);
        if (tid < BLK) bias_sh[nxt & 1][tid] = beta[(size_t)bh * nb_pad + (size_t)t * BLK + tid] * LOG2E;
      }
    }
    cp_async_commit();
    const uint16_t* ks = kbuf + (it & 1) * C::TILE;
    const uint16_t* vs = vbuf + (it & 1) * C::TILE;
    if (it < ksel) {
      attend_tile<D, false>(qf, ks, vs, o, m, l, sl2, nullptr, 0ull, lane);
    } else {
      const int t = it - ksel;
      // excluded columns: selected blocks and rows past nb
      const int c0 = t * BLK;
      uint64_t mask = ((uint64_t)selmask[c0 >> 5]) | ((uint64_t)selmask[(c0 >> 5) + 1] << 32);
      if (c0 + BLK > nb) {
        const int valid = nb - c0;
        mask |= ~0ull << valid;
        if (((c0 >> 5) + 1) >= nwords) mask |= 0xffffffff00000000ull;
      }
      attend_tile<D, true>(qf, ks, vs, o, m, l, sl2, bias_sh[it & 1], mask, lane);
    }
    cp_async_wait<0>();
    __syncthreads();
  }

  // epilogue: normalise, stage through smem, scatter rows to original order
  const float inv0 = 1.f / l[0], inv1 = 1.f / l[1];
  const int r0 = warp * 16 + (lane >> 2);
#pragma unroll
  for (int nt = 0; nt < C::NT_O; ++nt) {
    const int col = nt * 8 + 2 * (lane & 3);
    *reinterpret_cast<uint32_t*>(qs + r0 * C::RS + col) = pack_bf2(o[nt][0] * inv0, o[nt][1] * inv0);
    *reinterpret_cast<uint32_t*>(qs + (r0 + 8) * C::RS + col) = pack_bf2(o[nt][2] * inv1, o[nt][3] * inv1);
  }
  const int32_t* prow = perm + (size_t)bh * N + (size_t)a * BLK;
  if (lse != nullptr && (lane & 3) == 0 && (unsigned)prow[r0] < (unsigned)N &&
      (unsigned)prow[r0 + 8] < (unsigned)N) {
    const float LN2 = 0.6931471805599453f;
    lse[(size_t)bh * N + prow[r0]] = (m[0] + log2f(l[0])) * LN2;
    lse[(size_t)bh * N + prow[r0 + 8]] = (m[1] + log2f(l[1])) * LN2;
  }
  __syncthreads();
  constexpr int CH = D / 8;
  for (int c = tid; c < BLK * CH; c += C::THREADS) {
    const int r = c / CH, ch = c % CH;
    if ((unsigned)prow[r] >= (unsigned)N) continue;
    *reinterpret_cast<uint4*>(out + hb + (size_t)prow[r] * D + ch * 8) =
        *reinterpret_cast<const uint4*>(qs + r * C::RS + ch * 8);
  }
}

template <int D>
static cudaError_t run_attn(const Plan& pl, const int32_t* perm, const int32_t* sel, uint16_t* out,
                            float* lse, void* ws, int* status, cudaStream_t s) {
  using C = AttnCfg<D>;
  auto kern = attn_mma_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(pl.nb, pl.BH), C::THREADS, C::smem, s>>>(
      ws_at<uint16_t>(ws, pl.off_Qp), ws_at<uint16_t>(ws, pl.off_Kp), ws_at<uint16_t>(ws, pl.off_Vp),
      ws_at<uint16_t>(ws, pl.off_kt), ws_at<uint16_t>(ws, pl.off_vt), ws_at<float>(ws, pl.off_beta),
      perm, sel, pl.N, pl.nb, pl.nb_pad, pl.ksel, out, lse, status);
  return cudaGetLastError();
}

cudaError_t launch_attn(const Plan& pl, const int32_t* perm, const int32_t* sel, uint16_t* out,
                        float* lse, void* ws, int* status, cudaStream_t s) {
  if (pl.d == 128) return run_attn<128>(pl, perm, sel, out, lse, ws, status, s);
  return run_attn<64>(pl, perm, sel, out, lse, ws, status, s);
}

}  // namespace spark
