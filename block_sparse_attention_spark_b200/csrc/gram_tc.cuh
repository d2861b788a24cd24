// Gram sums G = sum_t x_t x_t^T and column sums over tiles of 64 rows of a
// [*, 128] bf16 matrix on the sm_100a tensor cores (tcgen05.mma, TMEM
// accumulators), for the moments (contiguous rows) and the reblock levels
// (rows gathered through an index list).
//
// A CTA of 256 threads streams its tiles through a two-group ring in shared
// memory (4 tiles = 256 rows per group, cp.async, 128-byte swizzle: the
// layout TMA would write). One thread issues G_group = X^T X for the group as
// M128 N128 K16 MMAs with X as the MN-major operand on both sides, into one
// of two TMEM accumulators (128 columns each), and commits to that
// accumulator's mbarrier. While the next group loads and multiplies, the
// eight warps add the previous group's float32 sums into float64 registers
// (warp w: rows 32 (w % 4).., columns 64 (w / 4)..): float32 sums over 256
// rows, float64 across groups, as in the mma.sync kernels.
#pragma once

#include "tc_ptx.cuh"

namespace spark {
namespace tc {

constexpr int GT_TOK = 64;      // rows per tile
constexpr int GT_GROUP = 4;     // tiles per accumulator group
constexpr int GT_THREADS = 256;

struct GramTcLayout {
  static constexpr int D = 128;
  static constexpr int ATOM = GT_TOK * 128;          // 64 rows x 128 B (64 columns)
  static constexpr int TILE = ATOM * (D / 64);       // 16 KB
  static constexpr int GROUP = TILE * GT_GROUP;      // 64 KB
  static constexpr int SMEM = 2 * GROUP + 1024;
  // kind::f16, F32 accumulate, BF16 A and B, both MN-major, N = M = 128
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                    ((uint32_t)(D >> 3) << 17) | ((uint32_t)(D >> 4) << 24);
};

// rowf(t, r): row index (into X, units of 128 elements) of row r of tile t.
// out: 128*128 Gram sums, then 128 column sums (float64). status: timeout bit.
// EXACT_CS: column sums added in float64 element by element (exact for bf16
// inputs, as the anchor mean needs); otherwise float32 within a tile.
template <bool EXACT_CS, class RowF>
__device__ void gram_tc_body(const uint16_t* __restrict__ X, RowF rowf, int ntiles, double* __restrict__ out,
                             int* status) {
  using L = GramTcLayout;
  constexpr int D = L::D;
  extern __shared__ unsigned char gsm_raw[];
  __shared__ __align__(8) uint64_t gbar[3];           // two accumulators' MMA done, drain
  __shared__ uint32_t gtmem_sh;
  __shared__ double gcs[2][D];
  __shared__ int gabort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(gsm_raw) + 1023u) & ~1023u;
  const uint32_t bar0 = smem_u32(&gbar[0]);
  if (tid == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
    mbar_init(bar0 + 16, 1);
    gabort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&gtmem_sh)),
                 "r"(256));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = gtmem_sh;
  const int ngroups = (ntiles + GT_GROUP - 1) / GT_GROUP;

  // cp.async of one group's tiles into ring half g & 1 (128-byte swizzle:
  // 16-byte chunk c of row r lands at chunk c ^ (r % 8) of the 128-byte row).
  // Thread tid copies chunk tid % 16 of rows tid / 16 + 16 k of each tile;
  // it reads all of its row indices first, so their latencies overlap and
  // the copies follow in one burst.
  constexpr int RSTEP = GT_THREADS / (D / 8), RPT = GT_TOK / RSTEP;
  auto load_group = [&](int g) {
    const uint32_t gb = base + (uint32_t)((g & 1) * L::GROUP);
    const int t0 = g * GT_GROUP;
    const int ch = tid % (D / 8), r0 = tid / (D / 8);
    const int a = ch >> 3, c = ch & 7;
    int src[GT_GROUP][RPT];
#pragma unroll
    for (int tt = 0; tt < GT_GROUP; ++tt)
#pragma unroll
      for (int k = 0; k < RPT; ++k) src[tt][k] = t0 + tt < ntiles ? (int)rowf(t0 + tt, r0 + RSTEP * k) : 0;
#pragma unroll
    for (int tt = 0; tt < GT_GROUP; ++tt) {
      if (t0 + tt >= ntiles) break;
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        const int r = r0 + RSTEP * k;
        const uint32_t dst = gb + (uint32_t)(tt * L::TILE + a * L::ATOM + r * 128 + ((c ^ (r & 7)) << 4));
        const uint16_t* srcp = X + (size_t)src[tt][k] * D + ch * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(srcp));
      }
    }
  };
  double acc[64];
#pragma unroll
  for (int j = 0; j < 64; ++j) acc[j] = 0.0;
  double csum = 0.0;                      // column tid % 128, rows of parity tid / 128
  const int col = tid & (D - 1), rpar = tid >> 7;
  const uint32_t trow = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t tcol = (uint32_t)((warp >> 2) * 64);

  auto flush = [&](int g) {
    const uint32_t t = tmem + trow + 128u * (uint32_t)(g & 1) + tcol;
    uint32_t v[32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tmem_ld32p(t + 32u * h, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) acc[32 * h + e] += (double)__uint_as_float(v[e]);
    }
  };

  bool ok = true;
  load_group(0);
  cp_async_commit();
  for (int g = 0; g < ngroups; ++g) {
    cp_async_wait<0>();
    fence_proxy_async();                   // cp.async (generic proxy) writes -> tensor core reads
    fence_before();
    __syncthreads();
    fence_after();
    const int nt = min(GT_GROUP, ntiles - g * GT_GROUP);
    const uint32_t gb = base + (uint32_t)((g & 1) * L::GROUP);
    if (tid == 0 && ok) {
      const uint32_t d = tmem + 128u * (uint32_t)(g & 1);
      for (int tt = 0; tt < nt; ++tt) {
        const uint64_t dx = sdesc(gb + (uint32_t)(tt * L::TILE), L::ATOM, 1024);
#pragma unroll
        for (int ks = 0; ks < GT_TOK / 16; ++ks) {
          const uint64_t o = (uint64_t)((ks * 2048) >> 4);
          mma_f16(d, dx + o, dx + o, L::IDESC, (tt > 0 || ks > 0) ? 1u : 0u);
        }
      }
      mma_commit(bar0 + 8u * (uint32_t)(g & 1));
    }
    if (g > 0) {
      // the previous group's MMAs done: its ring half can be refilled at once,
      // then its sums are folded into float64 while the loads are in flight
      ok = ok && __all_sync(0xffffffffu, mbar_wait(bar0 + 8u * (uint32_t)((g - 1) & 1), (uint32_t)(((g - 1) >> 1) & 1), status));
      fence_after();
    }
    if (g + 1 < ngroups) load_group(g + 1);
    cp_async_commit();
    if (g > 0) {
      if (ok) flush(g - 1);
      fence_before();
    }
    // column sums of this group (the MMAs read the same tiles)
    {
      const int a = col >> 6, c = (col & 63) >> 3, e = col & 7;
      for (int tt = 0; tt < nt; ++tt) {
        const unsigned char* tp = gsm_raw + (gb - smem_u32(gsm_raw)) + tt * L::TILE + a * L::ATOM;
        if constexpr (EXACT_CS) {
          double s2[2] = {0.0, 0.0};
#pragma unroll 8
          for (int r = rpar, j = 0; r < GT_TOK; r += 2, ++j)
            s2[j & 1] += (double)bf2f(*reinterpret_cast<const uint16_t*>(tp + r * 128 + ((c ^ (r & 7)) << 4) + e * 2));
          csum += s2[0] + s2[1];
        } else {
          float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
          for (int r = rpar, j = 0; r < GT_TOK; r += 2, ++j)
            s4[j & 3] += bf2f(*reinterpret_cast<const uint16_t*>(tp + r * 128 + ((c ^ (r & 7)) << 4) + e * 2));
          csum += (double)((s4[0] + s4[1]) + (s4[2] + s4[3]));
        }
      }
    }
  }
  if (ngroups > 0) {
    const int gl = ngroups - 1;
    ok = ok && __all_sync(0xffffffffu, mbar_wait(bar0 + 8u * (uint32_t)(gl & 1), (uint32_t)((gl >> 1) & 1), status));
    fence_after();
    if (ok) flush(gl);
  }
  if (!ok) atomicExch(&gabort, 1);
  cp_async_wait<0>();
  fence_before();
  __syncthreads();
  fence_after();
  // float64 results: this thread's row of G and its half of a column sum
  {
    const int row = (warp & 3) * 32 + lane, c0 = (warp >> 2) * 64;
    double* o = out + (size_t)row * D + c0;
#pragma unroll
    for (int j = 0; j < 64; ++j) o[j] = acc[j];
  }
  gcs[rpar][col] = csum;
  __syncthreads();
  if (tid < D) out[D * D + tid] = gcs[0][tid] + gcs[1][tid];
  if (gabort && tid == 0 && ngroups > 0) {
    // a wait gave up: one more commit, whose arrival means no MMA of this CTA is in flight
    mma_commit(bar0 + 16);
    mbar_wait(bar0 + 16, 0, status);
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256));
}

}  // namespace tc
}  // namespace spark
