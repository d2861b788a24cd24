// Gram-matrix tiles G += X^T X over 64-token tiles, used by the moments and
// the reblock kernels. 256 threads (8 warps); each warp owns a (D/4) x (D/2)
// patch of the D x D output. Per tile the legacy tensor-core mma.sync path
// accumulates in float32 registers; every FLUSH tiles the float32 partials
// are added into per-thread float64 accumulators kept in shared memory, so
// long token ranges keep float64 accuracy apart from the short float32 sums.
#pragma once

#include "common.cuh"

namespace spark {

template <int D>
struct Gram {
  static constexpr int THREADS = 256;
  static constexpr int WM = D / 4, WN = D / 2;
  static constexpr int MT = WM / 16, NT = WN / 8;
  static constexpr int RS = D + 8;                 // padded smem row (elements): conflict-free ldmatrix
  static constexpr int TILE = BLK * RS;            // elements per staged tile
  static constexpr int ACC = MT * NT * 4;          // float32 accumulators per thread
  static constexpr int CHUNKS = BLK * (D / 8);     // 16-byte chunks per tile
  static constexpr int FLUSH = 4;                  // tiles between float64 flushes
  static_assert(NT % 2 == 0, "pairs of n8 tiles");

  // Stage 64 rows of D bf16 into smem. rows[r] (if non-null) gives the source
  // row of tile row r, else row0 + r. base points at row 0 of the matrix.
  // Thread tid copies chunk tid % (D / 8) of rows tid / (D / 8) + RSTEP k;
  // all of its row indices are read before the first copy is issued.
  static constexpr int RSTEP = THREADS / (D / 8), LROWS = BLK / RSTEP;
  static_assert(CHUNKS % THREADS == 0, "whole chunks per thread");
  __device__ static void load_tile(uint16_t* sm, const uint16_t* base, const int32_t* rows,
                                   long row0, int tid) {
    const int ch = tid % (D / 8), r0 = tid / (D / 8);
    long src[LROWS];
#pragma unroll
    for (int k = 0; k < LROWS; ++k) src[k] = rows ? (long)rows[r0 + RSTEP * k] : row0 + r0 + RSTEP * k;
#pragma unroll
    for (int k = 0; k < LROWS; ++k) cp_async16(sm + (r0 + RSTEP * k) * RS + ch * 8, base + src[k] * D + ch * 8);
  }

  __device__ static void tile_mma(const uint16_t* sm, float (&acc)[ACC], int warp, int lane) {
    const int m0 = (warp % 4) * WM, n0 = (warp / 4) * WN;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const int t0 = ks * 16;
      uint32_t a[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
        ldsm_x4_t(a[mt][0], a[mt][1], a[mt][2], a[mt][3],
                  sm + (t0 + (lane & 7) + (lane >> 4) * 8) * RS + m0 + mt * 16 + ((lane >> 3) & 1) * 8);
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3,
                  sm + (t0 + (lane & 7) + ((lane >> 3) & 1) * 8) * RS + n0 + np * 16 + (lane >> 4) * 8);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma_bf16(&acc[(mt * NT + 2 * np) * 4], a[mt], b0, b1);
          mma_bf16(&acc[(mt * NT + 2 * np + 1) * 4], a[mt], b2, b3);
        }
      }
    }
  }

  // acc64 layout: [ACC][THREADS] doubles (thread-private columns).
  __device__ static void flush(float (&acc)[ACC], double* acc64, int tid) {
#pragma unroll
    for (int j = 0; j < ACC; ++j) {
      acc64[j * THREADS + tid] += (double)acc[j];
      acc[j] = 0.f;
    }
  }

  // (row, col) of accumulator j of this thread.
  __device__ static void coord(int j, int warp, int lane, int& row, int& col) {
    const int r = j & 3, nt = (j >> 2) % NT, mt = (j >> 2) / NT;
    row = (warp % 4) * WM + mt * 16 + (lane >> 2) + ((r >> 1) << 3);
    col = (warp / 4) * WN + nt * 8 + 2 * (lane & 3) + (r & 1);
  }
};

}  // namespace spark
