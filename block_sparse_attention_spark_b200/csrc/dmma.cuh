// Float64 tensor-core helpers (mma.sync m16n8k16 .f64) for the steps whose
// results must reproduce a float64 evaluation: the second moment that the
// partition whitens with, and the whitened tokens themselves. A bf16 value is
// exact in float64 and so is the product of two of them, so these Gram sums
// and products carry only float64 rounding, like the plain definition.
//
// Fragment layout of D(16x8) += A(16x16) B(16x8), lane = 4 g + t (g = lane / 4,
// t = lane % 4):
//   a[i] = A[g + 8 (i % 2)][t + 4 (i / 2)],  i = 0..7
//   b[i] = B[t + 4 i][g],                    i = 0..3
//   c[i] = D[g + 8 (i / 2)][2 t + (i % 2)],  i = 0..3
// Operand tiles live in shared memory as float64 rows with a leading
// dimension of D + 4 doubles: for every fragment above, the 16 lanes of a
// half-warp then hit 16 distinct bank pairs.
#pragma once

#include "common.cuh"

namespace spark {

__device__ __forceinline__ void dmma16816(double (&c)[4], const double (&a)[8], const double (&b)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7,%8,%9,%10,%11}, {%12,%13,%14,%15}, {%0,%1,%2,%3};\n"
      : "+d"(c[0]), "+d"(c[1]), "+d"(c[2]), "+d"(c[3])
      : "d"(a[0]), "d"(a[1]), "d"(a[2]), "d"(a[3]), "d"(a[4]), "d"(a[5]), "d"(a[6]), "d"(a[7]),
        "d"(b[0]), "d"(b[1]), "d"(b[2]), "d"(b[3]));
}

// Eight bf16 (one 16-byte chunk) widened to float64 and stored to shared
// memory as four 16-byte pairs. When the lanes of a warp hold consecutive
// chunks of a row, their destinations are 64 bytes apart; each lane stores
// its pairs in an order rotated by lane / 2, so that the eight lanes of a
// quarter-warp hit eight different 16-byte bank groups at every step.
__device__ __forceinline__ void bf8_to_f64(const uint4 w, double* dst, int lane) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = (i + (lane >> 1)) & 3;
    const uint32_t x = e == 0 ? w.x : e == 1 ? w.y : e == 2 ? w.z : w.w;
    reinterpret_cast<double2*>(dst)[e] = make_double2((double)bf_lo(x), (double)bf_hi(x));
  }
}

// The upper-triangle tiles of a symmetric D x D product in units of
// (16-row tile r, 8-column tile c) with c >= 2 r: every entry (i, j), i <= j,
// lies in exactly one of them. Enumerated row by row; pair p of the list.
template <int D>
struct TriTiles {
  static constexpr int RT = D / 16, CT = D / 8;
  static constexpr int PAIRS = RT * CT - RT * (RT - 1);
  __device__ static void decode(int p, int& r, int& c) {
    r = 0;
    int first = 0;
    while (r < RT - 1 && p >= first + (CT - 2 * r)) {
      first += CT - 2 * r;
      ++r;
    }
    c = 2 * r + (p - first);
  }
};

}  // namespace spark
