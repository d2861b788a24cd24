// Steps a5-a7 on the sm_100a tensor cores: exact branch, compressed branch,
// merge and un-permute in one kernel (tcgen05.mma + TMEM + TMA).
//
// Work unit: a pair of query blocks of one head = 128 query rows, the M of
// one tcgen05 MMA. The pairs come from pair_kernel: inside windows of 64
// consecutive (permuted) query blocks, blocks are matched greedily by the
// number of selected key blocks they share, so that the union each unit
// walks is small (each row's result does not depend on its partner: the
// partner's blocks carry zero weight for it). The exact branch ("Spark-H3" news
// post, "What Spark-Attn changed": the exact branch fully computes the
// top-ranked key/value blocks) runs over the UNION of the two blocks'
// selected key blocks in ascending order, one 64-key block per tile; the
// rows of a query block that did not select the tile's block give it zero
// weight (that MMA work is not counted as algorithmic). The compressed
// branch ("MiniMax H3 Spark Attention (SM89)", under the hood: a real Q per
// query, K/V downsampled) follows over the summary table, 64 summaries per
// tile, each row masking the blocks it selected. One running softmax over
// both term sets = the log-sum-exp merge of the two branches.
//
// A CTA runs one such unit (SLOTS = 1; the code also runs two units side by
// side, SLOTS = 2) with its own Q, K and V buffers and 256 TMEM columns, and
// two CTAs share an SM: one CTA's prologue (selection masks, Q and first K/V
// loads) and epilogue (O readout, scatter) overlap the other's tiles. The
// slot double-buffers S in TMEM, so the tensor cores compute S_{j+1} (and
// P_{j-1} V_{j-1}) while the slot's softmax works on S_j.
//
// Roles (192 threads; with SLOTS = 2 the softmax warps are 0-7, the
// producers 8-9 and the MMA threads 10-11, 384 threads):
//   warps 0-3  softmax: one thread per query row (TMEM lane = row), the 64
//              columns of a tile. Lazy-rescaled online softmax (the
//              reference max moves only when the row max grows by more
//              than 2^8); P (bf16 pairs) is written over the first 32
//              columns of the tile's S buffer.
//   warp 4     TMA producer: Q once, then K_j and V_j of every tile into
//              two-stage K and V rings.
//   warp 5     MMA-issuing thread (this warp also allocates TMEM):
//              S_j = Q K_j^T (M128 N64 K=d, K-major smem operands),
//              O += P_j V_j (M128 N=d K=64, P read from TMEM, V an MN-major
//              smem operand). S_{j+2} goes into S_j's buffer after P_j V_j;
//              the MMAs of one thread complete in issue order, so that
//              reuse needs no extra wait.
// TMEM columns of slot s (base 256 s): S buffers at +0 and +64, O at +128.
// Every mbarrier wait is bounded (about 2 s); on expiry the kernel records
// a timeout in the status word, drains its own copies and MMAs (again with a
// bound), frees TMEM and returns.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "plan.h"
#include "tc_ptx.cuh"

namespace spark {

// ------------------------------------------------------------------ query-block pairs
// grid (windows of PAIR_WIN query blocks, B*H), 256 threads. The window's
// selection bitmasks in shared memory, the shared-block count of every pair
// of its blocks (each thread keeps its 16 candidates in registers), then
// PAIR_WIN / 2 rounds of: take the free pair with the largest count (ties to
// the lower pair index), the used blocks one 64-bit mask. Unit w * PAIR_WIN / 2 + k of
// the head is the k-th pair taken; an odd window ends with its last free
// block alone (partner -1). Out-of-range selection entries are skipped (the
// attention kernel reports them).
constexpr int PAIR_WIN = 64;

__global__ void __launch_bounds__(256, 1) pair_kernel(const int32_t* __restrict__ sel, int nb, int ksel,
                                                   int2* __restrict__ pairs) {
  static_assert(PAIR_WIN == 64, "pair (i, j) is coded as i * 64 + j; the used set is one 64-bit mask");
  constexpr int KPT = PAIR_WIN * PAIR_WIN / 256;       // candidate pairs per thread
  extern __shared__ uint32_t pm[];                     // [PAIR_WIN][nwords] selection masks
  __shared__ unsigned best_w[2][8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int w = blockIdx.x, bh = blockIdx.y;
  const int b0 = w * PAIR_WIN, m = min(PAIR_WIN, nb - b0);
  const int nwords = (nb + 31) >> 5;
  const int npairs = (nb + 1) >> 1;
  for (int i = tid; i < m * nwords; i += 256) pm[i] = 0u;
  __syncthreads();
  for (int i = tid; i < m * ksel; i += 256) {
    const int r = i / ksel;
    const int b = sel[((size_t)bh * nb + b0 + r) * ksel + (i - r * ksel)];
    if ((unsigned)b < (unsigned)nb) atomicOr(&pm[r * nwords + (b >> 5)], 1u << (b & 31));
  }
  __syncthreads();
  // this thread's candidates q = tid + 256 s, q = i * 64 + j: key = shared
  // count, then the lower q; 0 = not a pair of the window
  unsigned key[KPT];
#pragma unroll
  for (int s = 0; s < KPT; ++s) {
    const int q = tid + 256 * s, i = q >> 6, j = q & 63;
    key[s] = 0u;
    if (i < j && j < m) {
      int c = 0;
      for (int x = 0; x < nwords; ++x) c += __popc(pm[i * nwords + x] & pm[j * nwords + x]);
      key[s] = (1u << 31) | ((unsigned)c << 12) | (unsigned)(4095 - q);
    }
  }
  int2* out = pairs + (size_t)bh * npairs + (size_t)w * (PAIR_WIN / 2);
  unsigned long long usedm = 0ull;
  for (int k = 0; k < m / 2; ++k) {
    unsigned best = 0u;
#pragma unroll
    for (int s = 0; s < KPT; ++s) {
      const int q = tid + 256 * s;
      const bool free = !((usedm >> (q >> 6)) & 1ull) && !((usedm >> (q & 63)) & 1ull);
      if (free) best = max(best, key[s]);
    }
    for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (lane == 0) best_w[k & 1][warp] = best;
    __syncthreads();                                   // best_w[k & 1] is rewritten two rounds on
    unsigned b = 0u;
#pragma unroll
    for (int x = 0; x < 8; ++x) b = max(b, best_w[k & 1][x]);
    const int pq = 4095 - (int)(b & 4095u);
    const int i = pq >> 6, j = pq & 63;
    usedm |= (1ull << i) | (1ull << j);
    if (tid == 0) out[k] = make_int2(b0 + i, b0 + j);
  }
  if ((m & 1) && tid == 0) {
    for (int i = 0; i < m; ++i)
      if (!((usedm >> i) & 1ull)) out[m / 2] = make_int2(b0 + i, -1);
  }
}

namespace tc {

constexpr int ROWS = 128;
constexpr int KEYS = 64;                 // keys (or summaries) per tile = one block
constexpr int SLOTS = 1;                 // units per CTA (two CTAs share an SM)
constexpr int CTAS_PER_SM = 2;
constexpr int STAGES = 2;                // K and V ring depth per slot
constexpr int SM_WARPS = 4 * SLOTS;      // softmax warps: 4 per slot
constexpr int PROD_WARP0 = SM_WARPS;     // TMA producer of slot s: warp PROD_WARP0 + s
constexpr int MMA_WARP0 = SM_WARPS + SLOTS;   // MMA issuer of slot s: warp MMA_WARP0 + s
constexpr int THREADS = 32 * (SM_WARPS + 2 * SLOTS);
constexpr uint32_t SLOT_COLS = 256;      // TMEM columns per slot
constexpr uint32_t TMEM_COLS = SLOT_COLS * SLOTS;
constexpr uint32_t O_OFF = 128;          // O within a slot's columns
constexpr float LAZY_RESCALE = 8.0f;     // log2 units
constexpr int MASK_WORDS = SPARK_MAX_BLOCKS / 32;

template <int D>
struct Layout {
  static constexpr int KATOMS = D / 64;                // 128-byte swizzle atoms along the head dim
  static constexpr int Q_ATOM = ROWS * 128;            // 128 rows x 128 B
  static constexpr int KV_ATOM = KEYS * 128;           // 64 rows x 128 B
  static constexpr int Q_BYTES = Q_ATOM * KATOMS;
  static constexpr int KV_TILE = KV_ATOM * KATOMS;
  // per slot: Q, STAGES K tiles, STAGES V tiles
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_V = Q_BYTES + STAGES * KV_TILE;
  static constexpr int SLOT_BYTES = Q_BYTES + 2 * STAGES * KV_TILE;
  static constexpr int BYTES = SLOTS * SLOT_BYTES;
  static constexpr int SMEM = BYTES + 1024;            // slack for 1024-byte alignment
  static constexpr uint32_t IDESC_S = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(KEYS >> 3) << 17) |
                                      ((uint32_t)(ROWS >> 4) << 24);
  static constexpr uint32_t IDESC_O = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t)(D >> 3) << 17) | ((uint32_t)(ROWS >> 4) << 24);
};

// exp2 on the MUFU unit (flushes subnormal results to zero; a softmax weight
// below 2^-126 of the row maximum is zero in bf16 P anyway).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unf2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// (lo, hi) -> packed bf16x2, lo in the low half, round to nearest even
__device__ __forceinline__ uint32_t cvt_bf2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Next set bit of the union mask at or after block `from`; nb if none.
__device__ __forceinline__ int next_block(const uint32_t* um, int from, int nwords) {
  int w = from >> 5;
  if (w >= nwords) return 1 << 30;
  uint32_t bits = um[w] & (0xFFFFFFFFu << (from & 31));
  while (bits == 0) {
    if (++w >= nwords) return 1 << 30;
    bits = um[w];
  }
  return (w << 5) + __ffs(bits) - 1;
}

struct Maps {
  CUtensorMap q, k, v, kt, vt;  // q: 64-row boxes (the two query blocks of a unit load separately)
  CUtensorMap qc, kc, vc;      // context segment (joint attention); copies of q, k, v when absent
};

// EXT: the block tail granularity or a context segment may be present (an
// instance without them carries none of their per-tile branches).
template <int D, bool EXT>
__global__ void __launch_bounds__(THREADS, CTAS_PER_SM)
attn_tc_kernel(const __grid_constant__ Maps maps, const float* __restrict__ beta, const float* __restrict__ ttab,
               const int32_t* __restrict__ perm, const int32_t* __restrict__ sel, const int2* __restrict__ pairs,
               int N, int nb, int nb_pad, int ksel, uint16_t* __restrict__ out, float* __restrict__ lse, int C,
               int nvid, uint16_t* __restrict__ outc, float* __restrict__ lsec, int* status) {
  using L = Layout<D>;
  constexpr int NBAR = 16;                             // barriers per slot
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t selm[SLOTS][2][MASK_WORDS];
  __shared__ uint32_t unionm[SLOTS][MASK_WORDS];
  __shared__ __align__(8) uint64_t bars[NBAR * SLOTS];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int count_sh[THREADS / 32][SLOTS];
  __shared__ int abort_sh, mma_used_sh[SLOTS];
  __shared__ int issued_sh[SLOTS][2], consumed_sh[SLOTS][2], q_seen_sh[SLOTS];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int npairs = (nb + 1) >> 1;
  const int nwords = (nb + 31) >> 5;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t bar0 = smem_u32(&bars[0]);
  // barrier b of slot s; rings take the stage / buffer index i
  auto bar = [&](int s, int b) { return bar0 + 8u * (uint32_t)(NBAR * s + b); };
  auto q_full = [&](int s) { return bar(s, 0); };
  auto k_full = [&](int s, int i) { return bar(s, 1 + i); };
  auto k_empty = [&](int s, int i) { return bar(s, 3 + i); };
  auto v_full = [&](int s, int i) { return bar(s, 5 + i); };
  auto v_empty = [&](int s, int i) { return bar(s, 7 + i); };
  auto s_full = [&](int s, int i) { return bar(s, 9 + i); };
  auto p_full = [&](int s, int i) { return bar(s, 11 + i); };
  // o_done(s, j & 1) completes with P_j V_j. Two barriers, because when S_j
  // has completed only P_{j-2} V_{j-2} is known to be complete, and a parity
  // wait must never run two phases behind its barrier.
  auto o_done = [&](int s, int i) { return bar(s, 13 + i); };
  auto drain = [&](int s) { return bar(s, 15); };
  auto sQ = [&](int s) { return base + (uint32_t)(s * L::SLOT_BYTES + L::OFF_Q); };
  auto sK = [&](int s, int i) { return base + (uint32_t)(s * L::SLOT_BYTES + L::OFF_K + i * L::KV_TILE); };
  auto sV = [&](int s, int i) { return base + (uint32_t)(s * L::SLOT_BYTES + L::OFF_V + i * L::KV_TILE); };

  // ---- prologue: selection masks of the four query blocks, per-slot unions
  for (int i = tid; i < SLOTS * 2 * MASK_WORDS; i += THREADS) (&selm[0][0][0])[i] = 0u;
  if (tid == 0) {
    abort_sh = 0;
    for (int s = 0; s < SLOTS; ++s) {
      mma_used_sh[s] = 0;
      q_seen_sh[s] = 0;
      issued_sh[s][0] = issued_sh[s][1] = 0;
      consumed_sh[s][0] = consumed_sh[s][1] = 0;
      for (int b = 0; b < NBAR; ++b) mbar_init(bar(s, b), (b == 11 || b == 12) ? ROWS : 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == MMA_WARP0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  __syncthreads();
  // the unit's two query blocks (video CTAs; context CTAs have no pairs)
  static_assert(SLOTS == 1 || SLOTS == 2, "one or two units per CTA");
  auto load_unit = [&](int s) -> int2 {
    const int u = SLOTS * blockIdx.x + s;
    return ((int)blockIdx.x < nvid && u < npairs) ? pairs[(size_t)bh * npairs + u] : make_int2(-1, -1);
  };
  const int2 unit0 = load_unit(0), unit1 = SLOTS > 1 ? load_unit(1) : make_int2(-1, -1);
  auto unit_of = [&](int s) -> int2 { return s == 0 ? unit0 : unit1; };
  for (int qb = 0; qb < 2 * SLOTS; ++qb) {
    const int2 un = unit_of(qb >> 1);
    const int blk = (qb & 1) ? un.y : un.x;
    if ((unsigned)blk >= (unsigned)nb) continue;
    const int32_t* sp = sel + ((size_t)bh * nb + blk) * ksel;
    uint32_t* m = selm[qb >> 1][qb & 1];
    for (int i = tid; i < ksel; i += THREADS) {
      const int b = sp[i];
      if ((unsigned)b < (unsigned)nb) atomicOr(&m[b >> 5], 1u << (b & 31));
      else set_status(status, STATUS_BAD_INPUT);
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  {
    int cs[SLOTS];
#pragma unroll
    for (int s = 0; s < SLOTS; ++s) cs[s] = 0;
    for (int w = tid; w < nwords; w += THREADS) {
#pragma unroll
      for (int s = 0; s < SLOTS; ++s) {
        const uint32_t u = selm[s][0][w] | selm[s][1][w];
        unionm[s][w] = u;
        cs[s] += __popc(u);
      }
    }
#pragma unroll
    for (int s = 0; s < SLOTS; ++s) {
      for (int o = 16; o > 0; o >>= 1) cs[s] += __shfl_xor_sync(0xffffffffu, cs[s], o);
      if (lane == 0) count_sh[warp][s] = cs[s];
    }
  }
  __syncthreads();
  // Tiles of a unit. Video pairs (blockIdx.x < nvid): the union blocks, then
  // the summaries, then the context keys (joint attention, C > 0). Context
  // query chunks (blockIdx.x >= nvid): every video block, then the context keys.
  const bool ctx_cta = EXT && (int)blockIdx.x >= nvid;
  int TE[SLOTS], T[SLOTS], TX[SLOTS];                  // exact (or dense) tiles, all tiles, first context tile
  const int TS = (nb + KEYS - 1) / KEYS;               // summary tiles
  const int TC = EXT ? (C + KEYS - 1) / KEYS : 0;     // context tiles
#pragma unroll
  for (int s = 0; s < SLOTS; ++s) {
    if (!ctx_cta) {
      int U = 0;
      for (int w = 0; w < THREADS / 32; ++w) U += count_sh[w][s];
      TE[s] = U;                                         // exact tiles: one union block each
      TX[s] = U + TS;
      T[s] = (SLOTS * blockIdx.x + s < npairs) ? U + TS + TC : 0;
    } else {
      const int cc = SLOTS * ((int)blockIdx.x - nvid) + s;
      TE[s] = nb;
      TX[s] = nb;
      T[s] = cc * ROWS < C ? nb + TC : 0;
    }
  }
  const uint32_t tmem = tmem_base_sh;

  if (warp < SM_WARPS) {
    // ------------------------------------------------ softmax of slot warp / 4, one thread per row
    const int s = warp >> 2;
    const int Ts = T[s], TEs = TE[s], TXs = TX[s];
    if (Ts > 0) {
      const int crow0 = (SLOTS * ((int)blockIdx.x - nvid) + s) * ROWS;   // context CTAs
      const int r = (warp & 3) * 32 + lane;              // query row 0..127 of the pair
      const int qh = r >> 6;                             // which of the two query blocks
      const int qa = qh ? unit_of(s).y : unit_of(s).x;   // that query block (-1: none)
      // uniform per warp (C - crow0 is a multiple of 32 only at whole warps; rows
      // of a partial warp past C still take part, their results are not written)
      const bool row_valid = ctx_cta ? (crow0 + (warp & 3) * 32 < C) : ((unsigned)qa < (unsigned)nb);
      const uint32_t* mymask = selm[s][qh];
      const uint32_t* um = unionm[s];
      const uint32_t tbase = tmem + ((uint32_t)((warp & 3) * 32) << 16) + SLOT_COLS * (uint32_t)s;
      const uint32_t oc = tbase + O_OFF;
      const float sl2 = (1.0f / sqrtf((float)D)) * 1.4426950408889634f;
      const uint64_t sc2 = f2(sl2, sl2);
      float m_ref = -INFINITY, l = 0.f;
      int cur = ctx_cta ? 0 : next_block(um, 0, nwords);
      bool ok = true;
      for (int j = 0; j < Ts; ++j) {
        const uint32_t sc = tbase + 64u * (uint32_t)(j & 1);   // this tile's S (and P) columns
        // the tile's block (or summary range) and this row's mask, before the wait;
        // kind 0: exact keys, 1: summaries, 2: context keys (per-column masks for 1, 2)
        const int kind = j < TEs ? 0 : ((!EXT || j < TXs) ? 1 : 2);
        const bool comp = kind != 0;
        bool take;
        uint32_t ex0 = ~0u, ex1 = ~0u;
        int c0 = 0;
        if (EXT && kind == 0 && ctx_cta) {
          take = row_valid;                              // dense: every video block
        } else if (kind == 0) {
          const int b = cur;
          cur = next_block(um, b + 1, nwords);
          take = row_valid && ((mymask[b >> 5] >> (b & 31)) & 1u);
        } else if (EXT && kind == 2) {
          const int vc = C - (j - TXs) * KEYS;           // valid context keys in this tile (>= 1)
          take = row_valid;
          ex0 = vc >= 32 ? 0u : (~0u << vc);
          ex1 = vc >= 64 ? 0u : (vc <= 32 ? ~0u : (~0u << (vc - 32)));
        } else {
          c0 = (j - TEs) * KEYS;
          take = row_valid;
          if (row_valid) {
            ex0 = (c0 >> 5) < nwords ? mymask[c0 >> 5] : ~0u;
            ex1 = (c0 >> 5) + 1 < nwords ? mymask[(c0 >> 5) + 1] : ~0u;
            if (c0 + 32 > nb) ex0 |= c0 >= nb ? ~0u : (~0u << (nb - c0));
            if (c0 + 64 > nb) ex1 |= c0 + 32 >= nb ? ~0u : (~0u << (nb - c0 - 32));
          }
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(s_full(s, j & 1), (j >> 1) & 1, status));
        fence_after();
        take = take && ok;                               // uniform per warp
        uint32_t sv[64];
        if (take) {
          tmem_ld32p(sc, sv);
          tmem_ld32p(sc + 32u, sv + 32);
          tmem_ld_wait();
        }
        float mt = -INFINITY;
        if (take) {
          if (!comp) {
            float mc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mc[i] = fmaxf(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]));
#pragma unroll
            for (int c = 16; c < 64; c += 16)
#pragma unroll
              for (int i = 0; i < 8; ++i)
                mc[i] = max3(mc[i], __uint_as_float(sv[c + 2 * i]), __uint_as_float(sv[c + 2 * i + 1]));
            mt = fmaxf(fmaxf(max3(mc[0], mc[1], mc[2]), max3(mc[3], mc[4], mc[5])), fmaxf(mc[6], mc[7])) * sl2;
          } else {
            // x = s / sqrt(d) + beta (log2 units), -inf where the row selected the block;
            // block tail granularity: the query block's precomputed logit row instead;
            // context keys: s / sqrt(d), -inf past the end of the segment
            const bool tab = EXT && kind == 1 && ttab != nullptr;
            const float* brow = (EXT && kind == 2) ? nullptr
                                : tab    ? ttab + ((size_t)bh * nb + qa) * nb_pad + c0
                                         : beta + (size_t)bh * nb_pad + c0;
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
              const float4 bb = brow ? __ldg(reinterpret_cast<const float4*>(brow) + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
              const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = 4 * c4 + e;
                const uint32_t w = c < 32 ? ex0 : ex1;
                const float xs = tab ? bv[e] : fmaf(__uint_as_float(sv[c]), sl2, bv[e] * 1.4426950408889634f);
                const float x = ((w >> (c & 31)) & 1u) ? -INFINITY : xs;
                sv[c] = __float_as_uint(x);
                mt = fmaxf(mt, x);
              }
            }
          }
        }
        // lazy reference maximum
        float m_new = m_ref, corr = 1.f;
        bool resc = false;
        if (mt > -INFINITY) {
          if (m_ref == -INFINITY) {
            m_new = mt;
          } else if (mt > m_ref + LAZY_RESCALE) {
            m_new = mt;
            corr = ex2(m_ref - mt);
            resc = true;
          }
        }
        if (ok && __any_sync(0xffffffffu, resc)) {
          // O in place, once P_{j-1} V_{j-1} has landed (P_j V_j needs P_j: not issued yet)
          if (j > 0) ok = __all_sync(0xffffffffu, mbar_wait(o_done(s, (j - 1) & 1), (uint32_t)((j - 1) >> 1) & 1u, status));
          fence_after();
          if (ok) {
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              tmem_ld32p(oc + 32u * cc, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
              tmem_st32p(oc + 32u * cc, o);
            }
          }
        }
        // P_j (bf16 pairs) over the first 32 columns of the tile's S buffer
        uint32_t pw[32];
        float rs = 0.f;
        if (take && m_new != -INFINITY) {
          const uint64_t mul2 = comp ? f2(1.f, 1.f) : sc2, nm2 = f2(-m_new, -m_new);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            float u0, u1;
            unf2(ffma2(f2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), mul2, nm2), u0, u1);
            const float p0 = ex2(u0), p1 = ex2(u1);
            acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], f2(p0, p1));
            pw[c >> 1] = cvt_bf2(p0, p1);
          }
          float r0, r1, r2, r3;
          unf2(fadd2(acc[0], acc[1]), r0, r1);
          unf2(fadd2(acc[2], acc[3]), r2, r3);
          rs = (r0 + r2) + (r1 + r3);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) pw[c] = 0u;
        }
        l = l * corr + rs;
        m_ref = m_new;
        if (ok) {
          tmem_st32p(sc, pw);
          tmem_st_wait();
          fence_before();
          mbar_arrive(p_full(s, j & 1));
        }
      }
      // ---- epilogue: O / l -> out[perm[row]]
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done(s, (Ts - 1) & 1), (uint32_t)((Ts - 1) >> 1) & 1u, status));
      if (!ok) atomicExch(&abort_sh, 1);
      fence_after();
      ok = __all_sync(0xffffffffu, ok && !(*(volatile int*)&abort_sh));
      if (ok && row_valid) {
        // video rows go to their original index, context rows to their own row
        size_t orow;
        bool dst_ok;
        if (!ctx_cta) {
          const int orig = perm[(size_t)bh * N + qa * BLK + (r & (BLK - 1))];
          dst_ok = (unsigned)orig < (unsigned)N;
          if (!dst_ok) set_status(status, STATUS_BAD_INPUT);
          orow = (size_t)bh * N + (dst_ok ? orig : 0);
        } else {
          dst_ok = crow0 + r < C;
          orow = (size_t)bh * C + (dst_ok ? crow0 + r : 0);
        }
        float* lse_out = ctx_cta ? lsec : lse;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint4* dst = reinterpret_cast<uint4*>((ctx_cta ? outc : out) + orow * D);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32p(oc + 32u * cc, o);
          tmem_ld_wait();
          if (dst_ok) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint32_t w[4];
#pragma unroll
              for (int e2 = 0; e2 < 4; ++e2) {
                const int e = 8 * q4 + 2 * e2;
                w[e2] = cvt_bf2(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
              }
              dst[cc * 4 + q4] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
        if (lse_out != nullptr && dst_ok) lse_out[orow] = (m_ref + log2f(l)) * 0.6931471805599453f;
      }
    }
  } else if (warp < MMA_WARP0) {
    // ------------------------------------------------ TMA producer of slot warp - PROD_WARP0
    const int s = warp - PROD_WARP0;
    if (lane == 0 && T[s] > 0) {
      const int crow0 = (SLOTS * ((int)blockIdx.x - nvid) + s) * ROWS;   // context CTAs
      mbar_arrive_tx(q_full(s), L::Q_BYTES);
      // video unit: the two query blocks' 64 rows each (a lone block fills both halves)
      const int2 un = unit_of(s);
      const int qa0 = un.x, qa1 = un.y >= 0 ? un.y : un.x;
#pragma unroll
      for (int a = 0; a < L::KATOMS; ++a) {
        if (!ctx_cta) {
          tma_load_2d(sQ(s) + a * L::Q_ATOM, &maps.q, 64 * a, bh * N + qa0 * BLK, q_full(s));
          tma_load_2d(sQ(s) + a * L::Q_ATOM + BLK * 128, &maps.q, 64 * a, bh * N + qa1 * BLK, q_full(s));
        } else {
          tma_load_2d(sQ(s) + a * L::Q_ATOM, &maps.qc, 64 * a, bh * C + crow0, q_full(s));
        }
      }
      const uint32_t* um = unionm[s];
      int cur = ctx_cta ? 0 : next_block(um, 0, nwords);
      int ik = 0, iv = 0;
      for (int j = 0; j < T[s]; ++j) {
        const int st = j % STAGES;
        const uint32_t ph = (uint32_t)((j / STAGES) - 1) & 1u;   // phase of the previous use of the stage
        const CUtensorMap *mk, *mv;
        int row;
        if (j < TE[s]) {
          // union block (video pair) or every block in turn (context chunk)
          const int b = ctx_cta ? j : cur;
          row = bh * N + b * BLK;
          if (!ctx_cta) cur = next_block(um, cur + 1, nwords);
          mk = &maps.k;
          mv = &maps.v;
        } else if (!EXT || j < TX[s]) {
          row = bh * nb_pad + (j - TE[s]) * KEYS;
          mk = &maps.kt;
          mv = &maps.vt;
        } else {
          row = bh * C + (j - TX[s]) * KEYS;
          mk = &maps.kc;
          mv = &maps.vc;
        }
        // K_j once S_{j-STAGES} has read the stage
        if (j >= STAGES && !mbar_wait(k_empty(s, st), ph, status)) {
          atomicExch(&abort_sh, 1);
          break;
        }
        if (*(volatile int*)&abort_sh) break;
        mbar_arrive_tx(k_full(s, st), L::KV_TILE);
#pragma unroll
        for (int a = 0; a < L::KATOMS; ++a) tma_load_2d(sK(s, st) + a * L::KV_ATOM, mk, 64 * a, row, k_full(s, st));
        ik = j + 1;
        // V_j once P_{j-STAGES} V_{j-STAGES} has read the stage
        if (j >= STAGES && !mbar_wait(v_empty(s, st), ph, status)) {
          atomicExch(&abort_sh, 1);
          break;
        }
        if (*(volatile int*)&abort_sh) break;
        mbar_arrive_tx(v_full(s, st), L::KV_TILE);
#pragma unroll
        for (int a = 0; a < L::KATOMS; ++a) tma_load_2d(sV(s, st) + a * L::KV_ATOM, mv, 64 * a, row, v_full(s, st));
        iv = j + 1;
      }
      issued_sh[s][0] = ik;
      issued_sh[s][1] = iv;
    }
  } else {
    // ------------------------------------------------ MMA issuer of slot warp - MMA_WARP0
    const int s = warp - MMA_WARP0;
    if (lane == 0 && T[s] > 0) {
      const int Ts = T[s];
      bool ok = true;
      int kc = 0, vc = 0;                                // K / V arrivals observed
      const uint32_t sbase = tmem + SLOT_COLS * (uint32_t)s;
      const uint32_t od = sbase + O_OFF;
      const uint64_t dq = sdesc(sQ(s), 16, 1024);
      // S_j = Q K_j^T into S buffer j & 1
      auto issue_s = [&](int j) -> bool {
        const int st = j % STAGES;
        if (!mbar_wait(k_full(s, st), (uint32_t)(j / STAGES) & 1u, status)) return false;
        kc = j + 1;
        fence_after();
        const uint64_t dk = sdesc(sK(s, st), 16, 1024);
        const uint32_t d = sbase + 64u * (uint32_t)(j & 1);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t qo = (uint64_t)(((ks >> 2) * L::Q_ATOM + (ks & 3) * 32) >> 4);
          const uint64_t ko = (uint64_t)(((ks >> 2) * L::KV_ATOM + (ks & 3) * 32) >> 4);
          mma_f16(d, dq + qo, dk + ko, L::IDESC_S, ks > 0 ? 1u : 0u);
        }
        mma_commit(k_empty(s, st));
        mma_commit(s_full(s, j & 1));
        return true;
      };
      ok = mbar_wait(q_full(s), 0, status);
      if (ok) q_seen_sh[s] = 1;
      if (ok) {
        mma_used_sh[s] = 1;
        ok = issue_s(0);
      }
      if (ok && Ts > 1) ok = issue_s(1);
      for (int j = 0; ok && j < Ts; ++j) {
        const int st = j % STAGES;
        if (!mbar_wait(p_full(s, j & 1), (uint32_t)(j >> 1) & 1u, status)) { ok = false; break; }
        if (!mbar_wait(v_full(s, st), (uint32_t)(j / STAGES) & 1u, status)) { ok = false; break; }
        vc = j + 1;
        fence_after();
        const uint64_t dv = sdesc(sV(s, st), L::KV_ATOM, 1024);
        const uint32_t pa = sbase + 64u * (uint32_t)(j & 1);
#pragma unroll
        for (int kk = 0; kk < KEYS / 16; ++kk)
          mma_ts(od, pa + 8u * kk, dv + (uint64_t)((kk * 2048) >> 4), L::IDESC_O, (kk > 0 || j > 0) ? 1u : 0u);
        mma_commit(v_empty(s, st));
        mma_commit(o_done(s, j & 1));
        // S buffer j & 1 is free again once P_j V_j has read P_j (issue order)
        if (j + 2 < Ts && !issue_s(j + 2)) { ok = false; break; }
      }
      // the last arrivals must land before this CTA's shared memory is released
      for (int jj = Ts - 2; ok && jj < Ts; ++jj) {
        if (jj < 0) continue;
        const uint32_t ph = (uint32_t)(jj / STAGES) & 1u;
        ok = mbar_wait(k_empty(s, jj % STAGES), ph, status) && mbar_wait(v_empty(s, jj % STAGES), ph, status);
      }
      if (ok) ok = mbar_wait(o_done(s, (Ts - 1) & 1), (uint32_t)((Ts - 1) >> 1) & 1u, status);
      if (!ok) atomicExch(&abort_sh, 1);
      consumed_sh[s][0] = kc;
      consumed_sh[s][1] = vc;
    }
  }

  // ---- teardown: drain own copies / MMAs (bounded), free TMEM
  fence_before();
  __syncthreads();
  fence_after();
  if (abort_sh) {
    if (warp >= PROD_WARP0 && warp < MMA_WARP0 && lane == 0) {
      // copies issued but never observed by the MMA thread
      const int s = warp - PROD_WARP0;
      if (T[s] > 0 && !q_seen_sh[s]) mbar_wait(q_full(s), 0, status);
      for (int j = consumed_sh[s][0]; j < issued_sh[s][0]; ++j)
        mbar_wait(k_full(s, j % STAGES), (uint32_t)(j / STAGES) & 1u, status);
      for (int j = consumed_sh[s][1]; j < issued_sh[s][1]; ++j)
        mbar_wait(v_full(s, j % STAGES), (uint32_t)(j / STAGES) & 1u, status);
    }
    if (warp >= MMA_WARP0 && lane == 0 && mma_used_sh[warp - MMA_WARP0]) {
      // one more commit: its arrival means every MMA of this thread has completed
      mma_commit(drain(warp - MMA_WARP0));
      mbar_wait(drain(warp - MMA_WARP0), 0, status);
    }
    fence_before();
    __syncthreads();
    fence_after();
  }
  if (warp == MMA_WARP0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D bf16 map over a [rows, d] row-major matrix, box = 64 columns x box_rows rows, 128B swizzle.
static bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
static cudaError_t run(const Plan& pl, const int32_t* perm, const int32_t* sel, uint16_t* out, float* lse,
                       void* ws, int* status, cudaStream_t s, const JointContext* ctx) {
  using Lay = Layout<D>;
  Maps maps;
  const uint64_t rows = (uint64_t)pl.BH * pl.N, srows = (uint64_t)pl.BH * pl.nb_pad;
  if (pl.nb_pad % KEYS != 0) return cudaErrorInvalidValue;
  if (!make_map(&maps.q, ws_at<void>(ws, pl.off_Qp), rows, D, 64) ||
      !make_map(&maps.k, ws_at<void>(ws, pl.off_Kp), rows, D, 64) ||
      !make_map(&maps.v, ws_at<void>(ws, pl.off_Vp), rows, D, 64) ||
      !make_map(&maps.kt, ws_at<void>(ws, pl.off_kt), srows, D, 64) ||
      !make_map(&maps.vt, ws_at<void>(ws, pl.off_vt), srows, D, 64))
    return cudaErrorInvalidValue;
  const int C = ctx ? ctx->C : 0;
  if (C > 0) {
    const uint64_t crows = (uint64_t)pl.BH * C;
    if (!make_map(&maps.qc, ctx->qc, crows, D, ROWS) || !make_map(&maps.kc, ctx->kc, crows, D, 64) ||
        !make_map(&maps.vc, ctx->vc, crows, D, 64))
      return cudaErrorInvalidValue;
  } else {
    maps.qc = maps.q;
    maps.kc = maps.k;
    maps.vc = maps.v;
  }
  const bool ext = pl.tail == SPARK_TAIL_BLOCK || (ctx != nullptr && ctx->C > 0);
  auto kern = ext ? attn_tc_kernel<D, true> : attn_tc_kernel<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
  if (e != cudaSuccess) return e;
  const int npairs = (pl.nb + 1) / 2;
  const int nvid = (npairs + SLOTS - 1) / SLOTS;
  const int nctx = C > 0 ? ((C + ROWS - 1) / ROWS + SLOTS - 1) / SLOTS : 0;   // context query chunks, two per CTA
  const float* ttab = pl.tail == SPARK_TAIL_BLOCK ? ws_at<float>(ws, pl.off_tail) : nullptr;
  int2* pairs = ws_at<int2>(ws, pl.off_pairs);
  const int nwin = (pl.nb + PAIR_WIN - 1) / PAIR_WIN;
  const size_t pair_smem = sizeof(uint32_t) * PAIR_WIN * (size_t)((pl.nb + 31) / 32);
  e = cudaFuncSetAttribute(pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pair_smem);
  if (e != cudaSuccess) return e;
  pair_kernel<<<dim3(nwin, pl.BH), 256, pair_smem, s>>>(sel, pl.nb, pl.ksel, pairs);
  kern<<<dim3(nvid + nctx, pl.BH), THREADS, Lay::SMEM, s>>>(
      maps, ws_at<float>(ws, pl.off_beta), ttab, perm, sel, pairs, pl.N, pl.nb, pl.nb_pad, pl.ksel, out, lse, C,
      nvid, ctx ? ctx->outc : nullptr, ctx ? ctx->lsec : nullptr, status);
  return cudaGetLastError();
}

}  // namespace tc

cudaError_t launch_attn_tc(const Plan& pl, const int32_t* perm, const int32_t* sel, uint16_t* out, float* lse,
                           void* ws, int* status, cudaStream_t s, const JointContext* ctx) {
  if (pl.d == 128) return tc::run<128>(pl, perm, sel, out, lse, ws, status, s, ctx);
  return tc::run<64>(pl, perm, sel, out, lse, ws, status, s, ctx);
}

}  // namespace spark

