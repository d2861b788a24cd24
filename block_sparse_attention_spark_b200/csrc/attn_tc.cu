// Steps a5-a7 on the sm_100a tensor cores: exact branch, compressed branch,
// merge and un-permute in one kernel (tcgen05.mma + TMEM + TMA).
//
// Work unit: a pair of adjacent query blocks (2p, 2p+1) of one head = 128
// query rows, the M of one tcgen05 MMA. The exact branch ("Spark-H3" news
// post, "What Spark-Attn changed": the exact branch fully computes the
// top-ranked key/value blocks) runs over the UNION of the two blocks'
// selected key blocks in ascending order, two 64-key blocks per 128-key
// tile; a row only keeps the columns of blocks its own query block selected
// (the others get zero weight; that MMA work is not counted as
// algorithmic). The compressed branch ("MiniMax H3 Spark Attention (SM89)",
// under the hood: a real Q per query, K/V downsampled) follows over the
// summary table, 128 summaries per tile, each row masking the blocks it
// selected. One running softmax over both term sets = the log-sum-exp merge
// of the two branches.
//
// Roles (352 threads):
//   warps 0-7  softmax: row r = 32 (w mod 4) + lane is TMEM lane r; warp w
//              takes columns 64 (w / 4) .. +63 of every 128-key S tile, so
//              the two threads of a row exchange their partial row maxima
//              through shared memory once per tile. Lazy-rescaled online
//              softmax (the reference max moves only when the row max grows
//              by more than 2^8); P (bf16 pairs) goes to TMEM.
//   warp 8     TMA producer of Q (once) and the K (or k~) tiles.
//   warp 10    TMA producer of the V (or v~) tiles.
//   warp 9     TMEM allocator + the MMA-issuing thread:
//              S_j = Q K_j^T (M128 N128 K=d, K-major smem operands) into one of
//              two TMEM S buffers; O += P_j V_j (M128 N=d K=128) with P read
//              from TMEM and V an MN-major smem operand.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+d) P0 [384,448) P1 [448,512).
// Every mbarrier wait is bounded (about 2 s); on expiry the kernel records
// a timeout in the status word, drains its own copies and MMAs (again with a
// bound), frees TMEM and returns.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "plan.h"

namespace spark {
namespace tc {

constexpr int ROWS = 128;
constexpr int KEYS = 128;                // keys (or summaries) per tile
constexpr int KSTAGES = 2;
constexpr int VSTAGES = 3;
constexpr int THREADS = 352;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t S_COL = 0;            // S buffer i at S_COL + 128 i
constexpr uint32_t O_COL = 256;
constexpr uint32_t P_COL = 384;          // P buffer i at P_COL + 64 i
constexpr float LAZY_RESCALE = 8.0f;     // log2 units
constexpr unsigned long long WAIT_NS = 2000000000ull;

template <int D>
struct Layout {
  static constexpr int KATOMS = D / 64;                // 128-byte swizzle atoms along the head dim
  static constexpr int Q_ATOM = ROWS * 128;            // 128 rows x 128 B
  static constexpr int KV_ATOM = KEYS * 128;           // 128 rows x 128 B
  static constexpr int Q_BYTES = Q_ATOM * KATOMS;
  static constexpr int KV_TILE = KV_ATOM * KATOMS;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KSTAGES * KV_TILE;
  static constexpr int BYTES = OFF_V + VSTAGES * KV_TILE;
  static constexpr int SMEM = BYTES + 1024;            // slack for 1024-byte alignment
  static constexpr uint32_t IDESC_S = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(KEYS >> 3) << 17) |
                                      ((uint32_t)(ROWS >> 4) << 24);
  static constexpr uint32_t IDESC_O = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t)(D >> 3) << 17) | ((uint32_t)(ROWS >> 4) << 24);
};

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\tmbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; false (and a timeout bit in *status) if the phase never came.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int* status) {
  if (mbar_test(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (!mbar_test(bar, parity)) {
    if (globaltimer() - t0 > WAIT_NS) {
      set_status(status, STATUS_TIMEOUT);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"((uint64_t)map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format:
// start >> 4 at [0,14), leading byte offset >> 4 at [16,30), stride byte
// offset >> 4 at [32,46), version 1 at [46,48), layout 2 = SWIZZLE_128B at [61,64)).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]),
        "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]),
        "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

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
  CUtensorMap q, k, v, kt, vt;
};

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
attn_tc_kernel(const __grid_constant__ Maps maps, const float* __restrict__ beta,
               const int32_t* __restrict__ perm, const int32_t* __restrict__ sel, int N, int nb,
               int nb_pad, int ksel, uint16_t* __restrict__ out, float* __restrict__ lse, int* status) {
  using L = Layout<D>;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t selm[2][SPARK_MAX_BLOCKS / 32];
  __shared__ uint32_t unionm[SPARK_MAX_BLOCKS / 32];
  __shared__ __align__(8) uint64_t bars[2 * KSTAGES + 2 * VSTAGES + 8];
  __shared__ float red_max[2][2][ROWS];   // [tile parity][column half][row]
  __shared__ float red_l[2][ROWS];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int count_sh[12];
  __shared__ int abort_sh;
  __shared__ int issued_sh[2], consumed_sh[2], q_seen_sh, mma_used_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int a0 = 2 * pair, a1 = 2 * pair + 1;
  const bool half1_valid = a1 < nb;
  const int nwords = (nb + 31) >> 5;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + L::OFF_Q, sK = base + L::OFF_K, sV = base + L::OFF_V;
  const uint32_t bar0 = smem_u32(&bars[0]);
  auto k_full = [&](int s) { return bar0 + 8u * s; };
  auto k_empty = [&](int s) { return bar0 + 8u * (KSTAGES + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (2 * KSTAGES + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (2 * KSTAGES + VSTAGES + s); };
  const uint32_t bx = bar0 + 8u * (2 * KSTAGES + 2 * VSTAGES);
  const uint32_t q_full = bx;
  auto s_full = [&](int i) { return bx + 8u * (1 + i); };
  auto p_full = [&](int i) { return bx + 8u * (3 + i); };
  const uint32_t o_done = bx + 8u * 5;
  const uint32_t drain = bx + 8u * 6;

  // ---- prologue: selection masks of both query blocks, their union
  for (int i = tid; i < SPARK_MAX_BLOCKS / 32; i += THREADS) { selm[0][i] = 0u; selm[1][i] = 0u; }
  if (tid == 0) {
    abort_sh = 0; q_seen_sh = 0; mma_used_sh = 0;
    issued_sh[0] = issued_sh[1] = 0; consumed_sh[0] = consumed_sh[1] = 0;
    for (int s = 0; s < KSTAGES; ++s) { mbar_init(k_full(s), 1); mbar_init(k_empty(s), 1); }
    for (int s = 0; s < VSTAGES; ++s) { mbar_init(v_full(s), 1); mbar_init(v_empty(s), 1); }
    mbar_init(q_full, 1);
    mbar_init(s_full(0), 1); mbar_init(s_full(1), 1);
    mbar_init(p_full(0), 256); mbar_init(p_full(1), 256);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_sh)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  __syncthreads();
  {
    const int32_t* s0 = sel + ((size_t)bh * nb + a0) * ksel;
    for (int i = tid; i < ksel; i += THREADS) {
      const int b = s0[i];
      if ((unsigned)b < (unsigned)nb) atomicOr(&selm[0][b >> 5], 1u << (b & 31));
      else set_status(status, STATUS_BAD_INPUT);
    }
    if (half1_valid) {
      const int32_t* s1 = sel + ((size_t)bh * nb + a1) * ksel;
      for (int i = tid; i < ksel; i += THREADS) {
        const int b = s1[i];
        if ((unsigned)b < (unsigned)nb) atomicOr(&selm[1][b >> 5], 1u << (b & 31));
        else set_status(status, STATUS_BAD_INPUT);
      }
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  int cnt = 0;
  for (int w = tid; w < nwords; w += THREADS) {
    const uint32_t u = selm[0][w] | selm[1][w];
    unionm[w] = u;
    cnt += __popc(u);
  }
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) count_sh[warp] = cnt;
  __syncthreads();
  int U = 0;
  for (int w = 0; w < THREADS / 32; ++w) U += count_sh[w];
  const int TE = (U + 1) >> 1;                         // exact tiles (two union blocks each)
  const int T = TE + (nb + KEYS - 1) / KEYS;           // plus summary tiles
  const uint32_t tmem = tmem_base_sh;
  constexpr int NONE = 1 << 30;

  if (warp == 8 || warp == 10) {
    // ------------------------------------------------ TMA producers (warp 8: Q and K, warp 10: V)
    const int pidx = warp == 8 ? 0 : 1;
    if (lane == 0) {
      const bool isk = pidx == 0;
      const int stages = isk ? KSTAGES : VSTAGES;
      if (isk) {
        const int qrow = bh * N + a0 * BLK;
        mbar_arrive_tx(q_full, L::Q_BYTES);
#pragma unroll
        for (int a = 0; a < L::KATOMS; ++a) tma_load_2d(sQ + a * L::Q_ATOM, &maps.q, 64 * a, qrow, q_full);
      }
      const uint32_t ring = isk ? sK : sV;
      int cur = next_block(unionm, 0, nwords);
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % stages;
        const uint32_t empty = isk ? k_empty(st) : v_empty(st);
        const uint32_t full = isk ? k_full(st) : v_full(st);
        if (j >= stages && !mbar_wait(empty, ((j / stages) - 1) & 1, status)) {
          atomicExch(&abort_sh, 1);
          break;
        }
        if (*(volatile int*)&abort_sh) break;
        const uint32_t dst = ring + st * L::KV_TILE;
        mbar_arrive_tx(full, L::KV_TILE);
        const CUtensorMap* m;
        int row0, row1;
        if (j < TE) {
          const int b0 = cur;
          int b1 = next_block(unionm, b0 + 1, nwords);
          cur = b1 < NONE ? next_block(unionm, b1 + 1, nwords) : NONE;
          if (b1 >= NONE) b1 = b0;                   // odd count: the second half repeats, masked
          row0 = bh * N + b0 * BLK;
          row1 = bh * N + b1 * BLK;
          m = isk ? &maps.k : &maps.v;
        } else {
          row0 = bh * nb_pad + (j - TE) * KEYS;
          row1 = row0 + BLK;
          m = isk ? &maps.kt : &maps.vt;
        }
#pragma unroll
        for (int a = 0; a < L::KATOMS; ++a) {
          tma_load_2d(dst + a * L::KV_ATOM, m, 64 * a, row0, full);
          tma_load_2d(dst + a * L::KV_ATOM + BLK * 128, m, 64 * a, row1, full);
        }
        issued = j + 1;
      }
      issued_sh[pidx] = issued;
    }
  } else if (warp == 9) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, status);
      if (ok) q_seen_sh = 1;
      int kc = 0, vc = 0;   // K / V tiles whose arrival was observed
      const uint64_t dQ0 = sdesc(sQ, 16, 1024);
      const uint64_t dK0 = sdesc(sK, 16, 1024);
      const uint64_t dV0 = sdesc(sV, L::KV_ATOM, 1024);
      auto issue_s = [&](int j) -> bool {
        const int st = j % KSTAGES;
        if (!mbar_wait(k_full(st), (j / KSTAGES) & 1, status)) return false;
        kc = j + 1;
        fence_after();
        const uint32_t d = tmem + S_COL + 128u * (uint32_t)(j & 1);
        const uint64_t dk = dK0 + (uint64_t)((st * L::KV_TILE) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t qo = (uint64_t)(((ks >> 2) * L::Q_ATOM + (ks & 3) * 32) >> 4);
          const uint64_t ko = (uint64_t)(((ks >> 2) * L::KV_ATOM + (ks & 3) * 32) >> 4);
          mma_f16(d, dQ0 + qo, dk + ko, L::IDESC_S, ks > 0 ? 1u : 0u);
        }
        mma_commit(s_full(j & 1));
        mma_commit(k_empty(st));
        mma_used_sh = 1;
        return true;
      };
      if (ok && T > 0) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % VSTAGES;
        if (!mbar_wait(p_full(j & 1), (j >> 1) & 1, status)) { ok = false; break; }
        if (!mbar_wait(v_full(st), (j / VSTAGES) & 1, status)) { ok = false; break; }
        vc = j + 1;
        fence_after();
        const uint64_t dv = dV0 + (uint64_t)((st * L::KV_TILE) >> 4);
        const uint32_t pa = tmem + P_COL + 64u * (uint32_t)(j & 1);
        const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < KEYS / 16; ++kk)
          mma_ts(tmem + O_COL, pa + 8u * kk, dv + (uint64_t)((kk * 2048) >> 4), L::IDESC_O, kk > 0 ? 1u : acc0);
        mma_commit(o_done);
        mma_commit(v_empty(st));
        // S buffer j&1 is free again (the softmax read S_j before releasing P_j)
        if (j + 2 < T && !issue_s(j + 2)) { ok = false; break; }
      }
      if (ok && T > 0) {
        // the last commit must land before this CTA's shared memory is released
        const int jl = T - 1;
        ok = mbar_wait(v_empty(jl % VSTAGES), (jl / VSTAGES) & 1, status);
      }
      if (!ok) atomicExch(&abort_sh, 1);
      consumed_sh[0] = kc;
      consumed_sh[1] = vc;
    }
  } else {
    // ------------------------------------------------ softmax warps 0-7
    const int h = warp >> 2;                 // column half of the 128-key tile
    const int r = (warp & 3) * 32 + lane;    // query row 0..127 of the pair
    const int qh = r >> 6;                   // which of the two query blocks
    const bool row_valid = qh == 0 || half1_valid;   // uniform per warp
    const uint32_t* mymask = selm[qh];
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = (1.0f / sqrtf((float)D)) * 1.4426950408889634f;
    float m_ref = -INFINITY, l = 0.f;
    int cur = next_block(unionm, 0, nwords);
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      // (a warp that gave up keeps taking part in the named barriers)
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(s_full(j & 1), (j >> 1) & 1, status));
      fence_after();
      uint32_t sa[32], sb[32];
      if (ok) {
        tmem_ld32(tmem + lane_base + S_COL + 128u * (uint32_t)(j & 1) + 64u * h, sa);
        tmem_ld32(tmem + lane_base + S_COL + 128u * (uint32_t)(j & 1) + 64u * h + 32u, sb);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) { sa[c] = 0u; sb[c] = 0u; }
      }
      auto sv = [&](int c) { return __uint_as_float(c < 32 ? sa[c] : sb[c - 32]); };
      bool take = false, comp = j >= TE;
      uint64_t excl = 0;
      float x[64];
      float mx = -INFINITY;
      if (!comp) {
        const int b0 = cur;
        const int b1 = next_block(unionm, b0 + 1, nwords);
        cur = b1 < NONE ? next_block(unionm, b1 + 1, nwords) : NONE;
        const int blk = h == 0 ? b0 : b1;
        take = row_valid && blk < NONE && ((mymask[blk >> 5] >> (blk & 31)) & 1u);   // uniform per warp
        if (take) {
          float mc[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) mc[i] = fmaxf(sv(2 * i), sv(2 * i + 1));
#pragma unroll
          for (int c = 8; c < 64; c += 8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) mc[i] = max3(mc[i], sv(c + 2 * i), sv(c + 2 * i + 1));
          }
          mx = fmaxf(max3(mc[0], mc[1], mc[2]), mc[3]) * sl2;
        }
      } else {
        const int c0 = (j - TE) * KEYS + 64 * h;
        if (c0 < nb) {
          excl = (uint64_t)mymask[c0 >> 5];
          if ((c0 >> 5) + 1 < nwords) excl |= (uint64_t)mymask[(c0 >> 5) + 1] << 32;
          if (c0 + BLK > nb) excl |= ~0ull << (nb - c0);
        } else {
          excl = ~0ull;
        }
        if (!row_valid) excl = ~0ull;
        const float4* bt = reinterpret_cast<const float4*>(beta + (size_t)bh * nb_pad + c0);
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 bb = __ldg(bt + c4);
          const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * c4 + e;
            const float v = fmaf(sv(c), sl2, bv[e] * 1.4426950408889634f);
            x[c] = ((excl >> c) & 1ull) ? -INFINITY : v;
            mx = fmaxf(mx, x[c]);
          }
        }
      }
      // row max over both column halves
      red_max[j & 1][h][r] = mx;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      const float mt = fmaxf(red_max[j & 1][0][r], red_max[j & 1][1][r]);
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
      uint32_t pw[32];
      float rs = 0.f;
      if (!comp && take) {
        const uint64_t sc2 = f2(sl2, sl2), nm2 = f2(-m_new, -m_new);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float t0, t1;
          unf2(ffma2(f2(sv(c), sv(c + 1)), sc2, nm2), t0, t1);
          const float p0 = ex2(t0), p1 = ex2(t1);
          acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], f2(p0, p1));
          pw[c >> 1] = cvt_bf2(p0, p1);
        }
        float r0, r1, r2, r3;
        unf2(fadd2(acc[0], acc[1]), r0, r1);
        unf2(fadd2(acc[2], acc[3]), r2, r3);
        rs = (r0 + r2) + (r1 + r3);
      } else if (comp && m_new != -INFINITY) {
        float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float p0 = ex2(x[c] - m_new), p1 = ex2(x[c + 1] - m_new);
          rs4[(c >> 1) & 3] += p0 + p1;
          pw[c >> 1] = cvt_bf2(p0, p1);
        }
        rs = (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pw[c] = 0u;
      }
      l = l * corr + rs;
      m_ref = m_new;
      // previous P V product complete: O may be rescaled, P buffer j&1 reused
      if (ok && j > 0) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, status));
      fence_after();
      if (ok) {
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int cc = 0; cc < 2; ++cc) {
            const uint32_t oc = tmem + lane_base + O_COL + 64u * h + 32u * cc;
            if (64 * h + 32 * cc < D) {
              uint32_t o[32];
              tmem_ld32(oc, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
              tmem_st32(oc, o);
            }
          }
          tmem_st_wait();
        }
        tmem_st32(tmem + lane_base + P_COL + 64u * (uint32_t)(j & 1) + 32u * h, pw);
        tmem_st_wait();
        fence_before();
        mbar_arrive(p_full(j & 1));
      }
    }
    // ---- epilogue: O / l -> out[perm[row]], each thread its 64 columns
    if (ok && T > 0) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (T - 1) & 1, status));
    if (!ok) atomicExch(&abort_sh, 1);
    fence_after();
    red_l[h][r] = l;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    const float lt = red_l[0][r] + red_l[1][r];
    ok = ok && !(*(volatile int*)&abort_sh);
    if (ok && row_valid && 64 * h < D) {
      const int pos = a0 * BLK + r;
      const int orig = perm[(size_t)bh * N + pos];
      const bool dst_ok = (unsigned)orig < (unsigned)N;
      if (!dst_ok) set_status(status, STATUS_BAD_INPUT);
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)bh * N + (dst_ok ? orig : 0)) * D + 64 * h);
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + O_COL + 64u * h + 32u * cc, o);
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
      if (h == 0 && lse != nullptr && dst_ok) lse[(size_t)bh * N + orig] = (m_ref + log2f(lt)) * 0.6931471805599453f;
    }
  }

  // ---- teardown: drain own copies / MMAs (bounded), free TMEM
  fence_before();
  __syncthreads();
  fence_after();
  if (abort_sh) {
    if ((warp == 8 || warp == 10) && lane == 0) {
      // copies issued but never observed by the MMA thread
      const int pi = warp == 8 ? 0 : 1;
      const int stages = pi == 0 ? KSTAGES : VSTAGES;
      if (pi == 0 && !q_seen_sh) mbar_wait(q_full, 0, status);
      for (int j = consumed_sh[pi]; j < issued_sh[pi]; ++j)
        mbar_wait(pi == 0 ? k_full(j % stages) : v_full(j % stages), (j / stages) & 1, status);
    }
    if (warp == 9 && lane == 0 && mma_used_sh) {
      mma_commit(drain);
      mbar_wait(drain, 0, status);
    }
    fence_before();
    __syncthreads();
    fence_after();
  }
  if (warp == 9) {
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
                       void* ws, int* status, cudaStream_t s) {
  using Lay = Layout<D>;
  Maps maps;
  const uint64_t rows = (uint64_t)pl.BH * pl.N, srows = (uint64_t)pl.BH * pl.nb_pad;
  if (pl.nb_pad % KEYS != 0) return cudaErrorInvalidValue;
  if (!make_map(&maps.q, ws_at<void>(ws, pl.off_Qp), rows, D, ROWS) ||
      !make_map(&maps.k, ws_at<void>(ws, pl.off_Kp), rows, D, 64) ||
      !make_map(&maps.v, ws_at<void>(ws, pl.off_Vp), rows, D, 64) ||
      !make_map(&maps.kt, ws_at<void>(ws, pl.off_kt), srows, D, 64) ||
      !make_map(&maps.vt, ws_at<void>(ws, pl.off_vt), srows, D, 64))
    return cudaErrorInvalidValue;
  auto kern = attn_tc_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<dim3((pl.nb + 1) / 2, pl.BH), THREADS, Lay::SMEM, s>>>(maps, ws_at<float>(ws, pl.off_beta), perm, sel,
                                                                 pl.N, pl.nb, pl.nb_pad, pl.ksel, out, lse, status);
  return cudaGetLastError();
}

}  // namespace tc

cudaError_t launch_attn_tc(const Plan& pl, const int32_t* perm, const int32_t* sel, uint16_t* out, float* lse,
                           void* ws, int* status, cudaStream_t s) {
  if (pl.d == 128) return tc::run<128>(pl, perm, sel, out, lse, ws, status, s);
  return tc::run<64>(pl, perm, sel, out, lse, ws, status, s);
}

}  // namespace spark

