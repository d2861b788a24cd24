// Steps a5-a7 on the sm_100a tensor cores: exact branch, compressed branch,
// merge and un-permute in one kernel (tcgen05.mma + TMEM + TMA).
//
// Work unit: a pair of adjacent query blocks (2p, 2p+1) of one head = 128
// query rows, the M of one tcgen05 MMA. The exact branch ("Spark-H3" news
// post, "What Spark-Attn changed": the exact branch fully computes the
// top-ranked key/value blocks) runs over the UNION of the two blocks'
// selected key blocks in ascending order; a row only keeps the columns of
// blocks its own query block selected (the other half's scores are masked to
// zero weight, so the extra MMA work is not counted as algorithmic). The
// compressed branch ("MiniMax H3 Spark Attention (SM89)", under the hood: a
// real Q per query, K/V downsampled) follows over the summary tiles, each
// row masking the blocks it selected. One running softmax over both term
// sets = the log-sum-exp merge of the two branches.
//
// Roles (320 threads):
//   warps 0-7  two softmax warpgroups; warpgroup g takes tiles j = g, g+2, ...
//              and keeps its own running (max, sum) and its own O accumulator
//              in TMEM. Thread r of a warpgroup owns query row r = TMEM lane
//              r: reads S, masks, lazy-rescaled online softmax (rescale only
//              when the running max grows by more than 2^8), writes P (bf16)
//              to smem. Epilogue: the two partial softmaxes are merged by
//              log-sum-exp, O / l -> out[perm[row]].
//   warp 8     TMA producers: lane 0 loads Q once and then the K (or k~)
//              tiles, lane 1 the V (or v~) tiles, each into its own
//              STAGES-deep ring of 128B-swizzled smem tiles; a K slot is freed
//              as soon as its S MMA completes, a V slot after its P V MMA.
//   warp 9     TMEM allocator + one MMA-issuing thread:
//              S_j = Q K_j^T (M128 N64 K=d) into a double-buffered TMEM tile,
//              O_g += P_j V_j (M128 N=d K=64, g = j mod 2) with V as an MN-major operand.
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
constexpr int STAGES = 4;
constexpr int THREADS = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t O_COL = 128;          // O of warpgroup g at O_COL + 128 g
constexpr float LAZY_RESCALE = 8.0f;    // log2 units
constexpr unsigned long long WAIT_NS = 2000000000ull;

template <int D>
struct Layout {
  static constexpr int KATOMS = D / 64;                // 128-byte swizzle atoms along the head dim
  static constexpr int Q_ATOM = ROWS * 128;            // bytes per Q atom (128 rows x 128 B)
  static constexpr int KV_ATOM = 64 * 128;             // bytes per K or V atom (64 rows x 128 B)
  static constexpr int Q_BYTES = Q_ATOM * KATOMS;
  static constexpr int KV_TILE = KV_ATOM * KATOMS;     // one K (or V) tile
  static constexpr int P_BYTES = ROWS * 128;           // 128 rows x 64 bf16
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;        // K ring: STAGES tiles
  static constexpr int OFF_V = OFF_K + STAGES * KV_TILE;   // V ring: STAGES tiles
  static constexpr int OFF_P = OFF_V + STAGES * KV_TILE;
  static constexpr int BYTES = OFF_P + 2 * P_BYTES;
  static constexpr int SMEM = BYTES + 1024;            // slack for 1024-byte alignment
  static constexpr uint32_t IDESC_S = (1u << 4) | (1u << 7) | (1u << 10) | ((64u >> 3) << 17) |
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
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
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
  __shared__ __align__(8) uint64_t bars[4 * STAGES + 8];
  __shared__ float m1_sh[ROWS], l1_sh[ROWS];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int count_sh[8];
  __shared__ int abort_sh;
  __shared__ int issued_sh[2], consumed_sh[2], q_seen_sh, mma_used_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int a0 = 2 * pair, a1 = 2 * pair + 1;
  const bool half1_valid = a1 < nb;
  const int nwords = (nb + 31) >> 5;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + L::OFF_Q, sK = base + L::OFF_K, sV = base + L::OFF_V, sP = base + L::OFF_P;
  const uint32_t bar0 = smem_u32(&bars[0]);
  auto k_full = [&](int s) { return bar0 + 8u * s; };
  auto k_empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (3 * STAGES + s); };
  const uint32_t q_full = bar0 + 8u * (4 * STAGES);
  auto s_full = [&](int i) { return bar0 + 8u * (4 * STAGES + 1 + i); };
  auto p_full = [&](int i) { return bar0 + 8u * (4 * STAGES + 3 + i); };
  auto o_done = [&](int g) { return bar0 + 8u * (4 * STAGES + 5 + g); };
  const uint32_t drain = bar0 + 8u * (4 * STAGES + 7);

  // ---- prologue: selection masks of both query blocks, their union
  for (int i = tid; i < SPARK_MAX_BLOCKS / 32; i += THREADS) { selm[0][i] = 0u; selm[1][i] = 0u; }
  if (tid == 0) {
    abort_sh = 0; q_seen_sh = 0; mma_used_sh = 0;
    issued_sh[0] = issued_sh[1] = 0; consumed_sh[0] = consumed_sh[1] = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(k_full(s), 1); mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1); mbar_init(v_empty(s), 1);
    }
    mbar_init(q_full, 1);
    mbar_init(s_full(0), 1); mbar_init(s_full(1), 1);
    mbar_init(p_full(0), 128); mbar_init(p_full(1), 128);
    mbar_init(o_done(0), 1); mbar_init(o_done(1), 1);
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
  const int ncomp = (nb + BLK - 1) / BLK;
  const int T = U + ncomp;
  const uint32_t tmem = tmem_base_sh;

  if (warp == 8) {
    // ------------------------------------------------ TMA producers (lane 0: Q, K; lane 1: V)
    if (lane < 2) {
      const bool isk = lane == 0;
      if (isk) {
        const int qrow = bh * N + a0 * BLK;
        mbar_arrive_tx(q_full, L::Q_BYTES);
#pragma unroll
        for (int a = 0; a < L::KATOMS; ++a) tma_load_2d(sQ + a * L::Q_ATOM, &maps.q, 64 * a, qrow, q_full);
      }
      const uint32_t ring = isk ? sK : sV;
      int b = next_block(unionm, 0, nwords);
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % STAGES;
        const uint32_t empty = isk ? k_empty(st) : v_empty(st);
        const uint32_t full = isk ? k_full(st) : v_full(st);
        if (j >= STAGES && !mbar_wait(empty, ((j / STAGES) - 1) & 1, status)) {
          atomicExch(&abort_sh, 1);
          break;
        }
        if (*(volatile int*)&abort_sh) break;
        const uint32_t dst = ring + st * L::KV_TILE;
        mbar_arrive_tx(full, L::KV_TILE);
        const CUtensorMap* m;
        int row;
        if (j < U) {
          row = bh * N + b * BLK;
          m = isk ? &maps.k : &maps.v;
          b = next_block(unionm, b + 1, nwords);
        } else {
          row = bh * nb_pad + (j - U) * BLK;
          m = isk ? &maps.kt : &maps.vt;
        }
#pragma unroll
        for (int a = 0; a < L::KATOMS; ++a) tma_load_2d(dst + a * L::KV_ATOM, m, 64 * a, row, full);
        issued = j + 1;
      }
      issued_sh[lane] = issued;
    }
  } else if (warp == 9) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, status);
      if (ok) q_seen_sh = 1;
      int kc = 0, vc = 0;   // K / V tiles whose arrival was observed
      auto issue_s = [&](int j) -> bool {
        const int st = j % STAGES;
        if (!mbar_wait(k_full(st), (j / STAGES) & 1, status)) return false;
        kc = j + 1;
        fence_after();
        const uint32_t kaddr = sK + st * L::KV_TILE;
        const uint32_t d = tmem + (uint32_t)((j & 1) * 64);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t da = sdesc(sQ + (ks >> 2) * L::Q_ATOM + (ks & 3) * 32, 16, 1024);
          const uint64_t db = sdesc(kaddr + (ks >> 2) * L::KV_ATOM + (ks & 3) * 32, 16, 1024);
          mma_f16(d, da, db, L::IDESC_S, ks > 0 ? 1u : 0u);
        }
        mma_commit(s_full(j & 1));
        mma_commit(k_empty(st));
        mma_used_sh = 1;
        return true;
      };
      if (ok && T > 0) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % STAGES;
        if (!mbar_wait(p_full(j & 1), (j >> 1) & 1, status)) { ok = false; break; }
        fence_after();
        // S buffer j&1 is free again (its warpgroup has read S_j): queue S_{j+2}
        if (j + 2 < T && !issue_s(j + 2)) { ok = false; break; }
        if (!mbar_wait(v_full(st), (j / STAGES) & 1, status)) { ok = false; break; }
        vc = j + 1;
        fence_after();
        const uint32_t vaddr = sV + st * L::KV_TILE;
        const uint32_t paddr = sP + (j & 1) * L::P_BYTES;
        const uint32_t od = tmem + O_COL + 128u * (uint32_t)(j & 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = sdesc(paddr + kk * 32, 16, 1024);
          const uint64_t db = sdesc(vaddr + kk * 2048, L::KV_ATOM, 1024);
          mma_f16(od, da, db, L::IDESC_O, (j >= 2 || kk > 0) ? 1u : 0u);
        }
        mma_commit(o_done(j & 1));
        mma_commit(v_empty(st));
      }
      if (ok && T > 0) {
        // the last commit must land before this CTA's shared memory is released
        const int jl = T - 1;
        ok = mbar_wait(v_empty(jl % STAGES), (jl / STAGES) & 1, status);
      }
      if (!ok) atomicExch(&abort_sh, 1);
      consumed_sh[0] = kc;
      consumed_sh[1] = vc;
    }
  } else {
    // ------------------------------------------------ softmax warpgroups
    const int g = warp >> 2;                 // warpgroup: tiles j with j % 2 == g
    const int r = tid & 127;                 // query row 0..127 of the pair
    const int half = r >> 6;
    const bool row_valid = half == 0 || half1_valid;   // uniform per warp
    const uint32_t* mymask = selm[half];
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t ocol = O_COL + 128u * (uint32_t)g;
    const float sl2 = (1.0f / sqrtf((float)D)) * 1.4426950408889634f;
    float m_ref = -INFINITY, l = 0.f;
    int b = next_block(unionm, 0, nwords);
    bool ok = true;
    int last_j = -1;
    for (int j = 0; j < T; ++j) {
      if ((j & 1) != g) {                    // the other warpgroup's tile: only advance the block cursor
        if (j < U) b = next_block(unionm, b + 1, nwords);
        continue;
      }
      last_j = j;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full(g), (j >> 1) & 1, status))) { ok = false; break; }
      fence_after();
      uint32_t sa[32], sb[32];
      tmem_ld32(tmem + lane_base + (uint32_t)(g * 64), sa);
      tmem_ld32(tmem + lane_base + (uint32_t)(g * 64 + 32), sb);
      tmem_ld_wait();
      float x[64];
      bool any = true;
      if (j < U) {
        const bool take = row_valid && ((mymask[b >> 5] >> (b & 31)) & 1u);   // uniform per warp
        any = take;
        b = next_block(unionm, b + 1, nwords);
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(c < 32 ? sa[c] : sb[c - 32]) * sl2;
        if (!take) {
#pragma unroll
          for (int c = 0; c < 64; ++c) x[c] = -INFINITY;
        }
      } else {
        const int c0 = (j - U) * BLK;
        uint64_t excl;
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
            const float v = fmaf(__uint_as_float(c < 32 ? sa[c] : sb[c - 32]), sl2, bv[e] * 1.4426950408889634f);
            x[c] = ((excl >> c) & 1ull) ? -INFINITY : v;
          }
        }
      }
      // row max as a tree (independent chains)
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = x[i];
#pragma unroll
      for (int c = 8; c < 64; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], x[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      // new reference max: only moves up when the row max exceeds it by 2^8
      float m_new = m_ref, corr = 1.f;
      bool resc = false;
      if (mx > -INFINITY) {
        if (m_ref == -INFINITY) {
          m_new = mx;
        } else if (mx > m_ref + LAZY_RESCALE) {
          m_new = mx;
          corr = exp2f(m_ref - mx);
          resc = true;
        }
      }
      uint32_t pw[32];
      float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (any && m_new != -INFINITY) {
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float p0 = exp2f(x[c] - m_new);
          const float p1 = exp2f(x[c + 1] - m_new);
          rs8[(c >> 1) & 7] += p0 + p1;
          pw[c >> 1] = pack_bf2(p0, p1);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pw[c] = 0u;
      }
      const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      l = l * corr + rs;
      m_ref = m_new;
      // this warpgroup's previous P V product must be complete before its O
      // is rescaled or its P buffer is rewritten
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(o_done(g), ((j >> 1) - 1) & 1, status))) { ok = false; break; }
      fence_after();
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + ocol + 32 * cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
          tmem_st32(tmem + lane_base + ocol + 32 * cc, o);
        }
        tmem_st_wait();
      }
      // P row r of the 128B-swizzled [128 x 64] bf16 tile
      const uint32_t prow = sP + g * L::P_BYTES + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const uint32_t addr = prow + (uint32_t)(((c8 ^ (r & 7)) & 7) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pw[4 * c8]), "r"(pw[4 * c8 + 1]),
                     "r"(pw[4 * c8 + 2]), "r"(pw[4 * c8 + 3])
                     : "memory");
      }
      fence_proxy_async();
      fence_before();
      mbar_arrive(p_full(g));
    }
    // ---- epilogue: wait for this warpgroup's last P V, merge the two partial
    // softmaxes (log-sum-exp), O / l -> out[perm[row]]
    if (ok && last_j >= 0) ok = mbar_wait(o_done(g), (last_j >> 1) & 1, status);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) atomicExch(&abort_sh, 1);
    fence_after();
    if (g == 1) {
      m1_sh[r] = m_ref;
      l1_sh[r] = l;
    }
    fence_before();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    fence_after();
    ok = !(*(volatile int*)&abort_sh);
    if (g == 0 && ok && row_valid) {
      const float m1 = m1_sh[r], l1 = l1_sh[r];
      const float M = fmaxf(m_ref, m1);
      const float w0 = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - M);
      const float w1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M);
      const float lt = w0 * l + w1 * l1;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float c0 = w0 * inv, c1 = w1 * inv;
      const int pos = a0 * BLK + r;
      const int orig = perm[(size_t)bh * N + pos];
      const bool dst_ok = (unsigned)orig < (unsigned)N;
      if (!dst_ok) set_status(status, STATUS_BAD_INPUT);
      uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)bh * N + (dst_ok ? orig : 0)) * D);
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o0[32], o1[32];
        tmem_ld32(tmem + lane_base + O_COL + 32 * cc, o0);
        tmem_ld32(tmem + lane_base + O_COL + 128 + 32 * cc, o1);
        tmem_ld_wait();
        if (dst_ok) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const int e = 8 * q4 + 2 * h;
              const float v0 = __uint_as_float(o0[e]) * c0 + __uint_as_float(o1[e]) * c1;
              const float v1 = __uint_as_float(o0[e + 1]) * c0 + __uint_as_float(o1[e + 1]) * c1;
              w[h] = pack_bf2(v0, v1);
            }
            dst[cc * 4 + q4] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (lse != nullptr && dst_ok) lse[(size_t)bh * N + orig] = (M + log2f(lt)) * 0.6931471805599453f;
    }
  }

  // ---- teardown: drain own copies / MMAs (bounded), free TMEM
  fence_before();
  __syncthreads();
  fence_after();
  if (abort_sh) {
    if (warp == 8 && lane < 2) {
      // copies issued but never observed by the MMA thread
      if (lane == 0 && !q_seen_sh) mbar_wait(q_full, 0, status);
      for (int j = consumed_sh[lane]; j < issued_sh[lane]; ++j)
        mbar_wait(lane == 0 ? k_full(j % STAGES) : v_full(j % STAGES), (j / STAGES) & 1, status);
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
