// C ABI of libspark: argument validation, workspace planning and the launch
// sequence of each step. See include/spark.h for the contract of each call.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "plan.h"

namespace spark {

// Device status word: bounded waits and the Cholesky pivot check set bits
// here; spark_get_status() reads and clears it.
__device__ int g_spark_status = 0;

static int* status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_spark_status) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

static int num_selected_impl(int nb, double ratio, int blocks) {
  if (blocks > 0) return std::min(blocks, nb);
  const int k = (int)ceil(ratio * (double)nb - 1e-9);
  return std::max(1, std::min(nb, k));
}

static spark_status validate(const spark_params* p) {
  if (p == nullptr) return SPARK_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->N < 1 || p->d < 1) return SPARK_ERR_INVALID_ARG;
  if (p->topk_blocks < 0) return SPARK_ERR_INVALID_ARG;
  if (p->layout != SPARK_LAYOUT_Q_REUSE_K && p->layout != SPARK_LAYOUT_K_REUSE_Q &&
      p->layout != SPARK_LAYOUT_SEPARATE)
    return SPARK_ERR_INVALID_ARG;
  if (p->summary != SPARK_SUMMARY_REWEIGHT && p->summary != SPARK_SUMMARY_MEANPOOL) return SPARK_ERR_INVALID_ARG;
  if (p->tail != SPARK_TAIL_QUERY && p->tail != SPARK_TAIL_BLOCK) return SPARK_ERR_INVALID_ARG;
  if (p->power_iters < 0 || p->power_iters > 64) return SPARK_ERR_INVALID_ARG;
  if (p->N % SPARK_BLOCK != 0) return SPARK_ERR_UNSUPPORTED;
  if (p->d != 64 && p->d != 128) return SPARK_ERR_UNSUPPORTED;
  const long nb = p->N / SPARK_BLOCK;
  if (nb < 2 || nb > SPARK_MAX_BLOCKS) return SPARK_ERR_UNSUPPORTED;
  if (p->topk_blocks == 0 && !(p->topk_ratio > 0.0 && p->topk_ratio <= 1.0)) return SPARK_ERR_UNSUPPORTED;
  if ((long)p->B * p->H > 65535) return SPARK_ERR_UNSUPPORTED;
  return SPARK_OK;
}

static size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

// spark_forward_host runs the flattened B*H heads as HOST_CHUNKS chunks of
// consecutive heads (fewer when there are fewer heads), each a problem of its
// own (B = 1, H = its heads), computed on HOST_LANES lanes: chunk c on lane
// c % lanes, in that lane's slice of the workspace.
constexpr int HOST_CHUNKS = 8;
constexpr int HOST_LANES = 2;
static int host_chunks(int BH) { return std::min(BH, HOST_CHUNKS); }
static int host_lanes(int BH) { return std::min(host_chunks(BH), HOST_LANES); }
static int host_head0(int BH, int c) { return (int)(((long)BH * c) / host_chunks(BH)); }
static spark_params host_chunk_params(const spark_params* p, int BH, int c) {
  spark_params pc = *p;
  pc.B = 1;
  pc.H = host_head0(BH, c + 1) - host_head0(BH, c);
  return pc;
}

static bool make_plan_impl(const spark_params* p, Plan* pl, bool host);

bool make_plan(const spark_params* p, Plan* pl) { return make_plan_impl(p, pl, true); }

static bool make_plan_impl(const spark_params* p, Plan* pl, bool host) {
  if (validate(p) != SPARK_OK) return false;
  Plan& P = *pl;
  P = Plan();
  P.B = p->B; P.H = p->H; P.N = p->N; P.d = p->d;
  P.BH = p->B * p->H;
  P.tail = p->tail;
  P.layout = p->layout;
  P.power_iters = p->power_iters > 0 ? p->power_iters : 16;
  P.nperm = p->layout == SPARK_LAYOUT_SEPARATE ? 2 : 1;
  P.nb = p->N / SPARK_BLOCK;
  P.ksel = num_selected_impl(P.nb, p->topk_ratio, p->topk_blocks);
  P.nb_pad = (P.nb + 2 * SPARK_BLOCK - 1) / (2 * SPARK_BLOCK) * (2 * SPARK_BLOCK);   // summary tiles of 128
  // tree: same recursion as the device tree builder
  {
    std::vector<std::pair<int, int>> cur{{0, P.nb}};
    int off = 0;
    while (!cur.empty()) {
      int maxg = 0;
      for (auto& n : cur) maxg = std::max(maxg, n.second);
      P.level_count.push_back((int)cur.size());
      P.level_off.push_back(off);
      P.level_maxg.push_back(maxg);
      off += (int)cur.size();
      std::vector<std::pair<int, int>> nxt;
      for (auto& n : cur) {
        const int gl = n.second / 2, gr = n.second - gl;
        if (gl >= 2) nxt.push_back({n.first, gl});
        if (gr >= 2) nxt.push_back({n.first + gl, gr});
      }
      cur.swap(nxt);
    }
    P.nlevels = (int)P.level_count.size();
    P.sub_level = P.nlevels;
    for (int lv = 0; lv < P.nlevels; ++lv)
      if (P.level_maxg[lv] <= 9) { P.sub_level = lv; break; }
    // every level above the subtree level: groups spread over one CTA per
    // 32-tile chunk; when a level's groups are exactly the children of the
    // previous level's (two per parent), only left children's Gram sums are
    // computed and right children's are derived from their parents'
    P.level_chunks.assign(P.nlevels, 0);
    P.level_derive.assign(P.nlevels, 0);
    P.level_store.assign(P.nlevels, 0);
    for (int lv = 0; lv < P.sub_level; ++lv) {
      P.level_chunks[lv] = std::max(1, (P.level_maxg[lv] + 31) / 32);
      if (lv > 0 && P.level_count[lv] == 2 * P.level_count[lv - 1]) {
        P.level_derive[lv] = 1;
        P.level_store[lv - 1] = 1;
      }
    }
  }
  P.moment_splits = std::min(MOMENT_SPLITS_MAX, (P.nb + MOMENT_BLOCKS_PER_SPLIT - 1) / MOMENT_BLOCKS_PER_SPLIT);
  const size_t BH = P.BH, N = P.N, d = P.d, nb = P.nb, nbp = P.nb_pad;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = align_up(o + bytes); return at; };
  P.off_MQ = take(BH * d * d * 8);
  P.off_MK = take(BH * d * d * 8);
  P.off_qmean = take(BH * d * 8);
  P.off_mpart = take(BH * 2 * (size_t)P.moment_splits * (d * d + d) * 8);
  P.off_L = take(BH * d * d * 8);
  P.off_uhat = take(BH * N * d * 2);
  P.off_idx = take(BH * N * 4);
  P.off_pval = take(BH * N * 8);
  P.off_pidx = take(BH * N * 4);
  P.off_nodes = take(nb * 8);
  {
    size_t part = 0, info = 0, cand = 0;
    for (int lv = 0; lv < P.nlevels; ++lv) {
      if (P.level_chunks[lv] == 0) continue;
      const size_t groups = (size_t)P.BH * P.level_count[lv];
      part = std::max(part, groups * P.level_chunks[lv] * (d * d + d) * 8);
      info = std::max(info, groups * (d + 1) * 8);
      cand = std::max(cand, groups * P.level_chunks[lv] * 3 * 8);
    }
    P.off_bigpart = take(std::max<size_t>(part, 8));
    P.off_biginfo = take(std::max<size_t>(info, 8));
    P.off_bigcand = take(std::max<size_t>(cand, 8));
    size_t gs = 8;
    for (int lv = 0; lv < P.nlevels; ++lv)
      if (P.level_store[lv]) gs = std::max(gs, (size_t)P.BH * P.level_count[lv] * (d * d + d) * 8);
    P.off_gstore[0] = take(gs);
    P.off_gstore[1] = take(gs);
  }
  P.off_perm = take((size_t)P.nperm * BH * N * 4);
  P.off_sel = take(BH * nb * (size_t)P.ksel * 4);
  P.off_Qp = take(BH * N * d * 2);
  P.off_Kp = take(BH * N * d * 2);
  P.off_Vp = take(BH * N * d * 2);
  P.off_qm = take(BH * nb * d * 8);
  P.off_km = take(BH * nb * d * 8);
  P.off_kt = take(BH * nbp * d * 2);
  P.off_vt = take(BH * nbp * d * 2);
  P.off_beta = take(BH * nbp * 4);
  P.off_tail = P.tail == SPARK_TAIL_BLOCK ? take(BH * nb * nbp * 4) : 0;
  P.off_pairs = take(BH * ((nb + 1) / 2) * 8);
  {
    // float64 block-score matrices, a chunk of heads at a time (at most
    // 1 GiB, at least one head)
    const size_t per_head = nb * nb * 8;
    P.score_heads = (int)std::min<size_t>(BH, std::max<size_t>(1, ((size_t)1 << 30) / per_head));
    P.off_scores = take((size_t)P.score_heads * per_head);
  }
  P.total = o;
  if (!host) return true;
  // host-buffer pass: one workspace slice per lane, large enough for the
  // largest chunk's plan, then device copies of q, k, v, out and lse
  P.host_slice = 0;
  for (int c = 0; c < host_chunks(P.BH); ++c) {
    const spark_params pc = host_chunk_params(p, P.BH, c);
    Plan plc;
    if (!make_plan_impl(&pc, &plc, false)) return false;
    P.host_slice = std::max(P.host_slice, align_up(plc.total));
  }
  o = (size_t)host_lanes(P.BH) * P.host_slice;
  P.off_hq = take(BH * N * d * 2);
  P.off_hk = take(BH * N * d * 2);
  P.off_hv = take(BH * N * d * 2);
  P.off_hout = take(BH * N * d * 2);
  P.off_hlse = take(BH * N * 4);
  P.host_total = o;
  return true;
}

static bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }

static spark_status check_ws(const Plan& pl, const void* ws, size_t ws_bytes) {
  if (ws == nullptr || !aligned16(ws)) return SPARK_ERR_INVALID_ARG;
  if (ws_bytes < pl.total) return SPARK_ERR_WORKSPACE;
  return SPARK_OK;
}

static spark_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA; }

// The moments a layout partitions under: queries are whitened with M_K, keys
// with M_Q. The whole pass forms only those (plus the anchor).
static bool needs_mk(const Plan& pl) { return pl.layout != SPARK_LAYOUT_K_REUSE_Q; }
static bool needs_mq(const Plan& pl) { return pl.layout != SPARK_LAYOUT_Q_REUSE_K; }

}  // namespace spark

using namespace spark;

extern "C" {

spark_status spark_validate(const spark_params* p) { return validate(p); }

int32_t spark_num_selected(const spark_params* p) {
  if (validate(p) != SPARK_OK) return -1;
  return num_selected_impl(p->N / SPARK_BLOCK, p->topk_ratio, p->topk_blocks);
}

size_t spark_workspace_size(const spark_params* p) {
  Plan pl;
  return make_plan(p, &pl) ? pl.total : 0;
}

int32_t spark_forward_launches(const spark_params* p) {
  Plan pl;
  if (!make_plan(p, &pl)) return -1;
  // moments: one Gram per moment the layout uses, the anchor's column sums
  // when the query moment is not formed, the reduce; reblock: whiten,
  // normalise, tree, init, per split level Gram (+ reduce of chunk partials),
  // solve, project, select, then subtree and leaves; select: block
  // statistics, then scores + top-K per chunk of heads; attention 2 (pairs, kernel)
  const int moments = (pl.layout == SPARK_LAYOUT_K_REUSE_Q) ? 2 : 3;
  int split_launches = 0;
  for (int lv = 0; lv < pl.sub_level; ++lv) split_launches += 4 + (pl.level_chunks[lv] > 1 ? 1 : 0);
  const int reblock = pl.nperm * (4 + split_launches + (pl.sub_level < pl.nlevels ? 1 : 0) + 1);
  const int select = 1 + 2 * ((pl.BH + pl.score_heads - 1) / pl.score_heads) + (pl.tail == SPARK_TAIL_BLOCK ? 1 : 0);
  return moments + reblock + select + 2;
}

size_t spark_host_workspace_size(const spark_params* p) {
  Plan pl;
  return make_plan(p, &pl) ? pl.host_total : 0;
}

spark_status spark_moments(const spark_params* p, const void* q, const void* k, double* MQ,
                           double* MK, double* qmean, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const spark_status v = validate(p);
  if (v != SPARK_OK) return v;
  Plan pl;
  make_plan(p, &pl);
  if (!q || !k || !qmean || !aligned16(q) || !aligned16(k)) return SPARK_ERR_INVALID_ARG;
  const spark_status w = check_ws(pl, ws, ws_bytes);
  if (w != SPARK_OK) return w;
  return cuda_status(launch_moments(pl, (const uint16_t*)q, (const uint16_t*)k, MQ, MK, qmean, ws, MQ != nullptr,
                                    MK != nullptr, stream));
}

// The partition(s) of the layout: queries under M_K, keys under M_Q, or both
// (SPARK_LAYOUT_SEPARATE: query permutation first, key permutation after it).
static cudaError_t reblock_layout(const Plan& pl, const void* q, const void* k, const double* MQ,
                                  const double* MK, int32_t* perm, void* ws, cudaStream_t s) {
  if (pl.layout == SPARK_LAYOUT_K_REUSE_Q) return launch_reblock(pl, (const uint16_t*)k, MQ, perm, ws, status_ptr(), s);
  cudaError_t e = launch_reblock(pl, (const uint16_t*)q, MK, perm, ws, status_ptr(), s);
  if (e != cudaSuccess || pl.layout != SPARK_LAYOUT_SEPARATE) return e;
  return launch_reblock(pl, (const uint16_t*)k, MQ, perm + (size_t)pl.BH * pl.N, ws, status_ptr(), s);
}

spark_status spark_reblock(const spark_params* p, const void* q, const void* k, const double* MQ,
                           const double* MK, int32_t* perm, void* ws, size_t ws_bytes,
                           cudaStream_t stream) {
  const spark_status v = validate(p);
  if (v != SPARK_OK) return v;
  Plan pl;
  make_plan(p, &pl);
  if (!q || !k || !perm || !aligned16(q) || !aligned16(k)) return SPARK_ERR_INVALID_ARG;
  if ((needs_mq(pl) && !MQ) || (needs_mk(pl) && !MK)) return SPARK_ERR_INVALID_ARG;
  const spark_status w = check_ws(pl, ws, ws_bytes);
  if (w != SPARK_OK) return w;
  return cuda_status(reblock_layout(pl, q, k, MQ, MK, perm, ws, stream));
}

spark_status spark_positional_perm(const spark_params* p, int32_t F, int32_t Hl, int32_t Wl,
                                   int32_t* perm, cudaStream_t stream) {
  const spark_status v = validate(p);
  if (v != SPARK_OK) return v;
  if (!perm || F < 1 || Hl < 1 || Wl < 1) return SPARK_ERR_INVALID_ARG;
  if ((long)F * Hl * Wl != p->N) return SPARK_ERR_INVALID_ARG;
  if (F % 2 != 0 || Hl % 8 != 0 || Wl % 4 != 0) return SPARK_ERR_UNSUPPORTED;
  Plan pl;
  make_plan(p, &pl);
  cudaError_t e = launch_positional(pl, F, Hl, Wl, perm, stream);
  // the separate layout takes the same fixed tiles for its key permutation
  if (e == cudaSuccess && pl.nperm == 2) e = launch_positional(pl, F, Hl, Wl, perm + (size_t)pl.BH * pl.N, stream);
  return cuda_status(e);
}

spark_status spark_select(const spark_params* p, const void* q, const void* k, const void* v,
                          const int32_t* perm, const double* qmean, int32_t* sel, void* ws,
                          size_t ws_bytes, cudaStream_t stream) {
  const spark_status vs = validate(p);
  if (vs != SPARK_OK) return vs;
  Plan pl;
  make_plan(p, &pl);
  if (!q || !k || !v || !perm || !qmean || !sel) return SPARK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return SPARK_ERR_INVALID_ARG;
  const spark_status w = check_ws(pl, ws, ws_bytes);
  if (w != SPARK_OK) return w;
  return cuda_status(launch_select(pl, (const uint16_t*)q, (const uint16_t*)k, (const uint16_t*)v,
                                   perm, qmean, sel, p->summary, ws, status_ptr(), stream));
}

spark_status spark_attn_fwd(const spark_params* p, const int32_t* perm, const int32_t* sel, void* out,
                            float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const spark_status v = validate(p);
  if (v != SPARK_OK) return v;
  Plan pl;
  make_plan(p, &pl);
  if (!perm || !sel || !out || !aligned16(out)) return SPARK_ERR_INVALID_ARG;
  const spark_status w = check_ws(pl, ws, ws_bytes);
  if (w != SPARK_OK) return w;
  return cuda_status(launch_attn_tc(pl, perm, sel, (uint16_t*)out, lse, ws, status_ptr(), stream));
}

static spark_status check_context(const spark_params* p, const void* qc, const void* kc, const void* vc,
                                  int32_t C, const void* outc) {
  if (C < 1 || !qc || !kc || !vc || !outc) return SPARK_ERR_INVALID_ARG;
  if (!aligned16(qc) || !aligned16(kc) || !aligned16(vc) || !aligned16(outc)) return SPARK_ERR_INVALID_ARG;
  if ((long)p->B * p->H * C > (long)INT32_MAX / 2) return SPARK_ERR_UNSUPPORTED;
  return SPARK_OK;
}

spark_status spark_attn_fwd_joint(const spark_params* p, const int32_t* perm, const int32_t* sel,
                                  const void* qc, const void* kc, const void* vc, int32_t C, void* out,
                                  float* lse, void* outc, float* lsec, void* ws, size_t ws_bytes,
                                  cudaStream_t stream) {
  const spark_status v = validate(p);
  if (v != SPARK_OK) return v;
  Plan pl;
  make_plan(p, &pl);
  if (!perm || !sel || !out || !aligned16(out)) return SPARK_ERR_INVALID_ARG;
  const spark_status c = check_context(p, qc, kc, vc, C, outc);
  if (c != SPARK_OK) return c;
  const spark_status w = check_ws(pl, ws, ws_bytes);
  if (w != SPARK_OK) return w;
  const JointContext ctx{qc, kc, vc, C, (uint16_t*)outc, lsec};
  return cuda_status(launch_attn_tc(pl, perm, sel, (uint16_t*)out, lse, ws, status_ptr(), stream, &ctx));
}

spark_status spark_forward_joint(const spark_params* p, const void* q, const void* k, const void* v,
                                 const void* qc, const void* kc, const void* vc, int32_t C, void* out,
                                 float* lse, void* outc, float* lsec, void* ws, size_t ws_bytes,
                                 cudaStream_t stream) {
  const spark_status vs = validate(p);
  if (vs != SPARK_OK) return vs;
  Plan pl;
  make_plan(p, &pl);
  if (!q || !k || !v || !out) return SPARK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SPARK_ERR_INVALID_ARG;
  const spark_status c = check_context(p, qc, kc, vc, C, outc);
  if (c != SPARK_OK) return c;
  const spark_status w = check_ws(pl, ws, ws_bytes);
  if (w != SPARK_OK) return w;
  double* MQ = ws_at<double>(ws, pl.off_MQ);
  double* MK = ws_at<double>(ws, pl.off_MK);
  double* qmean = ws_at<double>(ws, pl.off_qmean);
  int32_t* perm = ws_at<int32_t>(ws, pl.off_perm);
  int32_t* sel = ws_at<int32_t>(ws, pl.off_sel);
  cudaError_t e = launch_moments(pl, (const uint16_t*)q, (const uint16_t*)k, MQ, MK, qmean, ws, needs_mq(pl),
                                 needs_mk(pl), stream);
  if (e != cudaSuccess) return SPARK_ERR_CUDA;
  e = reblock_layout(pl, q, k, MQ, MK, perm, ws, stream);
  if (e != cudaSuccess) return SPARK_ERR_CUDA;
  e = launch_select(pl, (const uint16_t*)q, (const uint16_t*)k, (const uint16_t*)v, perm, qmean, sel,
                    p->summary, ws, status_ptr(), stream);
  if (e != cudaSuccess) return SPARK_ERR_CUDA;
  const JointContext ctx{qc, kc, vc, C, (uint16_t*)outc, lsec};
  return cuda_status(launch_attn_tc(pl, perm, sel, (uint16_t*)out, lse, ws, status_ptr(), stream, &ctx));
}

spark_status spark_forward(const spark_params* p, const void* q, const void* k, const void* v,
                           void* out, float* lse, int32_t* perm_out, int32_t* sel_out, void* ws,
                           size_t ws_bytes, cudaStream_t stream) {
  const spark_status vs = validate(p);
  if (vs != SPARK_OK) return vs;
  Plan pl;
  make_plan(p, &pl);
  if (!q || !k || !v || !out) return SPARK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SPARK_ERR_INVALID_ARG;
  const spark_status w = check_ws(pl, ws, ws_bytes);
  if (w != SPARK_OK) return w;
  double* MQ = ws_at<double>(ws, pl.off_MQ);
  double* MK = ws_at<double>(ws, pl.off_MK);
  double* qmean = ws_at<double>(ws, pl.off_qmean);
  int32_t* perm = perm_out ? perm_out : ws_at<int32_t>(ws, pl.off_perm);
  int32_t* sel = sel_out ? sel_out : ws_at<int32_t>(ws, pl.off_sel);
  cudaError_t e = launch_moments(pl, (const uint16_t*)q, (const uint16_t*)k, MQ, MK, qmean, ws, needs_mq(pl),
                                 needs_mk(pl), stream);
  if (e != cudaSuccess) return SPARK_ERR_CUDA;
  e = reblock_layout(pl, q, k, MQ, MK, perm, ws, stream);
  if (e != cudaSuccess) return SPARK_ERR_CUDA;
  e = launch_select(pl, (const uint16_t*)q, (const uint16_t*)k, (const uint16_t*)v, perm, qmean, sel,
                    p->summary, ws, status_ptr(), stream);
  if (e != cudaSuccess) return SPARK_ERR_CUDA;
  e = launch_attn_tc(pl, perm, sel, (uint16_t*)out, lse, ws, status_ptr(), stream);
  return cuda_status(e);
}

// Copy streams and events of the host-buffer entry point, one set per device,
// created on first use and kept for the life of the process.
namespace {
constexpr int HOST_MAX_DEVICES = 64;
struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr, lane[HOST_LANES] = {};
  cudaEvent_t entry = nullptr, done = nullptr, in[HOST_CHUNKS] = {}, comp[HOST_CHUNKS] = {};
  bool ready = false;
};
std::mutex g_host_mu;                       // one call enqueues at a time: the events are shared
HostPipe g_host_pipe[HOST_MAX_DEVICES];

HostPipe* host_pipe() {                     // call with g_host_mu held
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= HOST_MAX_DEVICES) return nullptr;
  HostPipe& hp = g_host_pipe[dev];
  if (!hp.ready) {
    bool ok = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.entry, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming) == cudaSuccess;
    for (int c = 0; ok && c < HOST_CHUNKS; ++c)
      ok = cudaEventCreateWithFlags(&hp.in[c], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.comp[c], cudaEventDisableTiming) == cudaSuccess;
    for (int l = 0; ok && l < HOST_LANES; ++l)
      ok = cudaStreamCreateWithFlags(&hp.lane[l], cudaStreamNonBlocking) == cudaSuccess;
    if (!ok) return nullptr;
    hp.ready = true;
  }
  return &hp;
}
}  // namespace

// Heads are independent, so the pass runs as up to HOST_CHUNKS chunks of
// consecutive heads: the chunks are copied in one after another (one copy
// stream), each is computed as soon as it has arrived on one of HOST_LANES
// compute streams (chunk c on lane c % lanes, in the lane's workspace slice,
// so two chunks' kernels can share the GPU: one chunk's latency-bound
// partition fills the SMs another chunk's attention leaves idle), and copied
// out when done (a second copy stream). Everything starts after the work
// already queued on the caller's stream, which waits for the last copy out.
spark_status spark_forward_host(const spark_params* p, const void* q_host, const void* k_host,
                                const void* v_host, void* out_host, float* lse_host, void* ws,
                                size_t ws_bytes, cudaStream_t stream) {
  const spark_status vs = validate(p);
  if (vs != SPARK_OK) return vs;
  Plan pl;
  if (!make_plan(p, &pl)) return SPARK_ERR_INVALID_ARG;
  if (!q_host || !k_host || !v_host || !out_host) return SPARK_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned16(ws)) return SPARK_ERR_INVALID_ARG;
  if (ws_bytes < pl.host_total) return SPARK_ERR_WORKSPACE;
  char* dq = ws_at<char>(ws, pl.off_hq);
  char* dk = ws_at<char>(ws, pl.off_hk);
  char* dv = ws_at<char>(ws, pl.off_hv);
  char* dout = ws_at<char>(ws, pl.off_hout);
  float* dlse = lse_host ? ws_at<float>(ws, pl.off_hlse) : nullptr;
  const size_t head_bytes = (size_t)pl.N * pl.d * 2;   // one head of q, k, v or out
  const int nch = host_chunks(pl.BH), lanes = host_lanes(pl.BH);

  // every chunk must fit its lane's slice: check them all before anything is queued
  for (int c = 0; c < nch; ++c) {
    const spark_params pc = host_chunk_params(p, pl.BH, c);
    Plan plc;
    if (validate(&pc) != SPARK_OK || !make_plan(&pc, &plc)) return SPARK_ERR_INVALID_ARG;
    if (plc.total > pl.host_slice) return SPARK_ERR_WORKSPACE;
  }
  std::lock_guard<std::mutex> guard(g_host_mu);
  HostPipe* hp = host_pipe();
  if (hp == nullptr) return SPARK_ERR_CUDA;
  if (cudaEventRecord(hp->entry, stream) != cudaSuccess) return SPARK_ERR_CUDA;
  // once anything is queued, a failure still orders the caller's stream after
  // all of it (the workspace and the host buffers stay in use until then)
  auto fail = [&](spark_status st) {
    for (int l = 0; l < lanes; ++l)
      if (cudaEventRecord(hp->comp[l], hp->lane[l]) == cudaSuccess) cudaStreamWaitEvent(hp->d2h, hp->comp[l], 0);
    if (cudaEventRecord(hp->in[0], hp->h2d) == cudaSuccess) cudaStreamWaitEvent(hp->d2h, hp->in[0], 0);
    if (cudaEventRecord(hp->done, hp->d2h) == cudaSuccess) cudaStreamWaitEvent(stream, hp->done, 0);
    return st;
  };
  if (cudaStreamWaitEvent(hp->h2d, hp->entry, 0) != cudaSuccess) return fail(SPARK_ERR_CUDA);
  if (cudaStreamWaitEvent(hp->d2h, hp->entry, 0) != cudaSuccess) return fail(SPARK_ERR_CUDA);
  for (int l = 0; l < lanes; ++l)
    if (cudaStreamWaitEvent(hp->lane[l], hp->entry, 0) != cudaSuccess) return fail(SPARK_ERR_CUDA);
  for (int c = 0; c < nch; ++c) {
    const int h0 = host_head0(pl.BH, c), h1 = host_head0(pl.BH, c + 1);
    const size_t off = (size_t)h0 * head_bytes, len = (size_t)(h1 - h0) * head_bytes;
    if (cudaMemcpyAsync(dq + off, (const char*)q_host + off, len, cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess ||
        cudaMemcpyAsync(dk + off, (const char*)k_host + off, len, cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess ||
        cudaMemcpyAsync(dv + off, (const char*)v_host + off, len, cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess ||
        cudaEventRecord(hp->in[c], hp->h2d) != cudaSuccess)
      return fail(SPARK_ERR_CUDA);
  }
  for (int c = 0; c < nch; ++c) {
    const int h0 = host_head0(pl.BH, c), hc = host_head0(pl.BH, c + 1) - h0;
    const size_t off = (size_t)h0 * head_bytes, len = (size_t)hc * head_bytes;
    cudaStream_t ls = hp->lane[c % lanes];
    void* lws = ws_at<char>(ws, (size_t)(c % lanes) * pl.host_slice);
    const spark_params pc = host_chunk_params(p, pl.BH, c);
    if (cudaStreamWaitEvent(ls, hp->in[c], 0) != cudaSuccess) return fail(SPARK_ERR_CUDA);
    const spark_status r = spark_forward(&pc, dq + off, dk + off, dv + off, dout + off,
                                         dlse ? dlse + (size_t)h0 * pl.N : nullptr, nullptr, nullptr, lws,
                                         pl.host_slice, ls);
    if (r != SPARK_OK) return fail(r);
    if (cudaEventRecord(hp->comp[c], ls) != cudaSuccess) return fail(SPARK_ERR_CUDA);
    if (cudaStreamWaitEvent(hp->d2h, hp->comp[c], 0) != cudaSuccess) return fail(SPARK_ERR_CUDA);
    if (cudaMemcpyAsync((char*)out_host + off, dout + off, len, cudaMemcpyDeviceToHost, hp->d2h) != cudaSuccess)
      return fail(SPARK_ERR_CUDA);
    if (lse_host && cudaMemcpyAsync(lse_host + (size_t)h0 * pl.N, dlse + (size_t)h0 * pl.N, (size_t)hc * pl.N * 4,
                                    cudaMemcpyDeviceToHost, hp->d2h) != cudaSuccess)
      return fail(SPARK_ERR_CUDA);
  }
  // the copy-out stream has waited for every chunk's compute
  if (cudaEventRecord(hp->done, hp->d2h) != cudaSuccess) return fail(SPARK_ERR_CUDA);
  if (cudaStreamWaitEvent(stream, hp->done, 0) != cudaSuccess) return fail(SPARK_ERR_CUDA);
  return SPARK_OK;
}

size_t spark_workspace_region(const spark_params* p, int32_t region, size_t* bytes) {
  Plan pl;
  if (!make_plan(p, &pl)) return (size_t)-1;
  const size_t BH = pl.BH, N = pl.N, d = pl.d, nb = pl.nb, nbp = pl.nb_pad;
  size_t off, sz;
  switch (region) {
    case SPARK_WS_MQ: off = pl.off_MQ; sz = BH * d * d * 8; break;
    case SPARK_WS_MK: off = pl.off_MK; sz = BH * d * d * 8; break;
    case SPARK_WS_QMEAN: off = pl.off_qmean; sz = BH * d * 8; break;
    case SPARK_WS_PERM: off = pl.off_perm; sz = (size_t)pl.nperm * BH * N * 4; break;
    case SPARK_WS_SEL: off = pl.off_sel; sz = BH * nb * (size_t)pl.ksel * 4; break;
    case SPARK_WS_QM: off = pl.off_qm; sz = BH * nb * d * 8; break;
    case SPARK_WS_KM: off = pl.off_km; sz = BH * nb * d * 8; break;
    case SPARK_WS_KT: off = pl.off_kt; sz = BH * nbp * d * 2; break;
    case SPARK_WS_VT: off = pl.off_vt; sz = BH * nbp * d * 2; break;
    case SPARK_WS_BETA: off = pl.off_beta; sz = BH * nbp * 4; break;
    case SPARK_WS_UHAT: off = pl.off_uhat; sz = BH * N * d * 2; break;
    case SPARK_WS_PAIRS: off = pl.off_pairs; sz = BH * ((nb + 1) / 2) * 8; break;
    default: return (size_t)-1;
  }
  if (bytes) *bytes = sz;
  return off;
}

spark_status spark_selftest_wait(int64_t limit_ns, cudaStream_t stream) {
  if (limit_ns < 1 || limit_ns > 2000000000ll) return SPARK_ERR_INVALID_ARG;
  return cuda_status(launch_selftest_wait((unsigned long long)limit_ns, status_ptr(), stream));
}

spark_status spark_get_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SPARK_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_spark_status, sizeof(int)) != cudaSuccess) return SPARK_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_spark_status, &zero, sizeof(int)) != cudaSuccess) return SPARK_ERR_CUDA;
  if (h & STATUS_TIMEOUT) return SPARK_ERR_TIMEOUT;
  if (h & (STATUS_BAD_PIVOT | STATUS_BAD_INPUT)) return SPARK_ERR_UNSUPPORTED;
  return SPARK_OK;
}

const char* spark_strerror(spark_status s) {
  switch (s) {
    case SPARK_OK: return "ok";
    case SPARK_ERR_INVALID_ARG: return "invalid argument";
    case SPARK_ERR_UNSUPPORTED: return "unsupported input";
    case SPARK_ERR_WORKSPACE: return "workspace too small";
    case SPARK_ERR_CUDA: return "CUDA error";
    case SPARK_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

}  // extern "C"
