// Host-side workspace plan and the launchers each kernel file exports.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <vector>

#include "../../include/spark.h"

namespace spark {

// Token chunks of the moments kernels: 32 blocks of 64 tokens each (fewer,
// larger chunks past MOMENT_SPLITS_MAX); the count depends on N only, and the
// float64 partial sums of a head are added in a fixed order.
constexpr int MOMENT_BLOCKS_PER_SPLIT = 32;
constexpr int MOMENT_SPLITS_MAX = 256;

struct Plan {
  int B = 0, H = 0, N = 0, d = 0, BH = 0, nb = 0, ksel = 0, nb_pad = 0;
  int tail = 0;                   // SPARK_TAIL_*
  int layout = 0;                 // SPARK_LAYOUT_*
  int nperm = 1;                  // permutations per pass (2 for SPARK_LAYOUT_SEPARATE)
  int power_iters = 16;           // power iterations per split
  int nlevels = 0;
  std::vector<int> level_count;   // nodes that split at each level
  std::vector<int> level_off;     // offset of each level in the node table
  std::vector<int> level_maxg;    // largest group (in blocks) at each level
  int moment_splits = 1;
  int sub_level = 0;              // first level whose nodes are split by the in-shared-memory subtree kernel
  std::vector<int> level_chunks;  // chunk CTAs per group at each level above the subtree level
  std::vector<int> level_derive;  // 1: right children's Gram sums derived from the parent level's
  std::vector<int> level_store;   // 1: the level's Gram sums are kept for the next level
  // byte offsets into the workspace
  size_t off_MQ = 0, off_MK = 0, off_qmean = 0;
  size_t off_mpart = 0;
  size_t off_L = 0, off_uhat = 0, off_idx = 0, off_pval = 0, off_pidx = 0;
  size_t off_nodes = 0;
  size_t off_bigpart = 0, off_biginfo = 0, off_bigcand = 0;
  size_t off_gstore[2] = {0, 0};   // Gram sums of consecutive levels (float64 [D*D + D] per group)
  size_t off_perm = 0, off_sel = 0;
  size_t off_Qp = 0, off_Kp = 0, off_Vp = 0;
  size_t off_qm = 0, off_km = 0;
  size_t off_kt = 0, off_vt = 0, off_beta = 0;
  size_t off_pairs = 0;            // query-block pairs of the attention units (int2 [BH][ceil(nb/2)])
  size_t off_scores = 0;           // block-score matrices of score_heads heads (float64 [nb][nb] each)
  size_t off_tail = 0;             // block-tail compressed logits (float32 [BH][nb][nb_pad], log2 units)
  int score_heads = 1;
  size_t total = 0;
  // extra device room used by spark_forward_host
  size_t off_hq = 0, off_hk = 0, off_hv = 0, off_hout = 0, off_hlse = 0;
  size_t host_slice = 0;   // spark_forward_host: workspace bytes of one compute lane
  size_t host_total = 0;
};

// Fills plan from validated params. Returns false if the params are invalid.
bool make_plan(const spark_params* p, Plan* plan);

template <class T>
inline T* ws_at(void* ws, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<char*>(ws) + off);
}

// ---- launchers (each returns cudaGetLastError() of its launches)
// gram_q / gram_k: form M_Q / M_K (the anchor qbar is always formed).
cudaError_t launch_moments(const Plan& pl, const uint16_t* q, const uint16_t* k, double* MQ,
                           double* MK, double* qmean, void* ws, bool gram_q, bool gram_k, cudaStream_t s);
cudaError_t launch_reblock(const Plan& pl, const uint16_t* x, const double* M, int32_t* perm,
                           void* ws, int* status, cudaStream_t s);
cudaError_t launch_positional(const Plan& pl, int F, int Hl, int Wl, int32_t* perm,
                              cudaStream_t s);
cudaError_t launch_select(const Plan& pl, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          const int32_t* perm, const double* qmean, int32_t* sel, int summary,
                          void* ws, int* status, cudaStream_t s);
// Diagnostic: a bounded wait that expires (see spark_selftest_wait).
cudaError_t launch_selftest_wait(unsigned long long limit_ns, int* status, cudaStream_t s);
// Context segment of joint attention: qc, kc, vc [BH, C, d] bf16 (C >= 1);
// outc [BH, C, d] bf16, lsec [BH, C] float32 or null.
struct JointContext {
  const void* qc;
  const void* kc;
  const void* vc;
  int C;
  uint16_t* outc;
  float* lsec;
};
cudaError_t launch_attn_tc(const Plan& pl, const int32_t* perm, const int32_t* sel, uint16_t* out,
                           float* lse, void* ws, int* status, cudaStream_t s,
                           const JointContext* ctx = nullptr);

}  // namespace spark
