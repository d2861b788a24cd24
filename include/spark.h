/*
 * spark.h - C ABI of libspark, a B200 (sm_100a) implementation of the
 * Spark-Attn block-sparse attention forward pass.
 *
 * Sources (web pages describing the method):
 *   [P1] "Spark-H3: block-sparse attention speeds up MiniMax-H3 in ComfyUI"
 *        (comfyui-wiki news post, 2026-10-11), sections "What Spark-Attn
 *        changed" and "Workflows".
 *   [P2] "MiniMax H3 Spark Attention (SM89)" (comfy.icu node page), sections
 *        "What it's doing under the hood" and "Inputs you'll actually set".
 *
 * The forward pass, per (batch item b, head h), on N tokens of head dim d:
 *   1. moments  : M_Q = E[q q^T], M_K = E[k k^T], anchor qbar = E[q]     [P2 under the hood]
 *   2. reblock  : capacity-constrained recursive bisection of the queries
 *                 (q_reuse_k) under the M_K Mahalanobis cosine into
 *                 exactly-64-token blocks, emitted as a permutation      [P1, P2]
 *   3. select   : block means, block scores, top-K key blocks per query
 *                 block; reweighted key/value summaries with a log-mass
 *                 bias anchored on qbar                                 [P1, P2 Inputs]
 *   4. attn_fwd : exact branch over the selected blocks + compressed
 *                 branch over the summaries of all other blocks, merged
 *                 in one softmax (log-sum-exp merge), rows written back
 *                 in original token order                               [P1, P2]
 *
 * Conventions shared by every entry point
 *   - Tensors q, k, v, out are [B, H, N, d] bfloat16, contiguous, row-major,
 *     base address 16-byte aligned. perm is [B, H, N] int32 ([2, B, H, N]
 *     for SPARK_LAYOUT_SEPARATE: query permutation, then key permutation); sel is
 *     [B, H, nb, Ksel] int32 with nb = N / 64 and Ksel = spark_num_selected().
 *   - All pointers are DEVICE pointers unless the entry point says "host".
 *     The caller owns all memory; the library allocates and frees nothing.
 *   - Calls are asynchronous on the given stream; nothing synchronises except
 *     spark_get_status().
 *   - Arguments are validated on the host before anything is launched.
 *     Unsupported input is an error, never a silent fallback ([P2] Inputs:
 *     "strict" makes unsupported inputs error out): N % 64 != 0, nb < 2,
 *     d not in {64, 128}, a ratio outside (0, 1], nb > SPARK_MAX_BLOCKS or
 *     misaligned pointers give SPARK_ERR_UNSUPPORTED / SPARK_ERR_INVALID_ARG.
 *   - A failed launch gives SPARK_ERR_CUDA. A device-side bounded wait that
 *     expired sets a status word that spark_get_status() reports as
 *     SPARK_ERR_TIMEOUT.
 *   - Inputs must be finite; NaN or Inf inputs give unspecified results.
 */
#ifndef SPARK_H_
#define SPARK_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPARK_BLOCK 64          /* tokens per block ([P2]: exactly 64-token leaves) */
#define SPARK_MAX_BLOCKS 8192   /* largest nb accepted (N <= 524288) */

typedef enum {
  SPARK_OK = 0,
  SPARK_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad enum, bad size */
  SPARK_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels support */
  SPARK_ERR_WORKSPACE = 3,     /* ws_bytes smaller than required */
  SPARK_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  SPARK_ERR_TIMEOUT = 5        /* a device-side bounded wait expired */
} spark_status;

/* reblock_layout ([P1] Workflows: every shipped workflow pins q_reuse_k). */
enum {
  SPARK_LAYOUT_Q_REUSE_K = 0,  /* partition the queries under M_K; K and V reuse it */
  SPARK_LAYOUT_K_REUSE_Q = 1,  /* mirror: partition the keys under M_Q; Q reuses it */
  SPARK_LAYOUT_SEPARATE = 2    /* queries under M_K and keys (with their values) under M_Q,
                                  each on its own ([P2] under the hood: two-sided reblock);
                                  every perm below then holds 2*B*H*N entries: the query
                                  permutation [B,H,N] followed by the key permutation */
};

/* compressed-branch summaries ([P2]: Reweight replaces mean pooling). */
enum {
  SPARK_SUMMARY_REWEIGHT = 0,  /* anchor-weighted k~, v~ plus log-mass bias beta */
  SPARK_SUMMARY_MEANPOOL = 1   /* ablation: mean k, mean v, beta = ln 64 */
};

/* tail granularity of the compressed branch ([P2] Inputs: tail_granularity;
 * "What it's doing under the hood": a real Q per query, only K/V downsampled). */
enum {
  SPARK_TAIL_QUERY = 0,        /* each query scores the summaries with its own q */
  SPARK_TAIL_BLOCK = 1         /* every query of a block scores them with the block's mean
                                  query (the exact block means the selection uses); the
                                  exact branch keeps each query's own q */
};

typedef struct {
  int32_t B, H, N, d;          /* batch, heads, tokens (multiple of 64), head dim (64|128) */
  double topk_ratio;           /* used when topk_blocks == 0: Ksel = ceil(r * nb), r in (0,1] */
  int32_t topk_blocks;         /* > 0: fixed count of kept blocks (clamped to nb) */
  int32_t layout;              /* SPARK_LAYOUT_* */
  int32_t summary;             /* SPARK_SUMMARY_* */
  int32_t tail;                /* SPARK_TAIL_* */
  int32_t power_iters;         /* power iterations per split: 0 = 16 (default); the "Lite"
                                  reblock ("Spark-H3" news post: halved reblock latency, method
                                  not given) takes fewer, e.g. 4; 1..64 accepted */
} spark_params;

/* Checks a parameter block. SPARK_OK or the error the other calls would give. */
spark_status spark_validate(const spark_params* p);

/* Key blocks kept per query block: topk_blocks if > 0 (clamped to nb), else
 * clamp(ceil(topk_ratio * nb - 1e-9), 1, nb) ([P2] Inputs: topk_ratio /
 * topk_blocks). Returns -1 for an invalid parameter block. */
int32_t spark_num_selected(const spark_params* p);

/* Bytes of device workspace every call below needs (one size for all, so a
 * single buffer serves the whole pass). 0 for an invalid parameter block. */
size_t spark_workspace_size(const spark_params* p);

/* Step 1 - second moments ([P2] under the hood: M_K = E[k k^T] for queries,
 * M_Q for keys) and the per-head mean query ([P1] Spark-Reweight bullet: the
 * mean video query is the anchor of each head). Uncentered, over all N tokens.
 * Products of the bf16 inputs are exact in float64 and the sums are float64
 * (float64 tensor cores), so the moments equal (1/N) sum x x^T up to float64
 * summation order: the partition's whitening, and every bf16 rounding of the
 * whitened tokens, then agree with a float64 evaluation of the definition.
 *   q, k   : [B,H,N,d] bf16 device, read only
 *   MQ, MK : [B,H,d,d] float64 device, written (row-major, symmetric); either
 *            may be NULL to skip that moment (q_reuse_k needs only M_K,
 *            k_reuse_q only M_Q; spark_forward forms only what its layout needs)
 *   qmean  : [B,H,d] float64 device, written
 *   ws     : workspace of spark_workspace_size() bytes (scratch) */
spark_status spark_moments(const spark_params* p, const void* q, const void* k,
                           double* MQ, double* MK, double* qmean,
                           void* ws, size_t ws_bytes, cudaStream_t stream);

/* Allocation-free variant of spark_moments. The pages have no counterpart:
 * this is a convenience of this library for callers that cannot allocate or
 * lend device memory - for example code embedded in a host framework that
 * owns every device allocation and forbids new ones on its hot path, or a
 * caller with a fixed memory plan and no workspace to hand over. It runs the
 * kernels spark_moments runs (float64 Gram sums and anchor), but keeps the
 * partial sums in a fixed device array inside the library instead of a
 * workspace, and always forms both moments (MQ, MK and qmean must be non-NULL).
 *   - The array is SPARK_NOALLOC_SCRATCH_BYTES (16 MiB) per device; every GPU
 *     that loads the library holds it until the process exits.
 *   - Limit: 2 * B * H partial sums of (d*d + d) doubles must fit, i.e.
 *     B*H <= 63 for d = 128 and B*H <= 252 for d = 64; larger inputs return
 *     SPARK_ERR_UNSUPPORTED without launching anything. Within the limit the
 *     token range of a head may be cut into fewer chunks than spark_moments
 *     uses, so it can be slower, and its float64 sums, added in another order,
 *     can differ from spark_moments' in the last bits (a reblock run on them
 *     can then, rarely, differ where a whitened value sits on a bf16 midpoint).
 *   - Every call looks up the array's device address (cudaGetSymbolAddress)
 *     with the current device, so it stays right after a device reset. That
 *     lookup is a runtime call: make the first call on a device before any
 *     stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (nothing in it needs to start at zero: each call writes every
 *     partial before reading it). Calls whose kernels may overlap on the GPU
 *     (other streams, other host threads) race on it: serialise them.
 *   - Never allocates or frees memory (no cudaMalloc / cudaFree).
 * Arguments as for spark_moments, minus the workspace. */
#define SPARK_NOALLOC_SCRATCH_BYTES (16u << 20)
spark_status spark_moments_noalloc(const spark_params* p, const void* q, const void* k,
                                   double* MQ, double* MK, double* qmean, cudaStream_t stream);

/* Step 2 - reblock ([P1] Spark-Reblock bullet; [P2] under the hood):
 * recursive bisection of the partitioned side (queries for q_reuse_k, keys
 * for k_reuse_q, both in turn for separate) along the top principal direction of its whitened,
 * normalised vectors (Cholesky factor of the opposite side's moment),
 * split by rank into 64*floor(g/2) and the rest, down to 64-token leaves.
 * The whitened tokens u = L^T x, their norms and the quotients u / |u| are
 * float64 (float64 tensor cores) and each is rounded once to bf16, as a
 * float64 evaluation of the definition rounds them.
 *   q, k   : [B,H,N,d] bf16 device, read only
 *   MQ, MK : from spark_moments, read only; only the moment(s) the layout
 *            uses must be non-NULL (M_K for q_reuse_k, M_Q for k_reuse_q)
 *   perm   : [B,H,N] int32 device, written: perm[pi] = original index of the
 *            token at permuted position pi; leaves in depth-first order,
 *            ascending original index inside each block. Q/K/V are never
 *            modified ([P2]: only which tokens share a block changes). */
spark_status spark_reblock(const spark_params* p, const void* q, const void* k,
                           const double* MQ, const double* MK, int32_t* perm,
                           void* ws, size_t ws_bytes, cudaStream_t stream);

/* The fixed-tile layout Spark-Reblock replaces ([P1] Spark-Reblock bullet:
 * "fixed spatio-temporal tiles"): 2x8x4 (frame,row,column) tiles of the
 * F x Hl x Wl latent grid in raster order, ascending index inside a tile.
 * Requires F*Hl*Wl == N and F%2 == Hl%8 == Wl%4 == 0. perm as above (for
 * SPARK_LAYOUT_SEPARATE both halves get the same tiles). */
spark_status spark_positional_perm(const spark_params* p, int32_t F, int32_t Hl, int32_t Wl,
                                   int32_t* perm, cudaStream_t stream);

/* Step 3 - block statistics, summaries and top-K selection ([P1] "the exact
 * branch fully computes the top-ranked key/value blocks"; [P2] Inputs
 * topk_ratio). Block score s_ab = mean(q over block a) . mean(k over block b)
 * / sqrt(d); per query block the Ksel largest, ties to the lower b, written in
 * ascending order. Also leaves in ws the permuted copies of q, k, v and the
 * key/value summaries spark_attn_fwd reads. With SPARK_LAYOUT_SEPARATE query
 * blocks follow the query permutation and key blocks (and the k, v copies and
 * summaries) the key permutation.
 *   perm  : [B,H,N] int32 device (from spark_reblock, spark_positional_perm
 *           or the caller; must be a bijection per head)
 *   qmean : [B,H,d] float64 device (from spark_moments)
 *   sel   : [B,H,nb,Ksel] int32 device, written */
spark_status spark_select(const spark_params* p, const void* q, const void* k, const void* v,
                          const int32_t* perm, const double* qmean, int32_t* sel,
                          void* ws, size_t ws_bytes, cudaStream_t stream);

/* Step 4 - exact branch + compressed branch + merge ([P1] two branches;
 * [P2] real Q per query). For query i in permuted block a: exact logits
 * q_i.k_j/sqrt(d) for keys of the blocks in sel[a], compressed logits
 * q_i.k~_b/sqrt(d) + beta_b for every other block b, one softmax over both,
 * output row written at original index perm[pi].
 *   perm, sel : as passed to / produced by spark_select on the same ws
 *   out       : [B,H,N,d] bf16 device, written
 *   lse       : [B,H,N] float32 device natural-log softmax denominators in
 *               original token order, or NULL
 * Reads the permuted copies and summaries spark_select left in ws: call it
 * after spark_select with the same parameters, perm and ws, on the same
 * stream (sel may be replaced by the caller's own ascending lists). */
spark_status spark_attn_fwd(const spark_params* p, const int32_t* perm, const int32_t* sel,
                            void* out, float* lse, void* ws, size_t ws_bytes,
                            cudaStream_t stream);

/* Joint attention with an exact context segment (the video pass joined with
 * C text / audio / conditioning tokens, as in the model's joint attention
 * layers; "Spark-H3" news post, model section; reading: context tokens take
 * no part in moments, partition, selection or summaries). Video query i gets,
 * in its one softmax, its exact and compressed terms as in spark_attn_fwd
 * plus every context key j (logit q_i.kc_j/sqrt(d), value vc_j); context
 * query c attends densely to all N video keys and all C context keys.
 *   perm, sel       : as for spark_attn_fwd (spark_select ran on this ws)
 *   qc, kc, vc      : [B,H,C,d] bf16 device, C >= 1, 16-byte aligned
 *   out, lse        : video rows, as for spark_attn_fwd
 *   outc            : [B,H,C,d] bf16 device, written; lsec: [B,H,C] f32 or NULL
 * One kernel launch: video query pairs and context query chunks of 128
 * share the grid. */
spark_status spark_attn_fwd_joint(const spark_params* p, const int32_t* perm, const int32_t* sel,
                                  const void* qc, const void* kc, const void* vc, int32_t C, void* out,
                                  float* lse, void* outc, float* lsec, void* ws, size_t ws_bytes,
                                  cudaStream_t stream);

/* Steps 1-3 on the video tokens, then spark_attn_fwd_joint (perm and sel
 * stay in ws). */
spark_status spark_forward_joint(const spark_params* p, const void* q, const void* k, const void* v,
                                 const void* qc, const void* kc, const void* vc, int32_t C, void* out,
                                 float* lse, void* outc, float* lsec, void* ws, size_t ws_bytes,
                                 cudaStream_t stream);

/* The whole pass (steps 1-4) for device tensors. perm_out / sel_out are
 * optional device outputs (NULL: kept in ws). */
spark_status spark_forward(const spark_params* p, const void* q, const void* k, const void* v,
                           void* out, float* lse, int32_t* perm_out, int32_t* sel_out,
                           void* ws, size_t ws_bytes, cudaStream_t stream);

/* Number of kernel launches one spark_forward call makes for these params
 * (moments 2 or 3: a Gram per moment the layout uses, column sums for the
 * anchor when M_Q is not formed, a reduce; per partition, reblock 6 - whiten,
 * normalise, tree, init, subtree, leaves - plus 4 per tree level above the
 * first level whose groups all have at most 9 blocks, 5 when that level's
 * groups span several chunk CTAs; select 1 + 2 per chunk of heads (+1 for
 * the block tail); attention 2: query-block pairing, then the kernel); -1 if
 * invalid. */
int32_t spark_forward_launches(const spark_params* p);

/* Device bytes spark_forward_host needs: one workspace per compute lane
 * (below), each spark_workspace_size() of the largest head chunk run as a
 * problem of its own, plus room for device copies of q, k, v, out and lse of
 * all heads. At large head counts this is less than spark_workspace_size()
 * of the whole problem. */
size_t spark_host_workspace_size(const spark_params* p);

/* The whole pass for HOST tensors (pinned memory recommended): copies q, k,
 * v to the device, runs spark_forward, copies out (and lse if not NULL)
 * back. Heads are independent, so the pass runs as up to eight chunks of
 * consecutive heads (B*H flattened), each a problem of its own (B = 1,
 * H = its heads; results equal spark_forward's on the whole problem bit for
 * bit), pipelined: chunks are copied in one after another on a copy stream,
 * each is computed once it has arrived on one of two compute streams (chunk
 * c on stream c % 2, in that stream's own part of ws, so two chunks' kernels
 * may run at the same time) and copied out when done on a second copy
 * stream. These four streams belong to the library (created on first use
 * per device, kept for the life of the process); all of them start after
 * the work already queued on `stream`, and `stream` waits for the last copy
 * out.
 * Asynchronous like every call: the host buffers must stay valid until the
 * stream reaches the end of the call. ws is DEVICE memory of
 * spark_host_workspace_size() bytes. Calls from several host threads are
 * enqueued one at a time. */
spark_status spark_forward_host(const spark_params* p, const void* q_host, const void* k_host,
                                const void* v_host, void* out_host, float* lse_host,
                                void* ws, size_t ws_bytes, cudaStream_t stream);

/* Inspection of the workspace (for tests and tools): byte offset of one
 * region of the workspace a call with these params uses, and its size in
 * *bytes (if not NULL). Returns (size_t)-1 for an invalid block or region.
 * Regions hold: SPARK_WS_MQ/MK [B,H,d,d] f64 and SPARK_WS_QMEAN [B,H,d] f64
 * (spark_forward's moments), SPARK_WS_PERM [B,H,N] i32 and SPARK_WS_SEL
 * [B,H,nb,Ksel] i32 (spark_forward's layout and selection), SPARK_WS_QM/KM
 * [B,H,nb,d] f64 block means, SPARK_WS_KT/VT [B,H,nbp,d] bf16 summaries and
 * SPARK_WS_BETA [B,H,nbp] f32 biases with nbp = nb rounded up to 128 (rows
 * past nb are zero), SPARK_WS_UHAT [B,H,N,d] bf16 normalised whitened
 * tokens of the partitioned side (original token order), SPARK_WS_PAIRS
 * [B,H,(nb+1)/2] pairs of int32 (the query blocks each attention unit runs
 * together, written by spark_attn_fwd; partner -1 for a lone block). */
enum {
  SPARK_WS_MQ = 0, SPARK_WS_MK = 1, SPARK_WS_QMEAN = 2, SPARK_WS_PERM = 3, SPARK_WS_SEL = 4,
  SPARK_WS_QM = 5, SPARK_WS_KM = 6, SPARK_WS_KT = 7, SPARK_WS_VT = 8, SPARK_WS_BETA = 9,
  SPARK_WS_UHAT = 10, SPARK_WS_PAIRS = 11
};
size_t spark_workspace_region(const spark_params* p, int32_t region, size_t* bytes);

/* Diagnostic (the pages have no counterpart): checks that a device-side
 * timeout surfaces as an error and leaves the context usable. One warp
 * allocates tensor memory, waits through the bounded-wait routine every
 * kernel here uses on a barrier phase that nothing completes, gives up after
 * limit_ns, sets the device status word, frees its tensor memory and
 * returns; the next spark_get_status() reports SPARK_ERR_TIMEOUT and clears
 * it. No fault, trap or endless loop is involved.
 *   limit_ns : 1 .. 2e9 (the kernels' own limit is 2 s); outside that range
 *              SPARK_ERR_INVALID_ARG, nothing launched. */
spark_status spark_selftest_wait(int64_t limit_ns, cudaStream_t stream);

/* Synchronises the stream, reads and clears the device status word:
 * SPARK_OK, SPARK_ERR_TIMEOUT (a bounded wait expired) or SPARK_ERR_CUDA. */
spark_status spark_get_status(cudaStream_t stream);

/* Static description of a status code. */
const char* spark_strerror(spark_status s);

#ifdef __cplusplus
}
#endif
#endif /* SPARK_H_ */
