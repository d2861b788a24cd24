"""CPU oracle for the Spark-Attn forward pass.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference legs may import this module. The CUDA library never
calls it and shares no code with it.

A plain, slow, float64 NumPy statement of what the forward pass computes, step
by step, in the order the pages describe it. Sources (web pages):
  [P1] "Spark-H3: block-sparse attention speeds up MiniMax-H3 in ComfyUI"
       (comfyui-wiki news, 2026-10-11), sections "What Spark-Attn changed",
       "Benchmark", "Workflows".
  [P2] "MiniMax H3 Spark Attention (SM89)" (comfy.icu node page), sections
       "What it's doing under the hood" and "Inputs you'll actually set".
No page prints a formula; every formula below is a reading of the prose. The
readings are numbered R1..R13 and listed with their reasons in the design
notes of this repository.

Inputs are per (batch item, head): q, k, v as float64 arrays [N, d] holding
bfloat16 values. Block size is 64 tokens (R1, [P2] "exactly 64-token leaves").
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 64          # R1: exactly 64-token leaves ([P2] under the hood)
POWER_ITERS = 16    # R6: fixed power-iteration count
REG_EPS = 1e-6      # R3: relative diagonal jitter before the Cholesky factor
SEL_EPS = 1e-9      # R9: guard in ceil(r * nb - eps)


# --------------------------------------------------------------------------
# helpers written for the oracle alone

def round_bf16(x):
    """Round float64 values to the nearest bfloat16 value (ties to even).

    Single rounding straight from float64: write x = m * 2**e with
    0.5 <= |m| < 1, keep 8 significant bits of m with round-half-even, scale
    back. (bfloat16 normal range only; the oracle's values stay inside it.)
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def num_selected(nb: int, ratio: float = 0.0, blocks: int = 0) -> int:
    """R9: blocks kept per query block. Fixed count if given ([P2] topk_blocks),
    else ceil(ratio * nb) clamped to [1, nb] ([P2] topk_ratio)."""
    if blocks > 0:
        return min(int(blocks), nb)
    k = math.ceil(ratio * nb - SEL_EPS)
    return max(1, min(nb, k))


# --------------------------------------------------------------------------
# a1. second moments and anchor

def second_moment(x):
    """R2: uncentered second moment E[x x^T] = (1/N) sum_i x_i x_i^T over all N
    tokens of one head ([P2] under the hood: M_K = E[k k^T], M_Q likewise)."""
    x = np.asarray(x, dtype=np.float64)
    return x.T @ x / x.shape[0]


def anchor(q):
    """R2: the per-head mean video query used as the anchor of the summaries
    ([P1] "What Spark-Attn changed", Spark-Reweight bullet)."""
    return np.asarray(q, dtype=np.float64).mean(axis=0)


# --------------------------------------------------------------------------
# a2. reblock

def whitening_factor(M):
    """R3/R4: lower Cholesky factor L of the regularised moment,
    M + 1e-6 * (tr M / d) * I = L L^T. Whitened token u = L^T x, so that
    u_i . u_j = x_i^T M x_j and the cosine of whitened vectors is the
    Mahalanobis cosine ([P1] Spark-Reblock bullet; [P2] under the hood).
    An all-zero moment (tr M == 0) whitens with the identity."""
    M = np.asarray(M, dtype=np.float64)
    d = M.shape[0]
    tr = float(np.trace(M))
    if tr == 0.0:
        return np.eye(d)
    return np.linalg.cholesky(M + REG_EPS * (tr / d) * np.eye(d))


def normalized_whitened(x, L):
    """R7: u_hat_i = bf16(u_i / ||u_i||) with u_i = L^T x_i; zero stays zero.
    Rows of the result are the vectors the partitioner works on."""
    u = np.asarray(x, dtype=np.float64) @ L
    n = np.sqrt((u * u).sum(axis=1))
    out = np.zeros_like(u)
    nz = n > 0
    out[nz] = u[nz] / n[nz, None]
    return round_bf16(out)


def split_direction(U, iters=POWER_ITERS):
    """R6: top principal direction of the group's centered covariance by a
    fixed number of power iterations from the all-ones direction (iters; the
    "Lite" reblock takes fewer, reading R18).

    U: [n, d] normalised whitened vectors of one group. Returns (v, mu, p)
    where p_i = v . (U_i - mu) is each token's projection."""
    n, d = U.shape
    mu = U.mean(axis=0)
    C = U - mu
    S = C.T @ C / n
    v = np.full(d, 1.0 / math.sqrt(d))
    for _ in range(iters):
        w = S @ v
        nw = math.sqrt(float(w @ w))
        if nw == 0.0:
            v = np.zeros(d)
            break
        v = w / nw
    p = C @ v
    return v, mu, p


def split_group(U, ids, iters=POWER_ITERS):
    """R6: capacity-constrained bisection of one group of g = n/64 blocks
    ([P1] "the hierarchical partitioner keeps splitting groups until every
    leaf reaches the target block size"; [P2] "capacity-constrained tree
    partition down to exactly 64-token leaves").

    U: [n, d] rows for the tokens ids (original token indices, any order).
    Orientation: the token with the largest |p| (lowest index on ties) gets a
    positive projection. Tokens are ranked by (p, index) ascending; the
    first 64*floor(g/2) go left. Returns (left_ids, right_ids, info)."""
    ids = np.asarray(ids)
    n = ids.shape[0]
    g = n // BLOCK
    v, mu, p = split_direction(U, iters)
    a = np.abs(p)
    top = ids[a == a.max()].min()
    if p[ids == top][0] < 0:
        p = -p
    order = np.lexsort((ids, p))       # primary p, then index
    nl = BLOCK * (g // 2)
    left, right = ids[order[:nl]], ids[order[nl:]]
    ps = p[order]
    cut = 0.5 * (ps[nl - 1] + ps[nl]) if 0 < nl < n else 0.0
    info = {"v": v, "mu": mu, "p": p, "ids": ids, "cut": cut,
            "range": float(p.max() - p.min())}
    return left, right, info


def tree_nodes(nb: int):
    """The tree's shape depends on nb alone: list per level of
    (first_block, g) for every group that still splits (g >= 2)."""
    levels = []
    cur = [(0, nb)]
    while True:
        todo = [(f, g) for (f, g) in cur if g >= 2]
        if not todo:
            break
        levels.append(todo)
        nxt = []
        for f, g in todo:
            nxt.append((f, g // 2))
            nxt.append((f + g // 2, g - g // 2))
        cur = nxt
    return levels


def reblock(x, M, iters=POWER_ITERS):
    """a2 Reblock, R5-R8: partition tokens of one head into 64-token blocks.

    x: the side that is partitioned (queries for q_reuse_k), M: the opposite
    side's second moment (M_K for queries). Returns perm [N] (int64):
    perm[pi] = original index of the token at permuted position pi. Leaves
    are laid out left to right in depth-first order; inside a leaf, tokens are
    in ascending original index (R8). Only membership matters: Q/K/V values
    are never modified ([P2] under the hood)."""
    x = np.asarray(x, dtype=np.float64)
    N = x.shape[0]
    U = normalized_whitened(x, whitening_factor(M))

    def rec(ids):
        if ids.shape[0] <= BLOCK:
            return [np.sort(ids)]
        left, right, _ = split_group(U[ids], ids, iters)
        return rec(left) + rec(right)

    leaves = rec(np.arange(N))
    return np.concatenate(leaves)


def positional_tiles(grid, tile=(2, 8, 4)):
    """R13: fixed spatio-temporal tiles (the plain block-sparse layout that
    Spark-Reblock replaces, [P1] Spark-Reblock bullet). Tiles of 2x8x4
    (frame, row, column) in raster order of tiles; inside a tile, ascending
    original index. Tokens are in raster order t = (f*Hl + y)*Wl + x (R14)."""
    F, Hl, Wl = grid
    tf, ty, tx = tile
    assert F % tf == 0 and Hl % ty == 0 and Wl % tx == 0
    t = np.arange(F * Hl * Wl).reshape(F, Hl, Wl)
    t = t.reshape(F // tf, tf, Hl // ty, ty, Wl // tx, tx)
    t = t.transpose(0, 2, 4, 1, 3, 5).reshape(-1, tf * ty * tx)
    return np.sort(t, axis=1).reshape(-1)


# --------------------------------------------------------------------------
# a3. block statistics and summaries

def block_means(x, perm):
    """Mean of the original (unpermuted) values over each permuted block."""
    x = np.asarray(x, dtype=np.float64)
    nb = perm.shape[0] // BLOCK
    return x[perm].reshape(nb, BLOCK, -1).mean(axis=1)


def summaries(k, v, perm, qbar, mode="reweight"):
    """a3, R10: one summary per key block ([P1] Spark-Reweight bullet and the
    figure caption; [P2] "Reweight replaces mean-pooled summaries ... with
    weighted ones plus a log-mass correction").

    reweight: anchor logits x_j = qbar . k_j / sqrt(d) inside block b,
      w = softmax(x), k~_b = sum w_j k_j, v~_b = sum w_j v_j and
      beta_b = ln sum_j exp(x_j) - qbar . k~_b / sqrt(d), so that the pooled
      logit qbar . k~_b / sqrt(d) + beta_b carries exactly the block's exp-mass
      for the anchor query (E[exp x] rather than exp E[x], times 64 tokens).
    meanpool (ablation): k~ = mean k, v~ = mean v, beta = ln 64.
    Returns (kt [nb,d], vt [nb,d], beta [nb])."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d = k.shape[1]
    nb = perm.shape[0] // BLOCK
    kt = np.zeros((nb, d))
    vt = np.zeros((nb, d))
    beta = np.zeros(nb)
    scale = 1.0 / math.sqrt(d)
    for b in range(nb):
        rows = perm[b * BLOCK:(b + 1) * BLOCK]
        Kb, Vb = k[rows], v[rows]
        if mode == "meanpool":
            kt[b] = Kb.mean(axis=0)
            vt[b] = Vb.mean(axis=0)
            beta[b] = math.log(BLOCK)
            continue
        xlog = Kb @ qbar * scale
        mx = xlog.max()
        e = np.exp(xlog - mx)
        Z = e.sum()
        w = e / Z
        kt[b] = w @ Kb
        vt[b] = w @ Vb
        beta[b] = (mx + math.log(Z)) - float(qbar @ kt[b]) * scale
    return kt, vt, beta


# --------------------------------------------------------------------------
# a4. block selection

def block_scores(qm, km):
    """s_ab = Qbar_a . Kbar_b / sqrt(d) for every query block a, key block b."""
    return qm @ km.T / math.sqrt(qm.shape[1])


def select(qm, km, ksel):
    """a4, R9: per query block the ksel key blocks with the highest block
    score ([P1] "the exact branch fully computes the top-ranked key/value
    blocks"), ties to the lower block index, returned in ascending order."""
    s = block_scores(qm, km)
    nb = s.shape[1]
    idx = np.arange(nb)
    sel = np.empty((s.shape[0], ksel), dtype=np.int64)
    for a in range(s.shape[0]):
        order = np.lexsort((idx, -s[a]))   # primary -s (descending), then b
        sel[a] = np.sort(order[:ksel])
    return sel


# --------------------------------------------------------------------------
# a5-a7. exact branch, compressed branch, merge

def attention(q, k, v, perm, sel, kt, vt, beta, rows=None, tail="query", qm=None, perm_k=None):
    """a5-a7, R11: each query i in permuted block a attends exactly to every
    key of its selected blocks ([P1] exact branch) and, with its own real q_i
    ([P2] "keeps a real Q per query and downsamples only K/V"), to the summary
    of every unselected block with logit q_i . k~_b / sqrt(d) + beta_b. The two
    branches are one softmax: o_i = (sum_exact e^s v_j + sum_comp e^l v~_b) /
    (sum_exact e^s + sum_comp e^l), i.e. the log-sum-exp merge of the two
    partial softmaxes. The row is written at the token's original index.

    tail="block" is the coarser tail granularity ([P2] Inputs,
    tail_granularity; reading R15): the compressed logits of every query in
    block a use the block's mean query Qbar_a (block_means of q, the same
    means the selection scores use) instead of the query itself; the exact
    branch keeps the real q_i. qm: those block means (computed if None).

    perm_k: the key (and value) permutation when keys are partitioned apart
    from the queries (layout "separate"; default: perm for both). Query block
    a is perm's block a; key block b is perm_k's block b.

    rows: optional iterable of query blocks to evaluate (default all).
    Returns out [N, d] (rows of skipped blocks are NaN) and lse [N] (natural
    log of the softmax denominator)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, d = q.shape
    nb = N // BLOCK
    scale = 1.0 / math.sqrt(d)
    if tail not in ("query", "block"):
        raise ValueError(tail)
    if perm_k is None:
        perm_k = perm
    if tail == "block" and qm is None:
        qm = block_means(q, perm)
    out = np.full((N, d), np.nan)
    lse = np.full(N, np.nan)
    blocks = range(nb) if rows is None else rows
    for a in blocks:
        qrow = perm[a * BLOCK:(a + 1) * BLOCK]
        Qa = q[qrow]
        chosen = np.zeros(nb, dtype=bool)
        chosen[sel[a]] = True
        krows = np.concatenate([perm_k[b * BLOCK:(b + 1) * BLOCK] for b in sel[a]])
        s_exact = Qa @ k[krows].T * scale
        if tail == "query":
            s_comp = Qa @ kt[~chosen].T * scale + beta[~chosen]
        else:
            s_comp = np.broadcast_to(np.asarray(qm[a], dtype=np.float64) @ kt[~chosen].T * scale + beta[~chosen],
                                     (BLOCK, int((~chosen).sum())))
        m = np.maximum(s_exact.max(axis=1),
                       s_comp.max(axis=1) if s_comp.shape[1] else -np.inf)
        e_exact = np.exp(s_exact - m[:, None])
        e_comp = np.exp(s_comp - m[:, None])
        den = e_exact.sum(axis=1) + e_comp.sum(axis=1)
        num = e_exact @ v[krows] + e_comp @ vt[~chosen]
        out[qrow] = num / den[:, None]
        lse[qrow] = m + np.log(den)
    return out, lse


def joint_attention(q, k, v, perm, sel, kt, vt, beta, qc, kc, vc, rows=None, tail="query", qm=None,
                    perm_k=None):
    """Joint attention with an exact, dense context segment (reading R17;
    the step either side of the path in the real model: text / audio /
    conditioning tokens attend jointly with the video tokens). The video
    tokens go through the method unchanged (moments, partition, selection and
    summaries from video tokens only); each video query additionally attends
    exactly to every context key, inside the same softmax as its exact and
    compressed terms; each context query attends densely to all N video keys
    and all C context keys.

    qc, kc, vc: [C, d] context tokens. Returns (out [N, d], lse [N], outc
    [C, d], lsec [C]); rows of skipped video blocks are NaN."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    qc = np.asarray(qc, dtype=np.float64)
    kc = np.asarray(kc, dtype=np.float64)
    vc = np.asarray(vc, dtype=np.float64)
    if perm_k is None:
        perm_k = perm
    N, d = q.shape
    nb = N // BLOCK
    scale = 1.0 / math.sqrt(d)
    if tail == "block" and qm is None:
        qm = block_means(q, perm)
    out = np.full((N, d), np.nan)
    lse = np.full(N, np.nan)
    blocks = range(nb) if rows is None else rows
    for a in blocks:
        qrow = perm[a * BLOCK:(a + 1) * BLOCK]
        Qa = q[qrow]
        chosen = np.zeros(nb, dtype=bool)
        chosen[sel[a]] = True
        krows = np.concatenate([perm_k[b * BLOCK:(b + 1) * BLOCK] for b in sel[a]])
        s_exact = np.concatenate([Qa @ k[krows].T, Qa @ kc.T], axis=1) * scale
        vals = np.concatenate([v[krows], vc], axis=0)
        if tail == "query":
            s_comp = Qa @ kt[~chosen].T * scale + beta[~chosen]
        else:
            s_comp = np.broadcast_to(np.asarray(qm[a], dtype=np.float64) @ kt[~chosen].T * scale + beta[~chosen],
                                     (BLOCK, int((~chosen).sum())))
        m = np.maximum(s_exact.max(axis=1), s_comp.max(axis=1) if s_comp.shape[1] else -np.inf)
        e_exact = np.exp(s_exact - m[:, None])
        e_comp = np.exp(s_comp - m[:, None])
        den = e_exact.sum(axis=1) + e_comp.sum(axis=1)
        out[qrow] = (e_exact @ vals + e_comp @ vt[~chosen]) / den[:, None]
        lse[qrow] = m + np.log(den)
    outc, lsec = dense_attention(qc, np.concatenate([k, kc]), np.concatenate([v, vc]))
    return out, lse, outc, lsec


def dense_attention(q, k, v):
    """Plain softmax attention (the density-1.0 limit of the method) and its
    natural-log denominators (lse)."""
    q = np.asarray(q, dtype=np.float64)
    s = q @ np.asarray(k, dtype=np.float64).T / math.sqrt(q.shape[1])
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    den = e.sum(axis=1, keepdims=True)
    return e @ np.asarray(v, dtype=np.float64) / den, (m + np.log(den))[:, 0]


# --------------------------------------------------------------------------
# whole forward pass of one head

def forward_head(q, k, v, ratio=0.2, topk_blocks=0, layout="q_reuse_k",
                 summary="reweight", perm=None, rows=None, tail="query", perm_k=None,
                 power_iters=POWER_ITERS):
    """Every intermediate of the forward pass for one (batch item, head).

    layout: "q_reuse_k" partitions the queries under M_K and reuses that
    partition for K and V (R5, [P1] workflows pin reblock_layout=q_reuse_k);
    "k_reuse_q" is the mirror (keys under M_Q); "separate" partitions the
    queries under M_K and the keys (with their values) under M_Q, each on its
    own ([P2] under the hood: queries grouped under E[kk^T], keys under
    E[qq^T]; reading R16); "given" uses perm as is (perm_k too, if given)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, d = q.shape
    nb = N // BLOCK
    MQ, MK, qbar = second_moment(q), second_moment(k), anchor(q)
    if layout == "q_reuse_k":
        perm = reblock(q, MK, power_iters)
    elif layout == "k_reuse_q":
        perm = reblock(k, MQ, power_iters)
    elif layout == "separate":
        perm, perm_k = reblock(q, MK, power_iters), reblock(k, MQ, power_iters)
    elif layout != "given":
        raise ValueError(layout)
    perm = np.asarray(perm)
    perm_k = perm if perm_k is None else np.asarray(perm_k)
    ksel = num_selected(nb, ratio, topk_blocks)
    qm, km = block_means(q, perm), block_means(k, perm_k)
    sel = select(qm, km, ksel)
    kt, vt, beta = summaries(k, v, perm_k, qbar, summary)
    out, lse = attention(q, k, v, perm, sel, kt, vt, beta, rows=rows, tail=tail, qm=qm, perm_k=perm_k)
    return {"MQ": MQ, "MK": MK, "qbar": qbar, "perm": perm, "perm_k": perm_k, "ksel": ksel,
            "qm": qm, "km": km, "sel": sel, "kt": kt, "vt": vt, "beta": beta,
            "out": out, "lse": lse}


# --------------------------------------------------------------------------
# statistics the pages name (oracle only)

def mass_recall(q, k, perm, sel, rows, perm_k=None):
    """R12: attention-mass recall ([P2] "+12.88 points of attention-mass
    recall"): for each sampled query, the share (in percent) of its dense
    softmax mass that falls on keys of its selected blocks. rows: permuted
    query blocks to sample; perm_k: the key permutation (default perm; the
    separate layout's key blocks, R16). Returns the mean over their queries."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    perm_k = perm if perm_k is None else perm_k
    N, d = q.shape
    nb = N // BLOCK
    blk = np.empty(N, dtype=np.int64)
    blk[perm_k] = np.arange(N) // BLOCK
    vals = []
    for a in rows:
        Qa = q[perm[a * BLOCK:(a + 1) * BLOCK]]
        s = Qa @ k.T / math.sqrt(d)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        chosen = np.zeros(nb, dtype=bool)
        chosen[sel[a]] = True
        vals.append(100.0 * e[:, chosen[blk]].sum(axis=1) / e.sum(axis=1))
    return float(np.concatenate(vals).mean())


def log_mass_error(q, k, perm, sel, kt, beta, rows, perm_k=None):
    """R12: absolute log-mass error ([P2] "-28% absolute log-mass error"):
    the plain (unweighted) mean over sampled queries i and unselected blocks b
    of |(q_i . k~_b / sqrt(d) + beta_b) - ln sum_{j in b} exp(q_i . k_j / sqrt(d))|.
    Key block b is block b of perm_k (default perm; the separate layout's key
    permutation, R16)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    perm_k = perm if perm_k is None else perm_k
    N, d = q.shape
    nb = N // BLOCK
    scale = 1.0 / math.sqrt(d)
    Kb = k[perm_k].reshape(nb, BLOCK, d)
    errs = []
    for a in rows:
        Qa = q[perm[a * BLOCK:(a + 1) * BLOCK]]
        chosen = np.zeros(nb, dtype=bool)
        chosen[sel[a]] = True
        for b in np.nonzero(~chosen)[0]:
            s = Qa @ Kb[b].T * scale
            m = s.max(axis=1)
            true = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
            pooled = Qa @ kt[b] * scale + beta[b]
            errs.append(np.abs(pooled - true))
    return float(np.concatenate(errs).mean()) if errs else 0.0
