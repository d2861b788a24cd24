"""Second, loop-free statement of the forward pass for tiny inputs (N <= 256).

TEST INFRASTRUCTURE ONLY (see spark_oracle). It shares no helper with
spark_oracle: given a permutation it rebuilds block membership as a one-hot
matrix, forms the full N x N logit matrix and applies the per-pair rules of
the pages' two-branch structure ([P1] "What Spark-Attn changed": the exact
branch fully computes the top-ranked key/value blocks, the compressed branch
covers the rest; [P2] "What it's doing under the hood": a real Q per query,
only K/V downsampled; summaries weighted by the per-head mean query with a
log-mass correction). Used to pin spark_oracle on inputs small enough to
enumerate every (query, key) pair.
"""

from __future__ import annotations

import math

import numpy as np


def forward(q, k, v, perm, ksel, summary="reweight", tail="query", perm_k=None, context=None):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, d = q.shape
    nb = N // 64
    c = 1.0 / math.sqrt(d)

    # one-hot block membership of every original token, for queries and (when
    # keys are partitioned on their own) for keys
    def membership(pm):
        b = np.empty(N, dtype=np.int64)
        b[np.asarray(pm)] = np.arange(N) // 64
        return b, (b[:, None] == np.arange(nb)[None, :]).astype(np.float64)   # [N], [N, nb]
    blk, onehot = membership(perm)
    kblk, konehot = membership(perm if perm_k is None else perm_k)

    # block means and block scores
    Qm = onehot.T @ q / 64.0
    Km = konehot.T @ k / 64.0
    s = Qm @ Km.T * c
    # rank of each key block within its row: strictly better scores, or equal
    # scores at a lower block index, come first
    better = (s[:, None, :] > s[:, :, None]) | (
        (s[:, None, :] == s[:, :, None]) & (np.arange(nb)[None, None, :] < np.arange(nb)[None, :, None]))
    rank = better.sum(axis=2)                     # [nb(a), nb(b)]
    chosen = rank < ksel                          # query block a keeps key block b

    # summaries, all blocks at once
    qbar = q.mean(axis=0)
    if summary == "meanpool":
        kt = Km.copy()
        vt = konehot.T @ v / 64.0
        beta = np.full(nb, math.log(64.0))
    else:
        x = k @ qbar * c                          # anchor logits [N]
        xmax = np.where(konehot > 0, x[:, None], -np.inf).max(axis=0)   # [nb]
        ex = np.exp(x - xmax[kblk])
        Z = konehot.T @ ex
        kt = (konehot.T @ (ex[:, None] * k)) / Z[:, None]
        vt = (konehot.T @ (ex[:, None] * v)) / Z[:, None]
        beta = xmax + np.log(Z) - kt @ qbar * c

    # per-pair rules
    exact_mask = chosen[blk][:, kblk]             # [N, N]: key j's block is kept for query i
    comp_mask = ~chosen[blk]                      # [N, nb]: block b is summarised for query i
    L_exact = np.where(exact_mask, q @ k.T * c, -np.inf)
    # compressed logits with each query's own q, or (tail granularity "block")
    # with the mean query of the permuted block it sits in
    qc = q if tail == "query" else Qm[blk]
    L_comp = np.where(comp_mask, qc @ kt.T * c + beta[None, :], -np.inf)
    if context is not None:
        # joint attention: every context key is an exact term for every video
        # query; context queries see every key of both segments
        qc, kc, vc = (np.asarray(x, dtype=np.float64) for x in context)
        L_exact = np.concatenate([L_exact, q @ kc.T * c], axis=1)
        v_exact = np.concatenate([v, vc], axis=0)
    else:
        v_exact = v
    m = np.maximum(L_exact.max(axis=1), L_comp.max(axis=1))
    E = np.exp(L_exact - m[:, None])
    C = np.exp(L_comp - m[:, None])
    den = E.sum(axis=1) + C.sum(axis=1)
    out = (E @ v_exact + C @ vt) / den[:, None]
    lse = m + np.log(den)
    res = {"out": out, "lse": lse, "chosen": chosen, "kt": kt, "vt": vt, "beta": beta,
           "qm": Qm, "km": Km}
    if context is not None:
        Lc = qc @ np.concatenate([k, kc]).T * c                         # [C, N + C]
        mc = Lc.max(axis=1)
        Ec = np.exp(Lc - mc[:, None])
        denc = Ec.sum(axis=1)
        res["outc"] = Ec @ np.concatenate([v, vc]) / denc[:, None]
        res["lsec"] = mc + np.log(denc)
    return res
