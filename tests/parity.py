"""Comparison protocol between the CUDA path and the CPU oracle.

Layered: the permutation is checked node by node with the oracle replaying
every split on the CUDA path's own parent set (so one near-tie does not
cascade); the selection is checked given the CUDA permutation; summaries
and outputs are checked given the CUDA permutation and selection.

Where floating point decides an integer (which side of a cut a token falls
on, whether a block makes the top-K) and the oracle's float64 value sits
within the tolerance of the decision boundary, both answers are correct up
to rounding: such a disagreement is a certified near-tie and is counted,
anything farther is a failure.

Tolerances (derived in the design notes):
  TAU_P   cut certification, relative to the projection range of the node
  TAU_S   selection certification, relative to 1 + max |score| of the row
  OUT_TOL spec output bound |err| <= 1e-2 * (1 + |ref|)
"""

from __future__ import annotations

import math

import numpy as np

from oracle import spark_oracle as so

TAU_P = 1e-5
TAU_S = 1e-9


def check_perm_structure(perm, N):
    """Bijection, and ascending original index inside every 64-token leaf."""
    assert perm.shape == (N,)
    assert np.array_equal(np.sort(perm), np.arange(N))
    blocks = perm.reshape(-1, 64)
    assert np.all(np.diff(blocks, axis=1) > 0)


def certify_perm(x, M, perm, tau=TAU_P, U=None, iters=so.POWER_ITERS):
    """Replay the oracle's splits on the CUDA path's sets.

    x: [N, d] float64 (partitioned side), M: float64 moment of the opposite
    side (the oracle's own). U: the normalised whitened vectors to split on;
    by default the oracle's own, or the CUDA path's (after they passed their
    own elementwise check) so that an isolated rounding flip of one element
    is judged at the normalisation step, not again at every cut. Returns
    dict(nodes, mismatched, certified, failures, worst) where worst is the
    largest |p - cut| / range among the mismatched tokens."""
    N = x.shape[0]
    nb = N // 64
    check_perm_structure(perm, N)
    if U is None:
        U = so.normalized_whitened(x, so.whitening_factor(M))
    stats = dict(nodes=0, mismatched=0, certified=0, failures=0, worst=0.0, fail_detail=[])
    for level in so.tree_nodes(nb):
        for first, g in level:
            ids = perm[64 * first:64 * (first + g)]
            left, _, info = so.split_group(U[ids], ids, iters)
            gl = set(perm[64 * first:64 * (first + g // 2)].tolist())
            ol = set(left.tolist())
            stats["nodes"] += 1
            if gl == ol:
                continue
            bad = np.array(sorted(gl ^ ol))
            where = {int(t): i for i, t in enumerate(ids)}
            p = info["p"][[where[int(t)] for t in bad]]
            rng = max(info["range"], 1e-300)
            dist = np.abs(p - info["cut"]) / rng
            stats["mismatched"] += len(bad)
            stats["worst"] = max(stats["worst"], float(dist.max()))
            ok = dist <= tau
            stats["certified"] += int(ok.sum())
            stats["failures"] += int((~ok).sum())
            if (~ok).any():
                stats["fail_detail"].append((first, g, float(dist.max())))
    return stats


def certify_select(qm, km, ksel, sel, tau=TAU_S):
    """sel (CUDA) against the oracle's top-K of the float64 block scores."""
    s = so.block_scores(qm, km)
    ref = so.select(qm, km, ksel)
    stats = dict(rows=s.shape[0], mismatched=0, certified=0, failures=0)
    for a in range(s.shape[0]):
        g = sel[a]
        assert np.all(np.diff(g) > 0), "selection must be ascending and unique"
        if np.array_equal(g, ref[a]):
            continue
        kth = np.sort(s[a])[::-1][ksel - 1]
        bad = np.setxor1d(g, ref[a])
        dist = np.abs(s[a][bad] - kth)
        tol = tau * (1.0 + np.abs(s[a]).max())
        stats["mismatched"] += len(bad)
        stats["certified"] += int((dist <= tol).sum())
        stats["failures"] += int((dist > tol).sum())
    return stats


def out_errors(got, ref):
    """Error summary of attention rows (float arrays of equal shape)."""
    err = np.abs(got - ref)
    bound = 1e-2 * (1.0 + np.abs(ref))
    return dict(max_abs=float(err.max()), mean_abs=float(err.mean()),
                max_rel_to_bound=float((err / bound).max()),
                ref_rms=float(math.sqrt((ref * ref).mean())))
