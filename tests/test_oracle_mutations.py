"""Plant plausible mistakes in the oracle (on the CPU) and check that at least
one pin catches each of them. The mutations are undone after every test."""

import math

import numpy as np
import pytest

import tests.test_oracle_pins as pins
from oracle import spark_oracle as so

_orig = {name: getattr(so, name) for name in
         ("summaries", "whitening_factor", "split_direction", "select", "attention",
          "split_group", "round_bf16", "block_means", "dense_attention", "log_mass_error")}


def _beta_without_anchor_term(k, v, perm, qbar, mode="reweight"):
    kt, vt, beta = _orig["summaries"](k, v, perm, qbar, mode)
    d = k.shape[1]
    return kt, vt, beta + kt @ qbar / math.sqrt(d)


def _meanpool_without_count(k, v, perm, qbar, mode="reweight"):
    kt, vt, beta = _orig["summaries"](k, v, perm, qbar, mode)
    return kt, vt, beta - math.log(64)


def _transposed_factor(M):
    return _orig["whitening_factor"](M).T


def _uncentered_direction(U):
    n, d = U.shape
    S = U.T @ U / n
    v = np.full(d, 1 / math.sqrt(d))
    for _ in range(so.POWER_ITERS):
        v = S @ v
        v /= np.linalg.norm(v)
    mu = U.mean(axis=0)
    return v, mu, (U - mu) @ v


def _select_lowest(qm, km, ksel):
    return _orig["select"](-qm, km, ksel)


def _attention_unscaled(q, k, v, perm, sel, kt, vt, beta, rows=None, **kw):
    s = math.sqrt(q.shape[1])
    return _orig["attention"](q * s, k, v, perm, sel, kt, vt, beta, rows, **kw)


def _block_tail_from_head_anchor(q, k, v, perm, sel, kt, vt, beta, rows=None, tail="query", qm=None, **kw):
    # block tail built from the head's mean query instead of each block's
    if tail == "block":
        qm = np.repeat(np.asarray(q, dtype=np.float64).mean(axis=0)[None, :], len(q) // 64, axis=0)
    return _orig["attention"](q, k, v, perm, sel, kt, vt, beta, rows, tail=tail, qm=qm, **kw)


def _context_rows_without_context_keys(q, k, v):
    # context queries that only see the video keys (the context segment dropped)
    return _orig["dense_attention"](q, k[: len(k) - len(k) % 64], v[: len(v) - len(v) % 64])


def _keys_through_query_perm(q, k, v, perm, sel, kt, vt, beta, rows=None, perm_k=None, **kw):
    # separate layout: key blocks looked up through the query permutation
    return _orig["attention"](q, k, v, perm, sel, kt, vt, beta, rows, perm_k=perm, **kw)


def _signed_log_mass_error(q, k, perm, sel, kt, beta, rows, perm_k=None):
    # the error without its absolute value (signed deviations cancel)
    d = q.shape[1]
    out = []
    for a in rows:
        Qa = q[perm[64 * a:64 * (a + 1)]]
        for b in np.setdiff1d(np.arange(len(q) // 64), sel[a]):
            s = Qa @ k[(perm if perm_k is None else perm_k)[64 * b:64 * (b + 1)]].T / math.sqrt(d)
            true = np.log(np.exp(s).sum(axis=1))
            out.append(Qa @ kt[b] / math.sqrt(d) + beta[b] - true)
    return float(np.concatenate(out).mean())


def _mass_weighted_log_mass_error(q, k, perm, sel, kt, beta, rows, perm_k=None):
    # the error averaged with each (query, block)'s true softmax mass as weight
    d = q.shape[1]
    num = den = 0.0
    for a in rows:
        Qa = q[perm[64 * a:64 * (a + 1)]]
        for b in np.setdiff1d(np.arange(len(q) // 64), sel[a]):
            s = Qa @ k[(perm if perm_k is None else perm_k)[64 * b:64 * (b + 1)]].T / math.sqrt(d)
            true = np.log(np.exp(s).sum(axis=1))
            w = np.exp(true)
            num += float((w * np.abs(Qa @ kt[b] / math.sqrt(d) + beta[b] - true)).sum())
            den += float(w.sum())
    return num / den


def _truncating_round(x):
    m, e = np.frexp(np.asarray(x, dtype=np.float64))
    return np.ldexp(np.trunc(np.ldexp(m, 8)), e - 8)


def _block_sum_not_mean(x, perm):
    return _orig["block_means"](x, perm) * 64


def _split_ceil_left(U, ids):
    left, right, info = _orig["split_group"](U, ids)
    g = len(ids) // 64
    if g % 2:
        both = np.concatenate([left, right])
        left, right = both[: 64 * (g // 2 + 1)], both[64 * (g // 2 + 1):]
    return left, right, info


MUTANTS = [
    ("summaries", _beta_without_anchor_term, [pins.test_beta_is_entropy_of_anchor_weights]),
    ("summaries", _meanpool_without_count, [pins.test_compressed_branch_exact_for_identical_keys]),
    ("whitening_factor", _transposed_factor, [pins.test_whitening_inner_products_are_mahalanobis]),
    ("split_direction", _uncentered_direction, [pins.test_split_direction_is_top_eigenvector]),
    ("select", _select_lowest, [pins.test_select_against_full_sort]),
    ("attention", _attention_unscaled, [pins.test_density_one_is_dense_attention]),
    ("attention", _block_tail_from_head_anchor,
     [lambda: pins.test_block_tail_matches_brute_force(256, 8, 0.25, "reweight")]),
    ("dense_attention", _context_rows_without_context_keys,
     [lambda: pins.test_joint_attention_matches_brute_force(128, 8, 0.5, 7)]),
    ("attention", _keys_through_query_perm,
     [lambda: pins.test_separate_layout_matches_brute_force(256, 8, 0.25, "reweight")]),
    ("round_bf16", _truncating_round, [pins.test_round_bf16_matches_bit_rounding]),
    ("log_mass_error", _signed_log_mass_error, [pins.test_log_mass_error_brute_force]),
    ("log_mass_error", _mass_weighted_log_mass_error, [pins.test_log_mass_error_brute_force]),
    ("split_group", _split_ceil_left, [pins.test_split_group_orientation_and_capacity]),
]


@pytest.mark.parametrize("name,mutant,catchers", MUTANTS, ids=[m[1].__name__ for m in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, name, mutant, catchers):
    monkeypatch.setattr(so, name, mutant)
    caught = 0
    for t in catchers:
        try:
            t()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the mutation of {name}"


def test_brute_force_catches_block_sum_mistake(monkeypatch):
    monkeypatch.setattr(so, "block_means", _block_sum_not_mean)
    # scaling block means by 64 keeps the ranking, so selection pins alone do
    # not see it; nothing downstream uses the scale, so this checks the pins
    # stay green for a harmless change (no false alarm)
    pins.test_oracle_matches_brute_force(256, 8, 0.25, "reweight")
