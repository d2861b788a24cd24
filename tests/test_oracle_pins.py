"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle function against a closed form, a textbook
routine, brute force or an invariant the pages fix. No GPU needed.
"""

import math

import numpy as np
import pytest

from oracle import brute_force
from oracle import spark_oracle as so
from spark_gen import WORKLOADS, bf16_bits_to_f64, f32_to_bf16_bits, make_inputs

RNG = np.random.default_rng(1234)


def bf16(x):
    """Values rounded to bfloat16 through the generator's bit routine."""
    return bf16_bits_to_f64(f32_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def rand_qkv(N, d, scale=1.0, seed=0):
    r = np.random.default_rng(seed)
    q = bf16(r.standard_normal((N, d)) * scale)
    k = bf16(r.standard_normal((N, d)) * scale)
    v = bf16(r.standard_normal((N, d)))
    return q, k, v


# ------------------------------------------------------------------ rounding

def test_round_bf16_matches_bit_rounding():
    x = RNG.standard_normal(20000).astype(np.float32) * np.exp(RNG.uniform(-20, 20, 20000)).astype(np.float32)
    assert np.array_equal(so.round_bf16(x.astype(np.float64)), bf16(x))


def test_round_bf16_ties_to_even():
    one = 1.0
    ulp = 2.0 ** -7            # bf16 spacing just above 1
    assert so.round_bf16(one + ulp / 2) == one                 # tie -> even (1.0)
    assert so.round_bf16(one + 1.5 * ulp) == one + 2 * ulp     # tie -> even mantissa
    assert so.round_bf16(one + ulp / 2 + 1e-12) == one + ulp   # just above the tie
    assert so.round_bf16(-(one + ulp / 2)) == -one
    assert so.round_bf16(0.0) == 0.0


# ------------------------------------------------------------------ Ksel

def test_num_selected_values():
    # ceil(r * nb), clamped; the ratios 0.1/0.2/0.3 of the node's topk_ratio input
    assert so.num_selected(1134, 0.1) == 114
    assert so.num_selected(1134, 0.2) == 227
    assert so.num_selected(1134, 0.3) == 341
    assert so.num_selected(64, 0.2) == 13
    assert so.num_selected(252, 0.1) == 26
    assert so.num_selected(1638, 0.1) == 164
    assert so.num_selected(2016, 0.2) == 404
    assert so.num_selected(10, 0.3) == 3          # exact product stays 3
    assert so.num_selected(1000, 0.3) == 300
    assert so.num_selected(64, 1.0) == 64
    assert so.num_selected(64, 1e-6) == 1
    assert so.num_selected(64, 0.2, blocks=5) == 5
    assert so.num_selected(64, 0.2, blocks=500) == 64


# ------------------------------------------------------------------ moments

def test_second_moment_against_fsum():
    x = bf16(RNG.standard_normal((300, 5)))
    M = so.second_moment(x)
    for i in range(5):
        for j in range(5):
            ref = math.fsum(x[:, i] * x[:, j]) / 300
            assert abs(M[i, j] - ref) <= 1e-15 * max(1.0, abs(ref))
    assert np.allclose(M, M.T, atol=0, rtol=0)
    assert np.linalg.eigvalsh(M).min() > 0


def test_anchor_is_mean():
    q = bf16(RNG.standard_normal((128, 7)))
    ref = np.array([math.fsum(q[:, j]) / 128 for j in range(7)])
    assert np.allclose(so.anchor(q), ref, rtol=1e-15, atol=1e-15)


# ------------------------------------------------------------------ whitening

def test_whitening_inner_products_are_mahalanobis():
    x = bf16(RNG.standard_normal((400, 6)) @ RNG.standard_normal((6, 6)))
    M = so.second_moment(x)
    L = so.whitening_factor(M)
    Mt = M + so.REG_EPS * np.trace(M) / 6 * np.eye(6)
    assert np.allclose(L @ L.T, Mt, rtol=1e-13, atol=1e-13)
    assert np.allclose(np.triu(L, 1), 0)
    a, b = x[3], x[11]
    ua, ub = a @ L, b @ L
    assert abs(ua @ ub - a @ Mt @ b) < 1e-10 * (1 + abs(a @ Mt @ b))
    # normalised whitened vectors have unit length up to bf16 rounding
    U = so.normalized_whitened(x, L)
    n = np.sqrt((U * U).sum(axis=1))
    assert np.all(np.abs(n - 1) < 2 ** -7)


def test_whitening_zero_moment_is_identity():
    assert np.array_equal(so.whitening_factor(np.zeros((4, 4))), np.eye(4))
    U = so.normalized_whitened(np.zeros((3, 4)), np.eye(4))
    assert np.array_equal(U, np.zeros((3, 4)))


# ------------------------------------------------------------------ split direction

def test_split_direction_is_top_eigenvector():
    # well separated spectrum: 16 power steps converge far below 1e-8
    d = 8
    basis, _ = np.linalg.qr(RNG.standard_normal((d, d)))
    scales = np.array([3.0, 1.0, 0.8, 0.6, 0.5, 0.4, 0.3, 0.2])
    U = (RNG.standard_normal((512, d)) * scales) @ basis.T + RNG.standard_normal(d)
    v, mu, p = so.split_direction(U)
    C = U - U.mean(axis=0)
    w, E = np.linalg.eigh(C.T @ C / 512)
    top = E[:, -1]
    assert w[-2] / w[-1] < 0.5
    assert abs(abs(v @ top) - 1) < 1e-9
    assert np.allclose(mu, U.mean(axis=0))
    assert np.allclose(p, C @ v)


def test_split_direction_2x2_closed_form():
    # covariance [[a, b], [b, c]]: principal axis angle = atan2(2b, a - c) / 2
    pts = RNG.standard_normal((1024, 2)) @ np.array([[2.0, 0.0], [0.9, 0.5]])
    v, _, _ = so.split_direction(pts)
    C = pts - pts.mean(axis=0)
    S = C.T @ C / 1024
    a, b, c = S[0, 0], S[0, 1], S[1, 1]
    th = 0.5 * math.atan2(2 * b, a - c)
    e = np.array([math.cos(th), math.sin(th)])
    w = np.linalg.eigvalsh(S)
    assert (w[0] / w[1]) ** 16 < 1e-6
    assert abs(abs(v @ e) - 1) < 1e-9


def test_split_projection_independent_of_whitening_factor():
    # Mahalanobis geometry: any A with A^T A = M gives the same projections
    # (up to sign) once the power iteration has converged. The tokens are
    # built in whitened space with one dominant axis of spread.
    d = 5
    M = so.second_moment(RNG.standard_normal((900, d)) @ RNG.standard_normal((d, d)))
    L = np.linalg.cholesky(M)
    w, E = np.linalg.eigh(M)
    Msqrt = E @ np.diag(np.sqrt(w)) @ E.T
    u = np.zeros((640, d))
    u[:, 0] = 1.0
    u[:, 1] = 0.4 * RNG.standard_normal(640)
    u[:, 2:] = 0.02 * RNG.standard_normal((640, d - 2))
    x = u @ np.linalg.inv(L)                 # so that x @ L == u

    def normed(U):
        return U / np.sqrt((U * U).sum(axis=1))[:, None]

    _, _, p1 = so.split_direction(normed(x @ L))
    _, _, p2 = so.split_direction(normed(x @ Msqrt))
    C = normed(x @ L)
    C = C - C.mean(axis=0)
    ev = np.linalg.eigvalsh(C.T @ C)
    assert (ev[-2] / ev[-1]) ** 16 < 1e-7
    s = np.sign(p1 @ p2)
    assert np.allclose(p1, s * p2, atol=1e-7)
    # a transposed factor (x @ L.T) is not a whitening of M and moves p
    _, _, p3 = so.split_direction(normed(x @ L.T))
    assert not np.allclose(np.abs(p1), np.abs(p3), atol=1e-3)


def test_split_group_orientation_and_capacity():
    U = bf16(RNG.standard_normal((64 * 5, 6)))
    ids = RNG.permutation(10_000)[: 64 * 5]
    left, right, info = so.split_group(U, ids)
    assert len(left) == 128 and len(right) == 192            # floor(5/2) blocks left
    assert set(left) | set(right) == set(ids)
    p = info["p"]
    a = np.abs(p)
    top = ids[a == a.max()].min()
    assert p[ids == top][0] > 0                              # orientation
    pl = p[np.isin(ids, left)]
    pr = p[np.isin(ids, right)]
    assert pl.max() <= pr.min()                              # sorted split


def test_split_group_all_identical_uses_index_order():
    U = np.tile(bf16(RNG.standard_normal(6)), (128, 1))
    ids = RNG.permutation(1000)[:128]
    left, right, info = so.split_group(U, ids)
    assert np.all(info["p"] == 0)
    assert set(left) == set(np.sort(ids)[:64])


# ------------------------------------------------------------------ reblock

@pytest.mark.parametrize("nb", [1, 2, 3, 5, 8, 13])
def test_tree_shape_depends_on_nb_only(nb):
    levels = so.tree_nodes(nb)
    assert len(levels) == (math.ceil(math.log2(nb)) if nb > 1 else 0)
    for lv in levels:
        for f, g in lv:
            assert g >= 2 and 0 <= f and f + g <= nb


@pytest.mark.parametrize("nb,d", [(1, 8), (2, 8), (3, 16), (7, 8), (16, 32)])
def test_reblock_leaves_and_bijection(nb, d):
    q, k, _ = rand_qkv(64 * nb, d, seed=nb)
    perm = so.reblock(q, so.second_moment(k))
    N = 64 * nb
    assert sorted(perm.tolist()) == list(range(N))            # bijection
    for b in range(nb):
        blk = perm[64 * b:64 * b + 64]
        assert np.all(np.diff(blk) > 0)                       # ascending inside a leaf


def test_reblock_relabel_equivariance():
    N, d = 64 * 6, 8
    q, k, _ = rand_qkv(N, d, seed=7)
    MK = so.second_moment(k)
    perm = so.reblock(q, MK)
    sigma = RNG.permutation(N)                 # new token i is old token sigma[i]
    perm2 = so.reblock(q[sigma], MK)
    blocks = [set(perm[64 * b:64 * b + 64]) for b in range(6)]
    blocks2 = [set(sigma[perm2[64 * b:64 * b + 64]]) for b in range(6)]
    assert blocks == blocks2


def test_reblock_groups_similar_queries():
    # two well separated query clusters of 128 tokens each end up in
    # different halves of the first split
    d = 8
    r = np.random.default_rng(3)
    c1, c2 = r.standard_normal(d), r.standard_normal(d)
    q = np.concatenate([c1 + 0.05 * r.standard_normal((128, d)),
                        c2 + 0.05 * r.standard_normal((128, d))])
    sigma = r.permutation(256)
    q = bf16(q[sigma])
    M = np.eye(d)
    perm = so.reblock(q, M)
    cluster = (sigma >= 128).astype(int)
    first = cluster[perm[:128]]
    assert first.min() == first.max()


def test_positional_tiles():
    grid = (4, 16, 64)
    perm = so.positional_tiles(grid)
    assert sorted(perm.tolist()) == list(range(4096))
    F, Hl, Wl = grid
    for b in range(64):
        t = perm[64 * b:64 * b + 64]
        f, y, x = t // (Hl * Wl), (t // Wl) % Hl, t % Wl
        assert f.max() - f.min() == 1 and y.max() - y.min() == 7 and x.max() - x.min() == 3


# ------------------------------------------------------------------ selection

def test_select_against_full_sort():
    qm = RNG.standard_normal((20, 4))
    km = RNG.standard_normal((20, 4))
    s = so.block_scores(qm, km)
    sel = so.select(qm, km, 6)
    for a in range(20):
        order = sorted(range(20), key=lambda b: (-s[a, b], b))
        assert sel[a].tolist() == sorted(order[:6])


def test_select_ties_go_to_lower_index():
    qm = np.ones((3, 2))
    km = np.array([[1, 0], [0, 1], [1, 0], [0, 1], [0.5, 0.5], [2, 2]], dtype=float)
    # scores per row: [1, 1, 1, 1, 1, 4] / sqrt(2): block 5 first, then ties by index
    sel = so.select(qm, km, 3)
    assert sel.tolist() == [[0, 1, 5]] * 3


def test_block_scores_scale():
    qm = np.array([[2.0, 0.0]])
    km = np.array([[3.0, 1.0]])
    assert so.block_scores(qm, km)[0, 0] == pytest.approx(6.0 / math.sqrt(2))


# ------------------------------------------------------------------ summaries

def test_beta_is_entropy_of_anchor_weights():
    N, d = 64 * 4, 16
    q, k, v = rand_qkv(N, d, seed=11, scale=2.0)
    perm = np.arange(N)
    qbar = so.anchor(q)
    kt, vt, beta = so.summaries(k, v, perm, qbar)
    for b in range(4):
        x = k[64 * b:64 * b + 64] @ qbar / math.sqrt(d)
        w = np.exp(x - x.max())
        w /= w.sum()
        H = -(w * np.log(w)).sum()
        assert beta[b] == pytest.approx(H, abs=1e-12)
        assert 0 <= beta[b] <= math.log(64) + 1e-12
        assert np.allclose(kt[b], w @ k[64 * b:64 * b + 64])
        assert np.allclose(vt[b], w @ v[64 * b:64 * b + 64])


def test_beta_identical_keys_is_log64():
    d = 8
    kb = np.tile(RNG.standard_normal(d), (64, 1))
    v = RNG.standard_normal((64, d))
    kt, vt, beta = so.summaries(kb, v, np.arange(64), RNG.standard_normal(d))
    assert beta[0] == pytest.approx(math.log(64), abs=1e-12)
    assert np.allclose(kt[0], kb[0])
    assert np.allclose(vt[0], v.mean(axis=0))


def test_meanpool_equals_reweight_for_zero_anchor():
    k = RNG.standard_normal((128, 8))
    v = RNG.standard_normal((128, 8))
    perm = RNG.permutation(128)
    a = so.summaries(k, v, perm, np.zeros(8), "reweight")
    b = so.summaries(k, v, perm, np.zeros(8), "meanpool")
    for x, y in zip(a, b):
        assert np.allclose(x, y, atol=1e-14)


def test_pooled_logit_matches_mean_exp_for_anchor():
    # [P1] figure caption: exp of the biased pooled logit equals E[exp x]
    d = 16
    k = RNG.standard_normal((64, d))
    qbar = RNG.standard_normal(d)
    kt, _, beta = so.summaries(k, np.zeros((64, d)), np.arange(64), qbar)
    x = k @ qbar / math.sqrt(d)
    pooled = qbar @ kt[0] / math.sqrt(d) + beta[0] - math.log(64)
    assert math.exp(pooled) == pytest.approx(np.exp(x).mean(), rel=1e-12)
    # mean pooling undershoots (Jensen): exp(E[x]) <= E[exp x]
    assert math.exp(x.mean()) <= np.exp(x).mean()


# ------------------------------------------------------------------ attention

def _run(q, k, v, ratio, perm=None, summary="reweight"):
    if perm is None:
        return so.forward_head(q, k, v, ratio=ratio, summary=summary)
    return so.forward_head(q, k, v, ratio=ratio, layout="given", perm=perm, summary=summary)


def test_density_one_is_dense_attention():
    q, k, v = rand_qkv(64 * 5, 16, seed=21, scale=1.5)
    ref, ref_lse = so.dense_attention(q, k, v)
    for perm in (None, np.arange(320), RNG.permutation(320)):
        r = _run(q, k, v, 1.0, perm)
        assert r["ksel"] == 5
        assert np.allclose(r["out"], ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(r["lse"], ref_lse, rtol=1e-12, atol=1e-12)


def test_dense_attention_matches_textbook_softmax():
    q, k, v = rand_qkv(70, 8, seed=5)
    out, lse = so.dense_attention(q, k, v)
    for i in (0, 33, 69):
        s = [math.fsum(q[i] * k[j]) / math.sqrt(8) for j in range(70)]
        w = [math.exp(x) for x in s]
        Z = math.fsum(w)
        for c in range(8):
            assert out[i, c] == pytest.approx(math.fsum(w[j] * v[j, c] for j in range(70)) / Z, abs=1e-13)
        assert lse[i] == pytest.approx(math.log(Z), abs=1e-13)


def test_constant_v_gives_constant_output():
    q, k, _ = rand_qkv(64 * 6, 8, seed=3)
    v = np.full((384, 8), 0.375)
    r = _run(q, k, v, 0.3)
    assert np.allclose(r["out"], 0.375, atol=1e-13)


def test_compressed_branch_exact_for_identical_keys():
    # all 64 keys of each block identical: e^{q.k + ln 64} * mean v equals the
    # exact sum, so any density reproduces dense attention
    nb, d = 6, 8
    r = np.random.default_rng(9)
    kb = np.repeat(r.standard_normal((nb, d)), 64, axis=0)
    q = r.standard_normal((64 * nb, d))
    v = r.standard_normal((64 * nb, d))
    perm = np.arange(64 * nb)
    ref, _ = so.dense_attention(q, kb, v)
    for summary in ("reweight", "meanpool"):
        res = _run(q, kb, v, 0.2, perm, summary)
        assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-12)


def test_compressed_branch_exact_for_anchor_query():
    # a query equal to the per-head mean query sees the exact block masses
    nb, d = 5, 8
    r = np.random.default_rng(4)
    c = r.standard_normal(d)
    half = r.standard_normal((64 * nb // 2, d))
    q = np.concatenate([c + half, c - half])        # mean of q is exactly c
    q[0] = c + 0.0
    q[64 * nb // 2] = c + 0.0                       # keep the mean at c
    k = r.standard_normal((64 * nb, d))
    v = r.standard_normal((64 * nb, d))
    perm = np.arange(64 * nb)
    assert np.allclose(q.mean(axis=0), c)
    ref, _ = so.dense_attention(q, k, v)
    res = _run(q, k, v, 0.2, perm)
    assert np.allclose(res["out"][0], ref[0], rtol=1e-11, atol=1e-12)
    # mean pooling is not exact for that query
    res_mp = _run(q, k, v, 0.2, perm, "meanpool")
    assert not np.allclose(res_mp["out"][0], ref[0], rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("N,d,ratio,summary", [
    (128, 2, 0.5, "reweight"), (256, 8, 0.25, "reweight"), (256, 64, 0.5, "reweight"),
    (256, 8, 0.25, "meanpool"), (192, 8, 0.34, "reweight")])
def test_oracle_matches_brute_force(N, d, ratio, summary):
    q, k, v = rand_qkv(N, d, seed=N + d, scale=1.3)
    res = so.forward_head(q, k, v, ratio=ratio, summary=summary)
    bf = brute_force.forward(q, k, v, res["perm"], res["ksel"], summary)
    nb = N // 64
    chosen = np.zeros((nb, nb), dtype=bool)
    for a in range(nb):
        chosen[a, res["sel"][a]] = True
    assert np.array_equal(chosen, bf["chosen"])
    assert np.allclose(res["kt"], bf["kt"], rtol=1e-12, atol=1e-12)
    assert np.allclose(res["vt"], bf["vt"], rtol=1e-12, atol=1e-12)
    assert np.allclose(res["beta"], bf["beta"], rtol=1e-12, atol=1e-12)
    assert np.allclose(res["out"], bf["out"], rtol=1e-12, atol=1e-12)
    assert np.allclose(res["lse"], bf["lse"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("N,d,ratio,summary", [(128, 8, 0.5, "reweight"), (256, 8, 0.25, "reweight"),
                                               (256, 4, 0.5, "meanpool")])
def test_block_tail_matches_brute_force(N, d, ratio, summary):
    """Tail granularity "block" (compressed logits from the block's mean
    query) against the loop-free brute-force statement."""
    q, k, v = rand_qkv(N, d, seed=3 * N + d, scale=1.3)
    res = so.forward_head(q, k, v, ratio=ratio, summary=summary, tail="block")
    bf = brute_force.forward(q, k, v, res["perm"], res["ksel"], summary, tail="block")
    assert np.allclose(res["out"], bf["out"], rtol=1e-12, atol=1e-12)
    assert np.allclose(res["lse"], bf["lse"], rtol=1e-12, atol=1e-12)
    ref = so.forward_head(q, k, v, ratio=ratio, summary=summary, tail="query")
    assert not np.allclose(res["out"], ref["out"], rtol=1e-6, atol=1e-6)   # the two tails differ


def test_block_tail_equals_query_tail_for_uniform_blocks():
    """When every query of a permuted block equals the block's mean query,
    the two tail granularities are the same computation."""
    r = np.random.default_rng(11)
    N, d = 256, 8
    base = bf16(r.standard_normal((N // 64, d)))
    q = np.repeat(base, 64, axis=0)                    # identical queries per positional block
    k = bf16(r.standard_normal((N, d)))
    v = bf16(r.standard_normal((N, d)))
    perm = np.arange(N)
    a = so.forward_head(q, k, v, ratio=0.25, layout="given", perm=perm, tail="block")
    b = so.forward_head(q, k, v, ratio=0.25, layout="given", perm=perm, tail="query")
    assert np.allclose(a["out"], b["out"], rtol=1e-13, atol=1e-13)
    assert np.allclose(a["lse"], b["lse"], rtol=1e-13, atol=1e-13)


def test_block_tail_density_one_is_dense():
    """At density 1.0 there are no compressed terms: both tails are dense."""
    q, k, v = rand_qkv(256, 8, seed=5)
    res = so.forward_head(q, k, v, ratio=1.0, tail="block")
    ref, _ = so.dense_attention(q, k, v)
    assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("N,d,ratio,summary", [(128, 8, 0.5, "reweight"), (256, 8, 0.25, "reweight"),
                                               (256, 4, 0.5, "meanpool")])
def test_separate_layout_matches_brute_force(N, d, ratio, summary):
    """Layout "separate" (queries grouped under M_K, keys under M_Q, each on
    its own) against the brute force given both permutations."""
    q, k, v = rand_qkv(N, d, seed=7 * N + d, scale=1.3)
    res = so.forward_head(q, k, v, ratio=ratio, summary=summary, layout="separate")
    assert not np.array_equal(res["perm"], res["perm_k"])      # the two partitions differ here
    bf = brute_force.forward(q, k, v, res["perm"], res["ksel"], summary, perm_k=res["perm_k"])
    nb = N // 64
    chosen = np.zeros((nb, nb), dtype=bool)
    for a in range(nb):
        chosen[a, res["sel"][a]] = True
    assert np.array_equal(chosen, bf["chosen"])
    assert np.allclose(res["kt"], bf["kt"], rtol=1e-12, atol=1e-12)
    assert np.allclose(res["out"], bf["out"], rtol=1e-12, atol=1e-12)
    assert np.allclose(res["lse"], bf["lse"], rtol=1e-12, atol=1e-12)


def test_separate_layout_is_shared_layout_when_q_equals_k():
    """With k = q the two moments coincide, so both partitions coincide and
    the separate layout is the shared one."""
    q, _, v = rand_qkv(256, 8, seed=9)
    a = so.forward_head(q, q, v, ratio=0.25, layout="separate")
    b = so.forward_head(q, q, v, ratio=0.25, layout="q_reuse_k")
    assert np.array_equal(a["perm"], a["perm_k"]) and np.array_equal(a["perm"], b["perm"])
    assert np.array_equal(a["out"], b["out"])


def test_separate_layout_density_one_is_dense():
    q, k, v = rand_qkv(256, 8, seed=13)
    res = so.forward_head(q, k, v, ratio=1.0, layout="separate")
    ref, _ = so.dense_attention(q, k, v)
    assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-12)


def _context(C, d, seed, scale=1.3):
    r = np.random.default_rng(seed)
    return (bf16(r.standard_normal((C, d)) * scale), bf16(r.standard_normal((C, d)) * scale),
            bf16(r.standard_normal((C, d))))


@pytest.mark.parametrize("N,d,ratio,C", [(128, 8, 0.5, 7), (256, 8, 0.25, 64), (256, 4, 0.5, 100)])
def test_joint_attention_matches_brute_force(N, d, ratio, C):
    """Joint attention (dense context segment) against the brute force."""
    q, k, v = rand_qkv(N, d, seed=11 * N + C, scale=1.3)
    qc, kc, vc = _context(C, d, seed=C)
    res = so.forward_head(q, k, v, ratio=ratio)
    out, lse, outc, lsec = so.joint_attention(q, k, v, res["perm"], res["sel"], res["kt"], res["vt"],
                                              res["beta"], qc, kc, vc)
    bf = brute_force.forward(q, k, v, res["perm"], res["ksel"], context=(qc, kc, vc))
    assert np.allclose(out, bf["out"], rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, bf["lse"], rtol=1e-12, atol=1e-12)
    assert np.allclose(outc, bf["outc"], rtol=1e-12, atol=1e-12)
    assert np.allclose(lsec, bf["lsec"], rtol=1e-12, atol=1e-12)


def test_joint_attention_density_one_is_dense_joint():
    """At density 1.0 the whole thing is dense attention over both segments,
    for video and context queries alike."""
    q, k, v = rand_qkv(256, 8, seed=21)
    qc, kc, vc = _context(40, 8, seed=22)
    res = so.forward_head(q, k, v, ratio=1.0)
    out, _, outc, _ = so.joint_attention(q, k, v, res["perm"], res["sel"], res["kt"], res["vt"], res["beta"],
                                         qc, kc, vc)
    K, V = np.concatenate([k, kc]), np.concatenate([v, vc])
    ref, _ = so.dense_attention(q, K, V)
    refc, _ = so.dense_attention(qc, K, V)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(outc, refc, rtol=1e-12, atol=1e-12)


def test_joint_attention_lse_merge():
    """A video row's joint lse is the log-sum-exp merge of its video-only lse
    and its lse over the context keys alone."""
    q, k, v = rand_qkv(256, 8, seed=31)
    qc, kc, vc = _context(33, 8, seed=32)
    res = so.forward_head(q, k, v, ratio=0.25)
    out, lse, _, _ = so.joint_attention(q, k, v, res["perm"], res["sel"], res["kt"], res["vt"], res["beta"],
                                        qc, kc, vc)
    _, lse_ctx = so.dense_attention(q, kc, vc)
    merged = np.logaddexp(res["lse"], lse_ctx)
    assert np.allclose(lse, merged, rtol=1e-12, atol=1e-12)
    # and the output is the matching convex combination of the two partial outputs
    o_ctx, _ = so.dense_attention(q, kc, vc)
    w = np.exp(res["lse"] - lse)[:, None]
    assert np.allclose(out, w * res["out"] + (1 - w) * o_ctx, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("iters", [1, 4, 16])
def test_split_direction_is_normalised_matrix_power(iters):
    """With T power steps the direction is S^T 1 / |S^T 1| (one matrix power,
    no per-step rescaling), for the Lite count as for the default."""
    r = np.random.default_rng(77)
    U = bf16(r.standard_normal((256, 12)))
    v, mu, p = so.split_direction(U, iters)
    C = U - U.mean(axis=0)
    S = C.T @ C / len(U)
    w = np.linalg.matrix_power(S, iters) @ np.ones(12)
    assert np.allclose(v, w / np.linalg.norm(w), rtol=1e-10, atol=1e-12)
    assert np.allclose(p, C @ v, rtol=1e-12, atol=1e-12)


def test_lite_split_equals_full_split_for_rank_one_groups():
    """A group whose centred vectors share one direction: one power step
    already finds it, so 4 and 16 steps give the same partition."""
    r = np.random.default_rng(78)
    d = 16
    u = r.standard_normal(d)
    x = np.outer(r.standard_normal(512), u) + 1e-3      # rank one after centring
    M = np.eye(d)
    assert np.array_equal(so.reblock(x, M, 4), so.reblock(x, M, 16))


# ------------------------------------------------------------------ statistics

def test_mass_recall_is_100_at_density_one():
    q, k, v = rand_qkv(256, 8, seed=2)
    r = _run(q, k, v, 1.0)
    assert so.mass_recall(q, k, r["perm"], r["sel"], range(4)) == pytest.approx(100.0)


def test_mass_recall_brute_force():
    q, k, v = rand_qkv(256, 8, seed=12, scale=2)
    r = _run(q, k, v, 0.25)
    s = q @ k.T / math.sqrt(8)
    P = np.exp(s - s.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    blk = np.empty(256, dtype=int)
    blk[r["perm"]] = np.arange(256) // 64
    rec = [100 * P[i, np.isin(blk, r["sel"][blk[i]])].sum() for i in range(256)]
    assert so.mass_recall(q, k, r["perm"], r["sel"], range(4)) == pytest.approx(np.mean(rec))


def test_log_mass_error_zero_for_identical_keys():
    nb, d = 4, 8
    r = np.random.default_rng(1)
    kb = np.repeat(r.standard_normal((nb, d)), 64, axis=0)
    q = r.standard_normal((64 * nb, d))
    res = _run(q, kb, r.standard_normal((64 * nb, d)), 0.25, np.arange(64 * nb))
    e = so.log_mass_error(q, kb, res["perm"], res["sel"], res["kt"], res["beta"], range(nb))
    assert e < 1e-12


def test_log_mass_error_brute_force():
    """Every (query, unselected block) pair spelled out with math.fsum over
    the 64 exponentials and math.log, then the plain mean of the absolute
    differences ([P2] "absolute log-mass error")."""
    q, k, v = rand_qkv(256, 8, seed=31, scale=2)
    r = _run(q, k, v, 0.25)
    perm, sel, kt, beta = r["perm"], r["sel"], r["kt"], r["beta"]
    rows = [0, 2, 3]
    errs = []
    for a in rows:
        for i in perm[64 * a:64 * (a + 1)]:
            for b in range(4):
                if b in set(sel[a].tolist()):
                    continue
                keys = perm[64 * b:64 * (b + 1)]
                true = math.log(math.fsum(math.exp(float(q[i] @ k[j]) / math.sqrt(8)) for j in keys))
                pooled = float(q[i] @ kt[b]) / math.sqrt(8) + float(beta[b])
                errs.append(abs(pooled - true))
    assert len(errs) == 3 * 64 * 3
    assert so.log_mass_error(q, k, perm, sel, kt, beta, rows) == pytest.approx(math.fsum(errs) / len(errs),
                                                                              rel=1e-12)


def test_statistics_take_the_key_permutation():
    """Separate layout (R16): key block b is block b of the key permutation,
    for both statistics."""
    q, k, v = rand_qkv(256, 8, seed=32, scale=2)
    r = so.forward_head(q, k, v, ratio=0.25, layout="separate")
    pq, pk = r["perm"], r["perm_k"]
    assert not np.array_equal(pq, pk)
    rows = [0, 1]
    s = q @ k.T / math.sqrt(8)
    P = np.exp(s - s.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    kblk = np.empty(256, dtype=int)
    kblk[pk] = np.arange(256) // 64
    rec = [100 * P[i, np.isin(kblk, r["sel"][a])].sum() for a in rows for i in pq[64 * a:64 * (a + 1)]]
    assert so.mass_recall(q, k, pq, r["sel"], rows, perm_k=pk) == pytest.approx(np.mean(rec), rel=1e-12)
    errs = []
    for a in rows:
        for i in pq[64 * a:64 * (a + 1)]:
            for b in sorted(set(range(4)) - set(r["sel"][a].tolist())):
                true = math.log(math.fsum(math.exp(float(q[i] @ k[j]) / math.sqrt(8)) for j in pk[64 * b:64 * (b + 1)]))
                errs.append(abs(float(q[i] @ r["kt"][b]) / math.sqrt(8) + float(r["beta"][b]) - true))
    got = so.log_mass_error(q, k, pq, r["sel"], r["kt"], r["beta"], rows, perm_k=pk)
    assert got == pytest.approx(math.fsum(errs) / len(errs), rel=1e-12)


@pytest.mark.parametrize("summary", ["reweight", "meanpool"])
def test_report_stats_helper_matches_oracle(summary):
    """The statistics helper of bench.py's stats report (float64 torch ops,
    run here on the CPU) equals the oracle's mass recall and log-mass error
    on the oracle's own permutation, selection and summaries."""
    import torch
    import bench
    w = WORKLOADS["tiny_4096"]
    q, k, v = (bf16_bits_to_f64(x[0, 0]) for x in make_inputs(w, heads=[0]))
    r = so.forward_head(q, k, v, ratio=0.2, summary=summary)
    nb = q.shape[0] // 64
    blocks = np.array([1, 9, 30, nb - 1])
    rec = so.mass_recall(q, k, r["perm"], r["sel"], blocks)
    lme = so.log_mass_error(q, k, r["perm"], r["sel"], r["kt"], r["beta"], blocks)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    rs, nr, es, ne = bench.head_block_stats(t(q), t(k), t(r["perm"]), t(r["sel"]), t(r["kt"]), t(r["beta"]),
                                            t(blocks), chunk=3)
    assert 100.0 * rs / nr == pytest.approx(rec, rel=1e-10)
    assert es / ne == pytest.approx(lme, rel=1e-10)


def test_oracle_matches_brute_force_random_sweep():
    """Seeded sweep over shapes, densities, summaries, tail granularities and
    layouts: the step-by-step oracle and the loop-free brute-force restatement
    agree to 1e-12 on selection, summaries, outputs and lse."""
    rng = np.random.default_rng(20261202)
    for case in range(24):
        N = int(rng.choice([128, 192, 256, 320]))
        d = int(rng.choice([2, 4, 8, 16]))
        ratio = float(rng.uniform(0.1, 0.9))
        summary = str(rng.choice(["reweight", "meanpool"]))
        tail = str(rng.choice(["query", "block"]))
        layout = str(rng.choice(["q_reuse_k", "k_reuse_q", "separate"]))
        q, k, v = rand_qkv(N, d, seed=1000 + case, scale=float(rng.uniform(0.5, 2.0)))
        res = so.forward_head(q, k, v, ratio=ratio, summary=summary, tail=tail, layout=layout)
        bf = brute_force.forward(q, k, v, res["perm"], res["ksel"], summary, tail=tail,
                                 perm_k=res.get("perm_k") if layout == "separate" else None)
        nb = N // 64
        chosen = np.zeros((nb, nb), dtype=bool)
        for a in range(nb):
            chosen[a, res["sel"][a]] = True
        tag = (case, N, d, round(ratio, 3), summary, tail, layout)
        assert np.array_equal(chosen, bf["chosen"]), tag
        for key in ("kt", "vt", "beta", "out", "lse"):
            assert np.allclose(res[key], bf[key], rtol=1e-12, atol=1e-12), (key, tag)
