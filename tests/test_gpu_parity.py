"""CUDA path against the CPU oracle on seeded inputs (needs a B200).

Every call goes through the C ABI (ctypes binding). Layered comparison: see
tests/parity.py."""

import math

import numpy as np
import pytest

import block_sparse_attention_spark_b200 as spark
from oracle import spark_oracle as so
from spark_gen import WORKLOADS, bf16_bits_to_f64, host_procs, make_inputs, tiny_workload
from tests import parity

pytestmark = pytest.mark.gpu

# moments: float64 sums of exact products on both sides (summation order only)
MOMENT_TOL = 1e-13


def to_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_to_f64(t):
    import torch
    return bf16_bits_to_f64(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def run_stages(w, ratio=None, layout="q_reuse_k", summary="reweight", topk_blocks=0, qkv=None,
               perm=None, tail="query", power_iters=0):
    import torch
    q, k, v = qkv if qkv is not None else make_inputs(w)
    B, H, N, d = q.shape
    p = spark.params(B, H, N, d, ratio if ratio is not None else w.ratio, topk_blocks, layout, summary, tail,
                     power_iters)
    ws = spark.alloc_workspace(p)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    MQ, MK, qmean = spark.moments(p, qd, kd, ws)
    gperm = spark.reblock(p, qd, kd, MQ, MK, ws) if perm is None else perm
    uhat = spark.ws_view(ws, p, "UHAT", torch.bfloat16, (B, H, N, d)).clone() if perm is None else None
    sel = spark.select(p, qd, kd, vd, gperm, qmean, ws)
    out, lse = spark.attn_fwd(p, gperm, sel, ws, return_lse=True)
    nbp = spark.workspace_region(p, "BETA")[1] // (4 * B * H)
    res = dict(p=p, q=q, k=k, v=v, MQ=MQ.cpu().numpy(), MK=MK.cpu().numpy(), qmean=qmean.cpu().numpy(),
               perm=gperm.cpu().numpy(), sel=sel.cpu().numpy(), out=bf16_to_f64(out),
               lse=lse.cpu().numpy().astype(np.float64),
               kt=bf16_to_f64(spark.ws_view(ws, p, "KT", torch.bfloat16, (B, H, nbp, d))),
               vt=bf16_to_f64(spark.ws_view(ws, p, "VT", torch.bfloat16, (B, H, nbp, d))),
               beta=spark.ws_view(ws, p, "BETA", torch.float32, (B, H, nbp)).cpu().numpy().astype(np.float64),
               qm=spark.ws_view(ws, p, "QM", torch.float64, (B, H, N // 64, d)).cpu().numpy(),
               km=spark.ws_view(ws, p, "KM", torch.float64, (B, H, N // 64, d)).cpu().numpy(),
               uhat=None if uhat is None else bf16_to_f64(uhat))
    assert spark.get_status() == 0
    return res


def check_beta(gk, gb, kt, beta, qbar, summary):
    """The log-mass bias. Reweight ("Spark-H3" news post, Spark-Reweight
    figure: the exp of the biased pooled logit is the block's E[exp x] at the
    anchor) makes qbar . k~_b / sqrt(d) + beta_b = ln sum_{j in b} exp(x_j).
    The GPU keeps that identity for the bf16 k~ it stores (and attention
    reads), so its beta differs from the oracle's, formed with the unrounded
    k~, by qbar . (rounding of k~) / sqrt(d); the identity itself is compared.
    Mean pooling: beta = ln 64."""
    d = gk.shape[1]
    if summary == "meanpool":
        assert np.abs(gb - beta).max() <= 1e-6
        return
    lnz_ref = kt @ qbar / math.sqrt(d) + beta
    lnz_gpu = gk @ qbar / math.sqrt(d) + gb
    assert np.abs(lnz_gpu - lnz_ref).max() <= 1e-4 * (1 + np.abs(lnz_ref).max())


def check_head(r, b, h, layout="q_reuse_k", summary="reweight", rows=None, check_perm=True,
               report=None, tail="query", power_iters=so.POWER_ITERS):
    q = bf16_bits_to_f64(r["q"][b, h])
    k = bf16_bits_to_f64(r["k"][b, h])
    v = bf16_bits_to_f64(r["v"][b, h])
    N, d = q.shape
    nb = N // 64
    p = r["p"]
    # a1 moments: float64 sums of exact products on both sides; only the
    # summation order differs
    MQ, MK, qbar = so.second_moment(q), so.second_moment(k), so.anchor(q)
    assert np.abs(r["MQ"][b, h] - MQ).max() <= MOMENT_TOL * np.abs(MQ).max()
    assert np.abs(r["MK"][b, h] - MK).max() <= MOMENT_TOL * np.abs(MK).max()
    assert np.abs(r["qmean"][b, h] - qbar).max() <= 1e-12 * (1 + np.abs(qbar).max())
    if layout == "separate":
        # query permutation (queries under M_K) and key permutation (keys under M_Q)
        perm, perm_k = r["perm"][0, b, h].astype(np.int64), r["perm"][1, b, h].astype(np.int64)
        if check_perm:
            # the workspace's u_hat is the key side's (the second reblock); the
            # query side is replayed with the oracle's own u_hat
            st = parity.certify_perm(q, MK, perm, iters=power_iters)
            print("perm q", b, h, st)
            assert st["failures"] == 0, st
        xs, Ms = k, MQ
        perm_side = perm_k
    else:
        perm = r["perm"][b, h].astype(np.int64)
        perm_k = perm
        xs, Ms = (q, MK) if layout == "q_reuse_k" else (k, MQ)
        perm_side = perm
    if check_perm:
        # normalised whitened tokens: both sides evaluate them in float64 and
        # round once to bf16, so they are equal element for element
        U = so.normalized_whitened(xs, so.whitening_factor(Ms))
        flips = int((r["uhat"][b, h] != U).sum())
        assert flips == 0, f"u_hat differs from the oracle's in {flips} elements"
        # every split replayed by the oracle on its own u_hat
        st = parity.certify_perm(xs, Ms, perm_side, iters=power_iters)
        print("perm", b, h, st)
        assert st["failures"] == 0, st
        if report is not None:
            report.append(("perm", b, h, st["nodes"], st["mismatched"], st["certified"], st["worst"]))
    else:
        parity.check_perm_structure(perm, N)
        parity.check_perm_structure(perm_k, N)
    # a3 block means (exact sums) and summaries, given the CUDA permutation
    qm, km = so.block_means(q, perm), so.block_means(k, perm_k)
    assert np.abs(r["qm"][b, h] - qm).max() <= 1e-14 * (1 + np.abs(qm).max())
    assert np.abs(r["km"][b, h] - km).max() <= 1e-14 * (1 + np.abs(km).max())
    kt, vt, beta = so.summaries(k, v, perm_k, qbar, summary)
    gk, gv, gb = r["kt"][b, h, :nb], r["vt"][b, h, :nb], r["beta"][b, h, :nb]
    assert np.all(np.abs(gk - kt) <= 2 ** -8 * np.abs(kt) + 1e-6 * np.abs(kt).max())
    assert np.all(np.abs(gv - vt) <= 2 ** -8 * np.abs(vt) + 1e-6 * np.abs(vt).max())
    check_beta(gk, gb, kt, beta, qbar, summary)
    assert np.all(r["kt"][b, h, nb:] == 0) and np.all(r["beta"][b, h, nb:] == 0)
    # a4 selection, given the CUDA permutation
    ksel = spark.num_selected(p)
    sel = r["sel"][b, h].astype(np.int64)
    st = parity.certify_select(qm, km, ksel, sel)
    assert st["failures"] == 0, st
    if report is not None:
        report.append(("sel", b, h, st["rows"], st["mismatched"], st["certified"]))
    # a5-a7 outputs, given the CUDA permutation and selection
    ref, ref_lse = so.attention(q, k, v, perm, sel, kt, vt, beta, rows=rows, tail=tail, qm=qm, perm_k=perm_k)
    mask = ~np.isnan(ref[:, 0])
    e = parity.out_errors(r["out"][b, h][mask], ref[mask])
    assert e["max_rel_to_bound"] <= 1.0, e
    # derived bound: bf16 output rounding plus bf16 P and summaries
    assert e["max_abs"] <= 2 ** -7 * np.abs(ref[mask]).max() + 4e-3 * e["ref_rms"], e
    assert np.abs(r["lse"][b, h][mask] - ref_lse[mask]).max() <= 1e-3 * (1 + np.abs(ref_lse[mask]).max())
    return e


def test_tiny_workload_all_stages():
    w = WORKLOADS["tiny_4096"]
    r = run_stages(w)
    rep = []
    for h in range(w.H):
        check_head(r, 0, h, report=rep)
    print(rep)


def test_mid_workload_all_stages():
    w = WORKLOADS["mid_16128"]
    r = run_stages(w)
    rep = []
    for h in range(w.H):
        check_head(r, 0, h, report=rep)
    print(rep)


@pytest.mark.parametrize("nb,d", [(2, 64), (3, 128), (5, 64), (7, 128), (13, 64), (33, 128)])
def test_ragged_trees(nb, d):
    w = tiny_workload(f"ragged{nb}", 2, (2, 8, 4 * nb), d, 0.3, seed_index=200 + nb)
    r = run_stages(w)
    for h in range(w.H):
        check_head(r, 0, h)


def test_density_one_is_dense_attention():
    w = tiny_workload("dense", 2, (2, 16, 32), 128, 1.0, seed_index=300)
    r = run_stages(w)
    for h in range(2):
        q, k, v = (bf16_bits_to_f64(r[t][0, h]) for t in ("q", "k", "v"))
        ref, lse = so.dense_attention(q, k, v)
        e = parity.out_errors(r["out"][0, h], ref)
        assert e["max_rel_to_bound"] <= 1.0
        assert e["max_abs"] <= 2 ** -7 * np.abs(ref).max() + 4e-3 * e["ref_rms"], e
        assert np.abs(r["lse"][0, h] - lse).max() <= 1e-3 * (1 + np.abs(lse).max())


@pytest.mark.parametrize("summary", ["reweight", "meanpool"])
@pytest.mark.parametrize("layout", ["q_reuse_k", "k_reuse_q", "separate"])
def test_layouts_and_summaries(layout, summary):
    w = tiny_workload("lay", 2, (2, 16, 64), 64, 0.25, seed_index=400)
    r = run_stages(w, layout=layout, summary=summary)
    for h in range(2):
        check_head(r, 0, h, layout=layout, summary=summary)


@pytest.mark.parametrize("summary", ["reweight", "meanpool"])
def test_block_tail_granularity(summary):
    """SPARK_TAIL_BLOCK: compressed logits from the block's mean query. An odd
    block count leaves the last query-block pair half empty."""
    w = tiny_workload("tail", 2, (3, 8, 40), 128, 0.3, seed_index=700)
    assert w.nb % 2 == 1
    r = run_stages(w, summary=summary, tail="block")
    for h in range(2):
        check_head(r, 0, h, summary=summary, tail="block")


def test_separate_layout_forward_matches_stages():
    """spark_forward with the separate layout writes both permutations and the
    same output as the step-by-step calls."""
    import torch
    w = tiny_workload("sep", 2, (2, 16, 64), 128, 0.2, seed_index=800)
    q, k, v = make_inputs(w)
    r = run_stages(w, layout="separate", qkv=(q, k, v))
    p = r["p"]
    ws = spark.alloc_workspace(p)
    perm = torch.empty(spark.perm_shape(p), dtype=torch.int32, device="cuda")
    out = spark.forward(p, to_dev(q), to_dev(k), to_dev(v), ws=ws, perm=perm)
    assert spark.get_status() == 0
    assert np.array_equal(perm.cpu().numpy(), r["perm"])
    assert np.array_equal(bf16_to_f64(out), r["out"])
    for h in range(2):
        check_head(r, 0, h, layout="separate")


@pytest.mark.parametrize("C", [100, 320])
def test_joint_attention_context_segment(C):
    """Joint attention: video rows with the context keys as exact terms, and
    context rows dense over both segments (C not a multiple of 64 or 128:
    ragged context tiles and a partial last context chunk)."""
    import torch
    from spark_gen import f32_to_bf16_bits
    w = tiny_workload("joint", 2, (2, 16, 64), 128, 0.25, seed_index=900)
    q, k, v = make_inputs(w)
    B, H, N, d = q.shape
    rng = np.random.default_rng(4242 + C)
    ctx = [f32_to_bf16_bits((rng.standard_normal((B, H, C, d)) * s).astype(np.float32)) for s in (0.8, 0.8, 1.0)]
    p = spark.params(B, H, N, d, w.ratio)
    ws = spark.alloc_workspace(p)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    MQ, MK, qmean = spark.moments(p, qd, kd, ws)
    perm = spark.reblock(p, qd, kd, MQ, MK, ws)
    sel = spark.select(p, qd, kd, vd, perm, qmean, ws)
    qc, kc, vc = (to_dev(c) for c in ctx)
    out, outc, lse, lsec = spark.attn_fwd_joint(p, perm, sel, qc, kc, vc, ws, return_lse=True)
    assert spark.get_status() == 0
    out, outc = bf16_to_f64(out), bf16_to_f64(outc)
    lse, lsec = lse.cpu().numpy(), lsec.cpu().numpy()
    perm_h, sel_h = perm.cpu().numpy(), sel.cpu().numpy()
    for h in range(H):
        qh, kh, vh = (bf16_bits_to_f64(x[0, h]) for x in (q, k, v))
        ch = [bf16_bits_to_f64(c[0, h]) for c in ctx]
        pm = perm_h[0, h].astype(np.int64)
        kt, vt, beta = so.summaries(kh, vh, pm, so.anchor(qh))
        ref, ref_lse, refc, refc_lse = so.joint_attention(qh, kh, vh, pm, sel_h[0, h].astype(np.int64), kt, vt, beta,
                                                          *ch)
        for got, want, gl, wl in ((out[0, h], ref, lse[0, h], ref_lse), (outc[0, h], refc, lsec[0, h], refc_lse)):
            e = parity.out_errors(got, want)
            assert e["max_rel_to_bound"] <= 1.0, e
            assert e["max_abs"] <= 2 ** -7 * np.abs(want).max() + 4e-3 * e["ref_rms"], e
            assert np.abs(gl - wl).max() <= 1e-3 * (1 + np.abs(wl).max())
    # the whole pass with the context segment gives the same rows
    o2, oc2 = spark.forward_joint(p, qd, kd, vd, qc, kc, vc, ws=ws)
    assert np.array_equal(bf16_to_f64(o2), out) and np.array_equal(bf16_to_f64(oc2), outc)


def test_reweight_with_an_offset_anchor():
    """Spark-Reweight with a mean query far from zero ("Spark-H3" news post,
    What Spark-Attn changed, Spark-Reweight bullet and figure: the bias
    restores E[exp x], which mean pooling replaces by exp E[x]). A common
    offset c is added to every query so that the anchor logits qbar . k_j /
    sqrt(d) spread by about three units inside a block; the GPU's k~, v~,
    beta and outputs must match the oracle, and they must be far from what
    mean pooling gives (a GPU that mean-pooled would fail here)."""
    from spark_gen import f32_to_bf16_bits
    w = tiny_workload("anchor", 2, (2, 16, 64), 128, 0.2, seed_index=1100)
    q, k, v = make_inputs(w)
    d = w.d
    rng = np.random.default_rng(77)
    for h in range(w.H):
        kf, qf = bf16_bits_to_f64(k[0, h]), bf16_bits_to_f64(q[0, h])
        u = rng.standard_normal(d)
        u /= np.linalg.norm(u)
        alpha = 3.0 * math.sqrt(d) / float(np.std(kf @ u))
        q[0, h] = f32_to_bf16_bits((qf + alpha * u).astype(np.float32))
    r = run_stages(w, qkv=(q, k, v))
    nb = w.nb
    for h in range(w.H):
        check_head(r, 0, h)
        qf, kf, vf = (bf16_bits_to_f64(x[0, h]) for x in (q, k, v))
        perm = r["perm"][0, h].astype(np.int64)
        qbar = so.anchor(qf)
        x = (kf @ qbar) / math.sqrt(d)
        spread = float(np.median([np.std(x[perm[64 * b:64 * (b + 1)]]) for b in range(nb)]))
        assert spread > 1.5, spread
        gk, gb = r["kt"][0, h, :nb], r["beta"][0, h, :nb]
        kmean, _, bmean = so.summaries(kf, vf, perm, qbar, "meanpool")
        beta_tol = 1e-4 * (1 + np.abs(gb).max())
        assert np.abs(gb - bmean).max() > 100 * beta_tol           # beta far from ln 64
        k_tol = 2 ** -8 * np.abs(gk) + 1e-6 * np.abs(gk).max()
        assert (np.abs(gk - kmean) / k_tol).max() > 100             # k~ far from the block mean


def test_forward_host_uneven_chunks_with_lse():
    """spark_forward_host with B = 2, H = 5 (ten heads in four uneven chunks,
    batch items flattened) and lse requested: out and lse equal
    spark_forward's bit for bit."""
    import torch
    w = tiny_workload("hostchunks", 5, (2, 16, 32), 128, 0.2, seed_index=1200, B=2)
    q, k, v = make_inputs(w)
    p = spark.params(2, 5, w.N, w.d, w.ratio)
    ws = spark.alloc_workspace(p)
    lse = torch.empty(2, 5, w.N, dtype=torch.float32, device="cuda")
    out = spark.forward(p, to_dev(q), to_dev(k), to_dev(v), ws=ws, lse=lse)
    assert spark.get_status() == 0
    hws = spark.alloc_workspace(p, host=True)
    qh, kh, vh = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty(2, 5, w.N, dtype=torch.float32).pin_memory()
    spark.forward_host(p, qh, kh, vh, oh, hws, lse_host=lh)
    assert spark.get_status() == 0
    assert torch.equal(oh, out.cpu())
    assert torch.equal(lh, lse.cpu())


def test_lite_reblock_power_iters():
    """The Lite reblock reading: 4 power iterations per split; every split is
    replayed by the oracle with the same count."""
    w = tiny_workload("lite", 2, (2, 16, 64), 128, 0.2, seed_index=1000)
    r = run_stages(w, power_iters=4)
    for h in range(2):
        check_head(r, 0, h, power_iters=4)


def test_topk_blocks_and_batch():
    w = tiny_workload("tb", 3, (2, 16, 32), 128, 0.2, seed_index=500, B=2)
    r = run_stages(w, topk_blocks=5)
    assert r["sel"].shape[-1] == 5
    for b in range(2):
        for h in range(3):
            check_head(r, b, h)


def test_positional_tiles_layout():
    import torch
    w = WORKLOADS["tiny_4096"]
    q, k, v = make_inputs(w)
    p = spark.params(1, 2, w.N, w.d, 0.2)
    perm = spark.positional_perm(p, w.grid)
    ref = so.positional_tiles(w.grid)
    got = perm.cpu().numpy()
    assert np.array_equal(got[0, 0], ref) and np.array_equal(got[0, 1], ref)
    r = run_stages(w, summary="meanpool", qkv=(q, k, v), perm=perm)
    for h in range(2):
        check_head(r, 0, h, summary="meanpool", check_perm=False)
    del torch


def test_degenerate_inputs():
    # identical keys inside every positional block, constant values, and an
    # all-zero query head (zero whitened vectors: index order decides)
    w = tiny_workload("deg", 2, (2, 8, 32), 64, 0.3, seed_index=600)
    q, k, v = make_inputs(w)
    N = w.N
    k[0, 0] = np.repeat(k[0, 0, ::64], 64, axis=0)
    v[0, 0] = v[0, 0, :1]
    q[0, 1] = 0
    r = run_stages(w, qkv=(q, k, v))
    check_head(r, 0, 0)
    check_head(r, 0, 1)
    assert np.allclose(r["out"][0, 0], bf16_bits_to_f64(v[0, 0, :1]), atol=0, rtol=2 ** -8)
    perm1 = r["perm"][0, 1]
    assert np.array_equal(perm1, np.arange(N))       # zero vectors: index order
    del N


def test_forward_matches_stages_and_is_deterministic():
    import torch
    w = WORKLOADS["mid_16128"]
    q, k, v = make_inputs(w, heads=[0, 1, 2])
    p = spark.params(1, 3, w.N, w.d, w.ratio)
    ws = spark.alloc_workspace(p)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    outs = []
    for _ in range(2):
        out = spark.forward(p, qd, kd, vd, ws=ws)
        outs.append(out.clone())
    assert torch.equal(outs[0], outs[1])
    r = run_stages(w, qkv=(q, k, v))
    assert np.array_equal(bf16_to_f64(outs[0]), r["out"])
    # host-buffer entry point
    hws = spark.alloc_workspace(p, host=True)
    qh, kh, vh = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    spark.forward_host(p, qh, kh, vh, oh, hws)
    assert spark.get_status() == 0
    assert torch.equal(oh, outs[0].cpu())


def sampled_workload_check(w, ratio, pairs, rows_per_head=12, seed=7, qkv=None):
    """One spark_forward pass over the whole workload (the launch the bench
    times), then per sampled (batch item, head): u_hat equal to the oracle's
    element for element, every split replayed by the oracle on its own u_hat
    (certified near-ties counted, failures none), the selection certified,
    summaries and sampled query blocks of the output against the oracle."""
    import torch
    qh, kh, vh = qkv if qkv is not None else make_inputs(w, procs=host_procs())
    B, H, N, d = qh.shape
    p = spark.params(B, H, N, d, ratio)
    ksel = spark.num_selected(p)
    nb = N // 64
    ws = spark.alloc_workspace(p)
    out = spark.forward(p, to_dev(qh), to_dev(kh), to_dev(vh), ws=ws)
    assert spark.get_status() == 0
    nbp = spark.workspace_region(p, "BETA")[1] // (4 * B * H)
    view = lambda n, dt, sh: spark.ws_view(ws, p, n, dt, sh)  # noqa: E731
    MK = view("MK", torch.float64, (B, H, d, d))
    qmean = view("QMEAN", torch.float64, (B, H, d))
    perm = view("PERM", torch.int32, (B, H, N))
    sel = view("SEL", torch.int32, (B, H, nb, ksel))
    uhat = view("UHAT", torch.bfloat16, (B, H, N, d))
    kt = view("KT", torch.bfloat16, (B, H, nbp, d))
    vt = view("VT", torch.bfloat16, (B, H, nbp, d))
    beta = view("BETA", torch.float32, (B, H, nbp))
    rng = np.random.default_rng(seed)
    rep = []
    for b, h in pairs:
        q, k, v = (bf16_bits_to_f64(x[b, h]) for x in (qh, kh, vh))
        Kk = so.second_moment(k)
        assert np.abs(MK[b, h].cpu().numpy() - Kk).max() <= MOMENT_TOL * np.abs(Kk).max()
        qbar = so.anchor(q)
        assert np.abs(qmean[b, h].cpu().numpy() - qbar).max() <= 1e-12 * (1 + np.abs(qbar).max())
        pm = perm[b, h].cpu().numpy().astype(np.int64)
        U = so.normalized_whitened(q, so.whitening_factor(Kk))
        flips = int((bf16_to_f64(uhat[b, h]) != U).sum())
        assert flips == 0, f"head {h}: u_hat differs from the oracle's in {flips} elements"
        st = parity.certify_perm(q, Kk, pm)
        print("item", b, "head", h, "splits", st["nodes"], "certified near-ties", st["certified"],
              "failures", st["failures"], "worst", st["worst"])
        assert st["failures"] == 0, st
        qm, km = so.block_means(q, pm), so.block_means(k, pm)
        sh = sel[b, h].cpu().numpy().astype(np.int64)
        sst = parity.certify_select(qm, km, ksel, sh)
        assert sst["failures"] == 0, sst
        rkt, rvt, rbeta = so.summaries(k, v, pm, qbar)
        gk = bf16_to_f64(kt[b, h, :nb])
        gv = bf16_to_f64(vt[b, h, :nb])
        gb = beta[b, h, :nb].cpu().numpy().astype(np.float64)
        assert np.all(np.abs(gk - rkt) <= 2 ** -8 * np.abs(rkt) + 1e-6 * np.abs(rkt).max())
        assert np.all(np.abs(gv - rvt) <= 2 ** -8 * np.abs(rvt) + 1e-6 * np.abs(rvt).max())
        check_beta(gk, gb, rkt, rbeta, qbar, "reweight")
        rows = sorted(rng.choice(nb, rows_per_head, replace=False).tolist()) + [nb - 1]
        ref, _ = so.attention(q, k, v, pm, sh, rkt, rvt, rbeta, rows=rows)
        mask = ~np.isnan(ref[:, 0])
        got = bf16_to_f64(out[b, h])
        e = parity.out_errors(got[mask], ref[mask])
        assert e["max_rel_to_bound"] <= 1.0, e
        assert e["max_abs"] <= 2 ** -7 * np.abs(ref[mask]).max() + 4e-3 * e["ref_rms"], e
        rep.append(dict(item=b, head=h, splits=st["nodes"], certified=st["certified"],
                        sel_certified=sst["certified"], max_abs=e["max_abs"]))
    print(rep)
    return rep


def test_reference_size_sampled():
    """The 72,576-token workload in the configuration bench.py times
    (spark_forward, ratio 0.2, all 40 heads); the oracle checks two temporal
    (0, 30) and two spatial (17, 33) heads in full for layout and selection,
    and sampled query blocks for the outputs."""
    sampled_workload_check(WORKLOADS["ref_72576"], 0.2, [(0, 0), (0, 17), (0, 30), (0, 33)])


@pytest.mark.parametrize("ratio", [0.1, 0.3])
def test_reference_size_other_ratios(ratio):
    """The other two densities of the bench's sweep (Ksel 114 and 341), all
    40 heads in one pass; one temporal and one spatial head checked."""
    sampled_workload_check(WORKLOADS["ref_72576"], ratio, [(0, 10), (0, 21)], seed=11)


def test_long_clip_two_items_sampled():
    """The B = 2, 104,832-token workload of the dense-comparison report
    (ratio 0.1, Ksel 164), both batch items in one pass; one head of each."""
    sampled_workload_check(WORKLOADS["long_104832"], 0.1, [(0, 3), (1, 20)], rows_per_head=8, seed=13)


def test_stress_size_sampled():
    """The 129,024-token workload of the statistics report (ratio 0.2,
    Ksel 404, nb = 2,016); one temporal and one spatial head."""
    sampled_workload_check(WORKLOADS["stress_129024"], 0.2, [(0, 0), (0, 7)], rows_per_head=8, seed=17)


@pytest.mark.parametrize("summary", ["reweight", "meanpool"])
def test_report_stats_match_oracle_definitions(summary):
    """bench.py --report stats computes mass recall and log-mass error on the
    device in float64; on the GPU's own perm, sel and summaries they equal
    the oracle's definitions of the two statistics."""
    import torch
    import bench
    w = WORKLOADS["mid_16128"]
    r = run_stages(w, summary=summary)
    B, H, N, d = r["q"].shape
    nb = N // 64
    ksel = r["sel"].shape[-1] if r["sel"].ndim == 4 else spark.num_selected(r["p"])
    sel = r["sel"].reshape(B, H, nb, ksel)
    blocks = np.array([0, 5, 17, nb - 1])
    for h in (0, 3):
        q = bf16_bits_to_f64(r["q"][0, h])
        k = bf16_bits_to_f64(r["k"][0, h])
        perm = r["perm"][0, h].astype(np.int64)
        rec = so.mass_recall(q, k, perm, sel[0, h], blocks)
        lme = so.log_mass_error(q, k, perm, sel[0, h], r["kt"][0, h], r["beta"][0, h], blocks)
        kt = torch.from_numpy(r["kt"][0, h]).cuda().to(torch.bfloat16)      # bf16 values, exactly
        rs, nr, es, ne = bench.head_block_stats(
            to_dev(r["q"][0, h]), to_dev(r["k"][0, h]), torch.from_numpy(perm).cuda(),
            torch.from_numpy(sel[0, h]).cuda(), kt, torch.from_numpy(r["beta"][0, h]).cuda(),
            torch.from_numpy(blocks).cuda(), chunk=3)
        assert nr == 64 * len(blocks)
        assert ne == 64 * len(blocks) * (nb - ksel)
        assert 100.0 * rs / nr == pytest.approx(rec, rel=1e-9, abs=1e-9)
        assert es / ne == pytest.approx(lme, rel=1e-9, abs=1e-12)
