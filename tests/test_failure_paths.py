"""Failure paths of the device code, made without any GPU fault.

(a) A bounded wait that expires: spark_selftest_wait waits, through the same
    routine every kernel uses, on a barrier phase that nothing completes; the
    wait gives up after a millisecond and the status word reports
    SPARK_ERR_TIMEOUT. The next normal call runs and matches the oracle.
(b) Caller indices out of range ("MiniMax H3 Spark Attention (SM89)",
    Inputs: strict mode errors out on unsupported input): a permutation or a
    selection entry outside its range is clamped or skipped by the kernels'
    own bounds checks and reported as SPARK_ERR_UNSUPPORTED; nothing reads or
    writes outside the buffers.
"""

import numpy as np
import pytest

import block_sparse_attention_spark_b200 as spark
from spark_gen import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TIMEOUT, UNSUPPORTED = 5, 2


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _stages():
    w = WORKLOADS["tiny_4096"]
    q, k, v = (_dev(x) for x in make_inputs(w))
    p = spark.params(w.B, w.H, w.N, w.d, w.ratio)
    ws = spark.alloc_workspace(p)
    MQ, MK, qm = spark.moments(p, q, k, ws)
    perm = spark.reblock(p, q, k, MQ, MK, ws)
    sel = spark.select(p, q, k, v, perm, qm, ws)
    out = spark.attn_fwd(p, perm, sel, ws)
    assert spark.get_status() == 0
    return w, p, ws, q, k, v, qm, perm, sel, out


def test_bounded_wait_expires_and_is_reported():
    import torch
    w, p, ws, q, k, v, qm, perm, sel, out = _stages()
    spark.selftest_wait(1_000_000)                       # 1 ms
    assert spark.get_status() == TIMEOUT
    assert spark.get_status() == 0                       # read and cleared
    # the context is still usable: the same pass gives the same rows
    out2 = spark.forward(p, q, k, v, ws=ws)
    assert spark.get_status() == 0
    assert torch.equal(out, out2)


def test_out_of_range_permutation_entry_in_select():
    w, p, ws, q, k, v, qm, perm, sel, out = _stages()
    bad = perm.clone()
    bad[0, 1, 77] = w.N + 11
    spark.select(p, q, k, v, bad, qm, ws)
    assert spark.get_status() == UNSUPPORTED
    spark.select(p, q, k, v, perm, qm, ws)
    assert spark.get_status() == 0


def test_out_of_range_selection_entry_in_attention():
    w, p, ws, q, k, v, qm, perm, sel, out = _stages()
    bad = sel.clone()
    bad[0, 0, 3, 1] = w.nb + 2
    spark.attn_fwd(p, perm, bad, ws)
    assert spark.get_status() == UNSUPPORTED
    spark.select(p, q, k, v, perm, qm, ws)               # restores the workspace copies
    spark.attn_fwd(p, perm, sel, ws)
    assert spark.get_status() == 0


def test_negative_permutation_entry_in_attention_output():
    import torch
    w, p, ws, q, k, v, qm, perm, sel, out = _stages()
    bad = perm.clone()
    bad[0, 0, 130] = -1
    spark.attn_fwd(p, bad, sel, ws)
    assert spark.get_status() == UNSUPPORTED
    out2 = spark.attn_fwd(p, perm, sel, ws)
    assert spark.get_status() == 0
    assert torch.equal(out, out2)
