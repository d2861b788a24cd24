"""The allocation-free moments entry point (spark_moments_noalloc).

Some callers cannot allocate or lend device memory (a host framework that
owns every device allocation, a fixed memory plan with no spare workspace).
For them the library offers one call that keeps its scratch in a fixed
device array of its own. This file checks, through the C ABI, that the call
gives the same moments as spark_moments (which uses the caller's workspace)
on two calls in a row, and that it refuses inputs too large for its array
without launching anything. It is named to be collected last.
"""

import ctypes

import numpy as np
import pytest

import block_sparse_attention_spark_b200 as spark
from spark_gen import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _compare(p, q, k):
    import torch
    ws = spark.alloc_workspace(p)
    MQ, MK, qm = spark.moments(p, q, k, ws)
    torch.cuda.synchronize()
    for _ in range(2):   # two calls in a row share the library's array
        MQ2 = torch.full_like(MQ, float("nan"))
        MK2 = torch.full_like(MK, float("nan"))
        qm2 = torch.full_like(qm, float("nan"))
        spark.moments_noalloc(p, q, k, MQ2, MK2, qm2)
        assert spark.get_status() == 0
        for a, b in ((MQ, MQ2), (MK, MK2)):
            a, b = a.cpu().numpy(), b.cpu().numpy()
            assert np.all(np.isfinite(b))
            assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max()
        a, b = qm.cpu().numpy(), qm2.cpu().numpy()
        assert np.abs(a - b).max() <= 1e-12 * (1 + np.abs(a).max())


def test_noalloc_moments_match_workspace_version_small_heads():
    w = WORKLOADS["tiny_4096"]
    q, k, _ = make_inputs(w)
    p = spark.params(w.B, w.H, w.N, w.d, w.ratio)
    _compare(p, _dev(q), _dev(k))


def test_noalloc_moments_match_workspace_version_d128():
    w = WORKLOADS["mid_16128"]
    q, k, _ = make_inputs(w)
    p = spark.params(w.B, w.H, w.N, w.d, w.ratio)
    _compare(p, _dev(q), _dev(k))


def test_noalloc_moments_at_the_head_limit():
    # B*H = 63 heads of d = 128 is the most the 16 MiB array holds
    import torch
    g = torch.Generator(device="cuda").manual_seed(11)
    shape = (1, 63, 2048, 128)
    q = (0.5 * torch.randn(shape, generator=g, device="cuda")).bfloat16()
    k = (0.5 * torch.randn(shape, generator=g, device="cuda")).bfloat16()
    p = spark.params(*shape, 0.2)
    _compare(p, q, k)


def test_noalloc_refuses_inputs_beyond_its_array():
    import torch
    p = spark.params(1, 64, 2048, 128, 0.2)      # 2 * 64 partials of 128*128+128 doubles > 16 MiB
    x = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    code = spark.lib().spark_moments_noalloc(ctypes.byref(p), x.data_ptr(), x.data_ptr(), out.data_ptr(),
                                             out.data_ptr(), out.data_ptr(), None)
    assert code == 2          # SPARK_ERR_UNSUPPORTED, nothing launched
    assert spark.get_status() == 0
