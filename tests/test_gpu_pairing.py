"""Query-block pairing of the attention units, read back through the
workspace region SPARK_WS_PAIRS after a full pass (needs a B200).

A row's output does not depend on the query block it is paired with (the
parity tests compare every output with the oracle), so what is checked here
is the pairing itself, against a plain restatement of its rule: inside each
window of 64 consecutive query blocks, repeatedly take the two free blocks
whose selections share the most key blocks (ties to the lower pair index
i * 64 + j, i < j), in that order; an odd last window ends with its free
block alone (partner -1). The units must equal that list exactly, and every
query block of a head must sit in exactly one unit."""

import numpy as np
import pytest

import block_sparse_attention_spark_b200 as spark
from spark_gen import WORKLOADS, host_procs, make_inputs, tiny_workload

pytestmark = pytest.mark.gpu

WIN = 64    # query blocks per pairing window


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _pairs_after_forward(w, heads=None):
    import torch
    q, k, v = make_inputs(w, heads=heads, procs=host_procs() if heads else 1)
    B, H, N, d = q.shape
    p = spark.params(B, H, N, d, w.ratio)
    nb, ksel = N // 64, spark.num_selected(p)
    ws = spark.alloc_workspace(p)
    sel = torch.empty(B, H, nb, ksel, dtype=torch.int32, device="cuda")
    spark.forward(p, _dev(q), _dev(k), _dev(v), ws=ws, sel=sel)
    assert spark.get_status() == 0
    pairs = spark.ws_view(ws, p, "PAIRS", torch.int32, (B, H, (nb + 1) // 2, 2)).cpu().numpy()
    return pairs, sel.cpu().numpy(), nb


def _greedy_pairs(sel, nb):
    """The pairing rule restated with plain loops over each window."""
    M = np.zeros((nb, nb), dtype=np.int64)
    for a in range(nb):
        M[a, sel[a]] = 1
    C = M @ M.T                                   # selected key blocks two query blocks share
    units = []
    for b0 in range(0, nb, WIN):
        m = min(WIN, nb - b0)
        free = set(range(m))
        while len(free) >= 2:
            best = None
            for i in sorted(free):
                for j in sorted(free):
                    if i < j:
                        key = (C[b0 + i, b0 + j], -(i * WIN + j))
                        if best is None or key > best[0]:
                            best = (key, i, j)
            _, i, j = best
            units.append((b0 + i, b0 + j))
            free -= {i, j}
        if free:
            units.append((b0 + free.pop(), -1))
    return np.array(units, dtype=np.int64)


def _check_head(pairs, sel, nb):
    flat = pairs.reshape(-1)
    assert np.array_equal(np.sort(flat[flat >= 0]), np.arange(nb))
    assert np.array_equal(pairs.astype(np.int64), _greedy_pairs(sel, nb))


@pytest.mark.parametrize("name", ["mid_16128", "odd_131"])
def test_pairs_follow_the_greedy_rule(name):
    w = WORKLOADS["mid_16128"] if name == "mid_16128" else \
        tiny_workload("odd131", 2, (2, 8, 4 * 131), 128, 0.2, seed_index=1300)
    pairs, sel, nb = _pairs_after_forward(w)
    for b in range(pairs.shape[0]):
        for h in range(pairs.shape[1]):
            _check_head(pairs[b, h], sel[b, h], nb)


def test_pairs_at_the_reference_size():
    """One temporal and one spatial head of the 72,576-token workload."""
    w = WORKLOADS["ref_72576"]
    pairs, sel, nb = _pairs_after_forward(w, heads=[0, 17])
    for h in range(2):
        _check_head(pairs[0, h], sel[0, h], nb)
