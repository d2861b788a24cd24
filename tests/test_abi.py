"""Host-side checks of the C ABI: the library loads, exports every entry
point include/spark.h declares, and validates arguments before launching
anything. No GPU is needed (no compute call is made)."""

import ctypes
import os
import re
import subprocess

import pytest

import block_sparse_attention_spark_b200 as spark
from oracle import spark_oracle as so
from spark_gen import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spark.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(spark_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = spark.lib()
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", spark.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (spark_\w+)", out))
    assert set(names) <= exported


def test_params_struct_layout():
    # B, H, N, d, topk_ratio (8-aligned), topk_blocks, layout, summary, tail, power_iters, padding
    assert ctypes.sizeof(spark.Params) == 48
    assert spark.Params.topk_ratio.offset == 16
    assert spark.Params.power_iters.offset == 40


def test_power_iters_range():
    assert spark.validate(P(power_iters=4)) == 0
    assert spark.validate(P(power_iters=64)) == 0
    assert spark.validate(P(power_iters=65)) == 1
    assert spark.validate(P(power_iters=-1)) == 1


def P(**kw):
    base = dict(B=1, H=2, N=4096, d=64, topk_ratio=0.2)
    base.update(kw)
    return spark.params(**base)


def test_validate_accepts_workloads():
    for w in WORKLOADS.values():
        for r in w.sweep():
            p = spark.params(w.B, w.H, w.N, w.d, r)
            assert spark.validate(p) == 0
            assert spark.num_selected(p) == so.num_selected(w.nb, r)
            assert spark.workspace_size(p) > 0
            assert spark.host_workspace_size(p) >= _host_bytes_at_least(w.B, w.H, w.N, w.d, r)


@pytest.mark.parametrize("B,H", [(1, 1), (1, 2), (1, 3), (2, 5), (1, 9), (1, 16), (2, 20), (1, 40), (3, 37)])
def test_host_workspace_holds_two_lanes_and_the_copies(B, H):
    """The host-buffer pass: room for the device copies of every head plus one
    workspace per compute lane for the largest head chunk; from 16 heads on
    (chunks of at most a quarter of the heads, two lanes) that is less than
    the whole problem's workspace plus the copies."""
    N, d, r = 64 * 40, 128, 0.2
    p = spark.params(B, H, N, d, r)
    staging = 4 * B * H * N * d * 2 + B * H * N * 4
    assert spark.host_workspace_size(p) >= _host_bytes_at_least(B, H, N, d, r)
    if B * H >= 16:
        assert spark.host_workspace_size(p) < spark.workspace_size(p) + staging


def _host_bytes_at_least(B, H, N, d, r):
    """The host-buffer pass keeps device copies of q, k, v, out and lse of
    every head, and one workspace per compute lane (two lanes when there are
    two or more heads), each for the largest of up to eight head chunks run
    as problems of their own."""
    BH = B * H
    chunks = min(BH, 8)
    largest = -(-BH // chunks)
    lanes = min(chunks, 2)
    staging = 4 * BH * N * d * 2 + BH * N * 4
    return lanes * spark.workspace_size(spark.params(1, largest, N, d, r)) + staging


@pytest.mark.parametrize("kw,code", [
    (dict(N=4100), 2), (dict(N=64), 2), (dict(d=96), 2), (dict(d=256), 2),
    (dict(topk_ratio=0.0), 2), (dict(topk_ratio=1.5), 2), (dict(topk_ratio=float("nan")), 2),
    (dict(N=64 * 8193), 2), (dict(B=0), 1), (dict(H=-1), 1),
])
def test_validate_rejects(kw, code):
    p = P(**kw)
    assert spark.validate(p) == code
    assert spark.workspace_size(p) == 0
    assert spark.num_selected(p) == -1


def test_bad_enums_rejected():
    p = P()
    p.layout = 7
    assert spark.validate(p) == 1
    p = P()
    p.summary = 3
    assert spark.validate(p) == 1
    p = P()
    p.tail = 2
    assert spark.validate(p) == 1
    p = P()
    p.tail = 1                      # SPARK_TAIL_BLOCK is a valid granularity
    assert spark.validate(p) == 0
    p = P(topk_blocks=-2)
    assert spark.validate(p) == 1


@pytest.mark.parametrize("nb,r,blocks", [(64, 0.2, 0), (1134, 0.1, 0), (1134, 0.3, 0), (2, 0.01, 0),
                                         (10, 0.3, 0), (1000, 0.3, 0), (64, 0.2, 5), (64, 0.2, 99)])
def test_num_selected_matches_oracle(nb, r, blocks):
    p = P(N=64 * nb, topk_ratio=r, topk_blocks=blocks)
    assert spark.num_selected(p) == so.num_selected(nb, r, blocks)


def test_entry_points_reject_null_and_small_workspace_without_launching():
    L = spark.lib()
    p = P()
    n = spark.workspace_size(p)
    fake = ctypes.c_void_p(1 << 20)           # never dereferenced: validation fails first
    assert L.spark_moments(ctypes.byref(p), None, fake, fake, fake, fake, fake, n, None) == 1
    assert L.spark_moments(ctypes.byref(p), fake, fake, fake, fake, fake, fake, n - 1, None) == 3
    assert L.spark_reblock(ctypes.byref(p), fake, fake, fake, fake, None, fake, n, None) == 1
    # q_reuse_k whitens the queries with M_K: M_K is required, M_Q is not read
    assert L.spark_reblock(ctypes.byref(p), fake, fake, fake, None, fake, fake, n, None) == 1
    # the bounded-wait diagnostic checks its limit before launching
    assert L.spark_selftest_wait(0, None) == 1
    assert L.spark_selftest_wait(3_000_000_000, None) == 1
    assert L.spark_select(ctypes.byref(p), fake, fake, fake, fake, fake, None, fake, n, None) == 1
    assert L.spark_attn_fwd(ctypes.byref(p), fake, fake, fake, None, None, n, None) == 1
    assert L.spark_attn_fwd(ctypes.byref(p), fake, fake, fake, None, fake, 16, None) == 3
    mis = ctypes.c_void_p((1 << 20) + 2)      # misaligned
    assert L.spark_forward(ctypes.byref(p), mis, fake, fake, fake, None, None, None, fake, n, None) == 1
    assert L.spark_forward_host(ctypes.byref(p), fake, fake, fake, fake, None, fake, n, None) == 3
    bad = P(N=100)
    assert L.spark_forward(ctypes.byref(bad), fake, fake, fake, fake, None, None, None, fake, n, None) == 2
    assert L.spark_positional_perm(ctypes.byref(p), 4, 16, 63, fake, None) == 1   # 4*16*63 != N
    assert L.spark_positional_perm(ctypes.byref(P(N=64 * 3 * 2 * 2)), 3, 8, 32, fake, None) == 2


def test_workspace_regions_are_disjoint_and_inside():
    p = P(B=2, H=3, N=64 * 37, d=128, topk_ratio=0.3)
    total = spark.workspace_size(p)
    spans = []
    for name in spark.WS:
        off, n = spark.workspace_region(p, name)
        assert off % 256 == 0 and off + n <= total
        spans.append((off, off + n))
    spans.sort()
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0


def test_strerror():
    L = spark.lib()
    for c in range(6):
        assert L.spark_strerror(c)
    assert L.spark_strerror(99) == b"unknown status"
