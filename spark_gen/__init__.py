"""Seeded synthetic inputs for the Spark-Attn forward pass.

This module is the only code the CPU oracle and the CUDA path share. It holds
none of the method's arithmetic: it draws Q, K and V, rounds them to bfloat16
and returns the raw bytes. Both sides then read the same bytes.

Workload recipe (a stand-in for real MiniMax-H3 activations on VBench prompts,
which are not available here). Shapes follow the node page "MiniMax H3 Spark
Attention (SM89)", section "What it's doing under the hood": a 10-second 768p
sample has 72,576 video tokens = 1,134 blocks of 64. With a 16x spatial
downsample, 1344x768 is a 84x48 latent, so 18 latent frames give 72,576 tokens.

Per (batch item, head):
  * 32 Fourier features phi_m(f, y, x) = cos(2*pi*(wf_m*f + wy_m*y + wx_m*x) + psi_m),
    each frequency drawn from +-Uniform(0.02, 0.2) cycles per token (random sign),
    psi ~ Uniform[0, 2*pi).
  * "temporal" heads (h % 10 == 0, only for the 40-head workloads) have
    wy = wx = 0; every other head of those workloads is "spatial" (wf = 0).
    The small workloads use all three axes.
  * Q = Phi @ W_Q + sigma * N(0,1), K = Phi @ W_K + sigma * N(0,1),
    W ~ randn(32, d) / sqrt(d). V ~ N(0, 1).
  * Everything is rounded to bfloat16 (round to nearest, ties to even).
Tokens are in raster order t = (f * Hl + y) * Wl + x.
Seeds: numpy SeedSequence(0x5EED + workload index), spawned per (batch, head),
then per tensor, so any head can be drawn on its own.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_head", "host_procs", "bf16_bits_to_f64",
           "bf16_bits_to_f32", "f32_to_bf16_bits", "tiny_workload"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes plus generator settings."""
    name: str
    index: int            # seed offset
    B: int
    H: int
    grid: tuple           # (F, Hl, Wl) latent grid
    d: int
    ratio: float          # default top-k ratio of this workload
    sigma: float          # Q/K noise level
    temporal: bool        # 10% temporal heads / 90% spatial heads
    ratios: tuple = ()    # sweep of ratios (defaults to (ratio,))

    @property
    def N(self) -> int:
        F, Hl, Wl = self.grid
        return F * Hl * Wl

    @property
    def nb(self) -> int:
        return self.N // 64

    def sweep(self) -> tuple:
        return self.ratios or (self.ratio,)


WORKLOADS = {
    # tiny: H=2, 4x16x64 grid, d=64, ratio 0.2, sigma 0.3
    "tiny_4096": Workload("tiny_4096", 0, 1, 2, (4, 16, 64), 64, 0.2, 0.3, False),
    # mid layer slice: H=8, 4x48x84 grid, d=128, ratio 0.1, sigma 0.2
    "mid_16128": Workload("mid_16128", 1, 1, 8, (4, 48, 84), 128, 0.1, 0.2, False),
    # the pages' reference size: H=40, 18x48x84 grid, d=128, ratios 0.1/0.2/0.3
    "ref_72576": Workload("ref_72576", 2, 1, 40, (18, 48, 84), 128, 0.2, 0.2, True,
                          (0.1, 0.2, 0.3)),
    # longer clip, batch 2 (two independent draws)
    "long_104832": Workload("long_104832", 3, 2, 40, (26, 48, 84), 128, 0.1, 0.2, True),
    # stress / ablation size
    "stress_129024": Workload("stress_129024", 4, 1, 40, (32, 48, 84), 128, 0.2, 0.2, True),
}


def tiny_workload(name: str, H: int, grid: tuple, d: int, ratio: float = 0.2,
                  sigma: float = 0.3, seed_index: int = 100, B: int = 1,
                  temporal: bool = False) -> Workload:
    """A small ad-hoc workload with the same recipe (for edge-case tests)."""
    return Workload(name, seed_index, B, H, tuple(grid), d, ratio, sigma, temporal)


# ---------------------------------------------------------------- bf16 bytes

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    rounding = 0x7FFF + ((bits >> 16) & 1)
    out = ((bits + rounding) >> 16).astype(np.uint16)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


# ---------------------------------------------------------------- generator

def _features(rng: np.random.Generator, w: Workload, head: int) -> np.ndarray:
    F, Hl, Wl = w.grid
    nfeat = 32

    def freq():
        mag = rng.uniform(0.02, 0.2, size=nfeat)
        sign = np.where(rng.random(nfeat) < 0.5, -1.0, 1.0)
        return mag * sign

    wf, wy, wx = freq(), freq(), freq()
    psi = rng.uniform(0.0, 2.0 * math.pi, size=nfeat)
    if w.temporal:
        if head % 10 == 0:
            wy[:] = 0.0
            wx[:] = 0.0
        else:
            wf[:] = 0.0
    f = np.arange(F, dtype=np.float64)[:, None, None]
    y = np.arange(Hl, dtype=np.float64)[None, :, None]
    x = np.arange(Wl, dtype=np.float64)[None, None, :]
    phase = (f[..., None] * wf + y[..., None] * wy + x[..., None] * wx)  # F,Hl,Wl,32
    phi = np.cos(2.0 * math.pi * phase + psi).reshape(F * Hl * Wl, nfeat)
    return phi


def make_head(w: Workload, b: int, h: int):
    """Draw (q, k, v) bf16 bit arrays [N, d] for one (batch item, head)."""
    root = np.random.SeedSequence(0x5EED + w.index)
    head_ss = root.spawn(w.B * w.H)[b * w.H + h]
    s_feat, s_q, s_k, s_v = head_ss.spawn(4)
    rng = np.random.Generator(np.random.PCG64(s_feat))
    phi = _features(rng, w, h)
    wq = rng.standard_normal((32, w.d)) / math.sqrt(w.d)
    wk = rng.standard_normal((32, w.d)) / math.sqrt(w.d)
    N = w.N
    zq = np.random.Generator(np.random.PCG64(s_q)).standard_normal((N, w.d), dtype=np.float32)
    zk = np.random.Generator(np.random.PCG64(s_k)).standard_normal((N, w.d), dtype=np.float32)
    vv = np.random.Generator(np.random.PCG64(s_v)).standard_normal((N, w.d), dtype=np.float32)
    q = (phi @ wq).astype(np.float32) + np.float32(w.sigma) * zq
    k = (phi @ wk).astype(np.float32) + np.float32(w.sigma) * zk
    return f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(vv)


def _head_job(args):
    w, b, h = args
    return make_head(w, b, h)


def make_inputs(w: Workload, heads=None, procs: int = 1):
    """Draw q, k, v as uint16 bf16 bit arrays of shape [B, H', N, d].

    heads: optional list of head indices (default: all H heads); batch items
    are always all drawn. procs > 1 draws the heads in a pool of that many
    fresh ("spawn") processes, which is safe after CUDA has been initialised
    in this process; every head has its own seed, so the result is the same.
    A spawned worker imports the calling program's main module again, so a
    script that calls this with procs > 1 must keep its top-level work under
    `if __name__ == "__main__":` (pytest's and bench.py's entry points do).
    """
    hs = list(range(w.H)) if heads is None else list(heads)
    shape = (w.B, len(hs), w.N, w.d)
    q = np.empty(shape, dtype=np.uint16)
    k = np.empty(shape, dtype=np.uint16)
    v = np.empty(shape, dtype=np.uint16)
    jobs = [(w, b, h) for b in range(w.B) for h in hs]
    if procs > 1 and len(jobs) > 1:
        import multiprocessing as mp
        with mp.get_context("spawn").Pool(min(procs, len(jobs))) as pool:
            res = pool.map(_head_job, jobs)
    else:
        res = map(_head_job, jobs)
    for (_, b, h), (qq, kk, vv) in zip(jobs, res):
        j = hs.index(h)
        q[b, j], k[b, j], v[b, j] = qq, kk, vv
    return q, k, v


def host_procs() -> int:
    """Host cores this process may use (for make_inputs' pool)."""
    import os
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1
