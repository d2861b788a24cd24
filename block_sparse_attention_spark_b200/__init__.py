"""Spark-Attn block-sparse attention forward pass on B200 (sm_100a).

Thin ctypes binding of libspark (include/spark.h): every function marshals
torch tensors into pointers and calls the C ABI on the current CUDA stream.
All arithmetic runs in the library's CUDA kernels; there is no CPU path.
Build the library first:  python -m block_sparse_attention_spark_b200.build
"""

from __future__ import annotations

import ctypes
import os

__all__ = ["SparkError", "Params", "lib", "params", "num_selected", "workspace_size",
           "host_workspace_size", "workspace_region", "alloc_workspace", "moments", "reblock",
           "positional_perm", "select", "attn_fwd", "attn_fwd_joint", "forward", "forward_joint",
           "forward_host", "get_status", "selftest_wait",
           "LAYOUTS", "SUMMARIES", "TAILS", "WS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspark.so")

LAYOUTS = {"q_reuse_k": 0, "k_reuse_q": 1, "separate": 2}
SUMMARIES = {"reweight": 0, "meanpool": 1}
TAILS = {"query": 0, "block": 1}
WS = {"MQ": 0, "MK": 1, "QMEAN": 2, "PERM": 3, "SEL": 4, "QM": 5, "KM": 6, "KT": 7, "VT": 8,
      "BETA": 9, "UHAT": 10, "PAIRS": 11}
STATUS = {0: "SPARK_OK", 1: "SPARK_ERR_INVALID_ARG", 2: "SPARK_ERR_UNSUPPORTED",
          3: "SPARK_ERR_WORKSPACE", 4: "SPARK_ERR_CUDA", 5: "SPARK_ERR_TIMEOUT"}


class SparkError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = lib().spark_strerror(code).decode() if _LIB is not None else ""
        super().__init__(f"{where}: {STATUS.get(code, code)} ({msg})")


class Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("topk_ratio", ctypes.c_double),
                ("topk_blocks", ctypes.c_int32), ("layout", ctypes.c_int32),
                ("summary", ctypes.c_int32), ("tail", ctypes.c_int32),
                ("power_iters", ctypes.c_int32)]

    def __repr__(self):
        return (f"Params(B={self.B}, H={self.H}, N={self.N}, d={self.d}, "
                f"topk_ratio={self.topk_ratio}, topk_blocks={self.topk_blocks}, "
                f"layout={self.layout}, summary={self.summary}, tail={self.tail})")


_LIB = None
_P = ctypes.POINTER(Params)
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_i32 = ctypes.c_int32

_SIGS = {
    "spark_validate": (_i32, [_P]),
    "spark_num_selected": (_i32, [_P]),
    "spark_workspace_size": (_sz, [_P]),
    "spark_host_workspace_size": (_sz, [_P]),
    "spark_forward_launches": (_i32, [_P]),
    "spark_workspace_region": (_sz, [_P, _i32, ctypes.POINTER(_sz)]),
    "spark_moments": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "spark_moments_noalloc": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _vp]),
    "spark_reblock": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "spark_positional_perm": (_i32, [_P, _i32, _i32, _i32, _vp, _vp]),
    "spark_select": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "spark_attn_fwd": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "spark_forward": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "spark_attn_fwd_joint": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "spark_forward_joint": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz,
                                   _vp]),
    "spark_forward_host": (_i32, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "spark_get_status": (_i32, [_vp]),
    "spark_selftest_wait": (_i32, [ctypes.c_int64, _vp]),
    "spark_strerror": (ctypes.c_char_p, [_i32]),
}


def lib():
    """The loaded libspark (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libspark.so not found at {LIB_PATH}; build it with "
                               "`python -m block_sparse_attention_spark_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _check(code: int, where: str):
    if code != 0:
        raise SparkError(code, where)


def params(B, H, N, d, topk_ratio=0.2, topk_blocks=0, layout="q_reuse_k",
           summary="reweight", tail="query", power_iters=0) -> Params:
    return Params(B, H, N, d, float(topk_ratio), int(topk_blocks), LAYOUTS[layout],
                  SUMMARIES[summary], TAILS[tail], int(power_iters))


def validate(p: Params) -> int:
    return lib().spark_validate(ctypes.byref(p))


def num_selected(p: Params) -> int:
    return lib().spark_num_selected(ctypes.byref(p))


def workspace_size(p: Params) -> int:
    return lib().spark_workspace_size(ctypes.byref(p))


def forward_launches(p: Params) -> int:
    """Kernel launches one spark_forward call makes."""
    return lib().spark_forward_launches(ctypes.byref(p))


def host_workspace_size(p: Params) -> int:
    return lib().spark_host_workspace_size(ctypes.byref(p))


def workspace_region(p: Params, name: str):
    """(byte offset, byte size) of a named workspace region."""
    n = _sz(0)
    off = lib().spark_workspace_region(ctypes.byref(p), WS[name], ctypes.byref(n))
    if off == ctypes.c_size_t(-1).value:
        raise SparkError(1, "spark_workspace_region")
    return off, n.value


# ---------------------------------------------------------------- torch glue

def _torch():
    import torch
    return torch


def _stream():
    return _torch().cuda.current_stream().cuda_stream


def _ptr(t):
    if t is None:
        return None
    return t.data_ptr()


def _need(t, dtype, shape, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}, "
                        f"got {t.dtype} {tuple(t.shape)}")


def alloc_workspace(p: Params, host=False):
    torch = _torch()
    n = host_workspace_size(p) if host else workspace_size(p)
    if n == 0:
        _check(validate(p) or 1, "workspace_size")
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def ws_view(ws, p: Params, name: str, dtype, shape):
    """A typed view of one workspace region (no copy)."""
    off, n = workspace_region(p, name)
    esz = _torch().tensor([], dtype=dtype).element_size()
    count = 1
    for s in shape:
        count *= s
    assert count * esz <= n
    return ws[off:off + count * esz].view(dtype).view(*shape)


def moments(p: Params, q, k, ws, which="both"):
    """M_Q, M_K (float64 [B,H,d,d]) and the anchor qbar ([B,H,d]).
    which="layout" forms only the moment(s) the layout partitions under (the
    others come back as None), as spark_forward does."""
    torch = _torch()
    shp = (p.B, p.H, p.N, p.d)
    _need(q, torch.bfloat16, shp, "q")
    _need(k, torch.bfloat16, shp, "k")
    if which not in ("both", "layout"):
        raise ValueError(which)
    lay = p.layout
    want_q = which == "both" or lay != LAYOUTS["q_reuse_k"]
    want_k = which == "both" or lay != LAYOUTS["k_reuse_q"]
    MQ = torch.empty(p.B, p.H, p.d, p.d, dtype=torch.float64, device="cuda") if want_q else None
    MK = torch.empty(p.B, p.H, p.d, p.d, dtype=torch.float64, device="cuda") if want_k else None
    qmean = torch.empty(p.B, p.H, p.d, dtype=torch.float64, device="cuda")
    _check(lib().spark_moments(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(MQ), _ptr(MK), _ptr(qmean),
                               _ptr(ws), ws.numel(), _stream()), "spark_moments")
    return MQ, MK, qmean


def moments_noalloc(p: Params, q, k, MQ, MK, qmean):
    """spark_moments without a workspace: the library's own fixed device
    array holds the partial sums (see include/spark.h for its limit and the
    rules on overlapping calls). Outputs are written into the given tensors."""
    torch = _torch()
    shp = (p.B, p.H, p.N, p.d)
    _need(q, torch.bfloat16, shp, "q")
    _need(k, torch.bfloat16, shp, "k")
    _need(MQ, torch.float64, (p.B, p.H, p.d, p.d), "MQ")
    _need(MK, torch.float64, (p.B, p.H, p.d, p.d), "MK")
    _need(qmean, torch.float64, (p.B, p.H, p.d), "qmean")
    _check(lib().spark_moments_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(MQ), _ptr(MK),
                                       _ptr(qmean), _stream()), "spark_moments_noalloc")
    return MQ, MK, qmean


def perm_shape(p: Params):
    """[B, H, N], or [2, B, H, N] (query, then key permutation) for the separate layout."""
    return (2, p.B, p.H, p.N) if p.layout == LAYOUTS["separate"] else (p.B, p.H, p.N)


def reblock(p: Params, q, k, MQ, MK, ws):
    torch = _torch()
    perm = torch.empty(perm_shape(p), dtype=torch.int32, device="cuda")
    _check(lib().spark_reblock(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(MQ), _ptr(MK), _ptr(perm),
                               _ptr(ws), ws.numel(), _stream()), "spark_reblock")
    return perm


def positional_perm(p: Params, grid):
    torch = _torch()
    F, Hl, Wl = grid
    perm = torch.empty(perm_shape(p), dtype=torch.int32, device="cuda")
    _check(lib().spark_positional_perm(ctypes.byref(p), F, Hl, Wl, _ptr(perm), _stream()),
           "spark_positional_perm")
    return perm


def select(p: Params, q, k, v, perm, qmean, ws):
    torch = _torch()
    ksel = num_selected(p)
    sel = torch.empty(p.B, p.H, p.N // 64, ksel, dtype=torch.int32, device="cuda")
    _check(lib().spark_select(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(perm), _ptr(qmean),
                              _ptr(sel), _ptr(ws), ws.numel(), _stream()), "spark_select")
    return sel


def attn_fwd(p: Params, perm, sel, ws, return_lse=False):
    torch = _torch()
    out = torch.empty(p.B, p.H, p.N, p.d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(p.B, p.H, p.N, dtype=torch.float32, device="cuda") if return_lse else None
    _check(lib().spark_attn_fwd(ctypes.byref(p), _ptr(perm), _ptr(sel), _ptr(out), _ptr(lse),
                                _ptr(ws), ws.numel(), _stream()), "spark_attn_fwd")
    return (out, lse) if return_lse else out


def attn_fwd_joint(p: Params, perm, sel, qc, kc, vc, ws, return_lse=False):
    """Video rows with the context segment, and the context rows (dense).
    qc, kc, vc: [B, H, C, d] bf16. Returns (out, outc) or (out, outc, lse, lsec)."""
    torch = _torch()
    C = qc.shape[2]
    for t, n in ((qc, "qc"), (kc, "kc"), (vc, "vc")):
        _need(t, torch.bfloat16, (p.B, p.H, C, p.d), n)
    out = torch.empty(p.B, p.H, p.N, p.d, dtype=torch.bfloat16, device="cuda")
    outc = torch.empty(p.B, p.H, C, p.d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(p.B, p.H, p.N, dtype=torch.float32, device="cuda") if return_lse else None
    lsec = torch.empty(p.B, p.H, C, dtype=torch.float32, device="cuda") if return_lse else None
    _check(lib().spark_attn_fwd_joint(ctypes.byref(p), _ptr(perm), _ptr(sel), _ptr(qc), _ptr(kc), _ptr(vc), C,
                                      _ptr(out), _ptr(lse), _ptr(outc), _ptr(lsec), _ptr(ws), ws.numel(),
                                      _stream()), "spark_attn_fwd_joint")
    return (out, outc, lse, lsec) if return_lse else (out, outc)


def forward_joint(p: Params, q, k, v, qc, kc, vc, ws=None):
    """The whole pass with a context segment. Returns (out, outc)."""
    torch = _torch()
    C = qc.shape[2]
    shp = (p.B, p.H, p.N, p.d)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, shp, n)
    for t, n in ((qc, "qc"), (kc, "kc"), (vc, "vc")):
        _need(t, torch.bfloat16, (p.B, p.H, C, p.d), n)
    if ws is None:
        ws = alloc_workspace(p)
    out = torch.empty(shp, dtype=torch.bfloat16, device="cuda")
    outc = torch.empty(p.B, p.H, C, p.d, dtype=torch.bfloat16, device="cuda")
    _check(lib().spark_forward_joint(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(qc), _ptr(kc), _ptr(vc), C,
                                     _ptr(out), None, _ptr(outc), None, _ptr(ws), ws.numel(), _stream()),
           "spark_forward_joint")
    return out, outc


def forward(p: Params, q, k, v, ws=None, out=None, lse=None, perm=None, sel=None):
    """The whole pass on device tensors. Returns out (and writes lse/perm/sel
    into the given tensors when they are passed)."""
    torch = _torch()
    shp = (p.B, p.H, p.N, p.d)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, shp, n)
    if ws is None:
        ws = alloc_workspace(p)
    if out is None:
        out = torch.empty(shp, dtype=torch.bfloat16, device="cuda")
    _check(lib().spark_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                               _ptr(perm), _ptr(sel), _ptr(ws), ws.numel(), _stream()),
           "spark_forward")
    return out


def forward_host(p: Params, q_host, k_host, v_host, out_host, ws, lse_host=None):
    """The whole pass on host tensors (CPU torch tensors, pinned for speed)."""
    _check(lib().spark_forward_host(ctypes.byref(p), _ptr(q_host), _ptr(k_host), _ptr(v_host),
                                    _ptr(out_host), _ptr(lse_host), _ptr(ws), ws.numel(),
                                    _stream()), "spark_forward_host")
    return out_host


def selftest_wait(limit_ns: int):
    """Launch the bounded-wait diagnostic (see include/spark.h); the timeout
    shows up in the next get_status()."""
    _check(lib().spark_selftest_wait(int(limit_ns), _stream()), "spark_selftest_wait")


def get_status():
    """Synchronises the current stream and returns the device status code."""
    return lib().spark_get_status(_stream())
