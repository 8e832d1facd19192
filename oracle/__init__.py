"""ORACLE -- test infrastructure, not product code.

Python access to the plain fp64 C oracle in veda_oracle.c (tile pooling ->
selector projection -> tile scoring -> fixed-budget top-k -> restricted
softmax attention).  Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference legs may import this package.  It never imports the
CUDA library, and the CUDA library never imports it.

Inputs are CPU torch tensors in the library's layout ([B, N, H, d] with d
contiguous, fp32 or bf16; weights [H, d, r]); every element is read exactly
into fp64 by the C code.  Outputs are numpy fp64 / int32 arrays.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Dict, Optional, Sequence, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "veda_oracle.c")
_LIB = os.path.join(_HERE, "libveda_oracle.so")

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, OpenMP, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None

_c_i64 = ctypes.c_int64
_c_ptr = ctypes.c_void_p


class _Segment(ctypes.Structure):
    _fields_ = [("k", _c_ptr), ("v", _c_ptr), ("n", _c_i64),
                ("sb", _c_i64), ("st", _c_i64), ("sh", _c_i64)]


class _Problem(ctypes.Structure):
    _fields_ = [("q", _c_ptr), ("qsb", _c_i64), ("qst", _c_i64), ("qsh", _c_i64),
                ("dtype", ctypes.c_int), ("B", _c_i64), ("H", _c_i64), ("d", _c_i64),
                ("T", _c_i64), ("video", _Segment), ("ref", _Segment), ("dense", _Segment),
                ("scale", ctypes.c_double), ("nq_tok", _c_i64)]


def lib():
    global _lib
    if _lib is None:
        # VEDA_ORACLE_LIB loads another build of veda_oracle.c (the mutation
        # tests use it to check that the pins catch planted mistakes)
        path = os.environ.get("VEDA_ORACLE_LIB") or build()
        L = ctypes.CDLL(path)
        L.oracle_pool.argtypes = [_c_ptr, ctypes.c_int] + [_c_i64] * 8 + [_c_ptr]
        L.oracle_project.argtypes = [_c_ptr] + [_c_i64] * 4 + [_c_ptr, ctypes.c_int, _c_i64, _c_ptr]
        L.oracle_scores.argtypes = [_c_ptr, _c_ptr] + [_c_i64] * 5 + [_c_ptr, _c_i64, _c_ptr]
        L.oracle_select.argtypes = [_c_ptr, _c_ptr] + [_c_i64] * 6 + [_c_ptr, _c_ptr, _c_ptr]
        L.oracle_attend.argtypes = [ctypes.POINTER(_Problem), _c_ptr, _c_i64, _c_ptr, _c_i64,
                                    _c_ptr, _c_i64, _c_ptr, _c_ptr]
        for f in ("oracle_pool", "oracle_project", "oracle_scores", "oracle_select", "oracle_attend"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def _code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"oracle takes fp32 or bf16 tensors, got {t.dtype}")


def _cpu(t: torch.Tensor) -> torch.Tensor:
    if t.device.type != "cpu":
        raise ValueError("oracle inputs must be CPU tensors")
    if t.stride(-1) != 1:
        raise ValueError("last dimension must be contiguous")
    return t


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


# ---------------------------------------------------------------------------
# the steps
# ---------------------------------------------------------------------------

def pool(x: torch.Tensor, T: int) -> np.ndarray:
    """Mean over the valid tokens of each tile of T tokens: [B,N,H,d] -> [B,H,n,d] fp64."""
    x = _cpu(x)
    B, N, H, d = x.shape
    n = -(-N // T)
    out = np.empty((B, H, n, d), np.float64)
    sb, st, sh, _ = x.stride()
    lib().oracle_pool(x.data_ptr(), _code(x), B, N, H, d, sb, st, sh, T, _ptr(out))
    return out


def project(pooled: np.ndarray, w: torch.Tensor) -> np.ndarray:
    """pooled [B,H,n,d] fp64 times W[h] ([H,d,r], fp32/bf16) -> [B,H,n,r] fp64."""
    pooled = np.ascontiguousarray(pooled, np.float64)
    w = _cpu(w).contiguous()
    B, H, n, d = pooled.shape
    Hw, dw, r = w.shape
    assert (Hw, dw) == (H, d)
    out = np.empty((B, H, n, r), np.float64)
    lib().oracle_project(_ptr(pooled), B, H, n, d, w.data_ptr(), _code(w), r, _ptr(out))
    return out


def scores(qhat: np.ndarray, khat: np.ndarray, rows: Sequence[int]) -> np.ndarray:
    """Full score rows (raw dot products) for row ids (b*H + h)*nq + i -> [len(rows), nk]."""
    qhat = np.ascontiguousarray(qhat, np.float64)
    khat = np.ascontiguousarray(khat, np.float64)
    B, H, nq, r = qhat.shape
    nk = khat.shape[2]
    rows = np.ascontiguousarray(np.asarray(rows, np.int64))
    out = np.empty((len(rows), nk), np.float64)
    lib().oracle_scores(_ptr(qhat), _ptr(khat), B, H, nq, nk, r, _ptr(rows), len(rows), _ptr(out))
    return out


def select(qhat: np.ndarray, khat: np.ndarray, k: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Fixed-budget top-k per (b,h,i): (idx [B,H,nq,k] int32 ascending,
    k-th score [B,H,nq], (k+1)-th score [B,H,nq] (NaN when k == nk))."""
    qhat = np.ascontiguousarray(qhat, np.float64)
    khat = np.ascontiguousarray(khat, np.float64)
    B, H, nq, r = qhat.shape
    nk = khat.shape[2]
    if not (1 <= k <= nk):
        raise ValueError(f"budget {k} outside [1, {nk}]")
    idx = np.empty((B, H, nq, k), np.int32)
    kth = np.empty((B, H, nq), np.float64)
    nxt = np.empty((B, H, nq), np.float64)
    lib().oracle_select(_ptr(qhat), _ptr(khat), B, H, nq, nk, r, k, _ptr(idx), _ptr(kth), _ptr(nxt))
    return idx, kth, nxt


def attend(q: torch.Tensor, video: Tuple[torch.Tensor, torch.Tensor], T: int,
           idx_v: np.ndarray, units: Sequence[Tuple[int, int, int]],
           ref: Optional[Tuple[torch.Tensor, torch.Tensor]] = None, idx_r: Optional[np.ndarray] = None,
           dense: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
           scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Restricted softmax attention for the listed (b, h, query tile) units.

    q holds the query tokens: the video's own, or the rows of non-video
    (dense) queries, which the caller pairs with every tile (`all_tiles`).
    Returns out [n_units, T, d] and lse [n_units, T] in fp64 (NaN rows past the
    last query token)."""
    q = _cpu(q)
    B, N, H, d = q.shape
    keep = []

    def seg(kv):
        s = _Segment()
        if kv is None:
            s.k = s.v = None
            s.n = s.sb = s.st = s.sh = 0
            return s
        k, v = _cpu(kv[0]), _cpu(kv[1])
        if k.shape != v.shape or k.stride() != v.stride():
            raise ValueError("K and V of a segment must share shape and strides")
        if k.dtype != q.dtype or v.dtype != q.dtype:
            raise ValueError("all tensors of a problem share one dtype")
        keep.extend([k, v])
        s.k, s.v = k.data_ptr(), v.data_ptr()
        s.n = k.shape[1]
        s.sb, s.st, s.sh, _ = k.stride()
        return s

    p = _Problem()
    p.q = q.data_ptr()
    p.qsb, p.qst, p.qsh, _ = q.stride()
    p.dtype = _code(q)
    p.B, p.H, p.d, p.T = B, H, d, T
    p.video = seg(video)
    p.ref = seg(ref)
    p.dense = seg(dense)
    p.scale = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    p.nq_tok = N

    idx_v = np.ascontiguousarray(idx_v, np.int32)
    k_v = idx_v.shape[-1]
    if ref is not None:
        idx_r = np.ascontiguousarray(idx_r, np.int32)
        k_r = idx_r.shape[-1]
    else:
        idx_r, k_r = None, 0
    u = np.ascontiguousarray(np.asarray(units, np.int64).reshape(-1, 3))
    out = np.empty((len(u), T, d), np.float64)
    lse = np.empty((len(u), T), np.float64)
    lib().oracle_attend(ctypes.byref(p), _ptr(idx_v), k_v,
                        _ptr(idx_r) if idx_r is not None else None, k_r,
                        _ptr(u), len(u), _ptr(out), _ptr(lse))
    return out, lse


# ---------------------------------------------------------------------------
# conveniences over one generated problem (dict from workloads.make_inputs)
# ---------------------------------------------------------------------------

def select_tiles(inp: Dict[str, torch.Tensor], T: int, budget_video: int,
                 budget_ref: int = 0) -> Dict[str, np.ndarray]:
    """pool -> project -> score -> top-k for the video segment (and the
    reference segment when present, selected independently with the same
    projections)."""
    qhat = project(pool(inp["q"], T), inp["w_q"])
    khat = project(pool(inp["k"], T), inp["w_k"])
    res = {"qhat": qhat, "khat": khat}
    res["idx_v"], res["kth_v"], res["next_v"] = select(qhat, khat, budget_video)
    if "k_ref" in inp and budget_ref > 0:
        khat_r = project(pool(inp["k_ref"], T), inp["w_k"])
        res["khat_r"] = khat_r
        res["idx_r"], res["kth_r"], res["next_r"] = select(qhat, khat_r, budget_ref)
    return res


def attend_units(inp: Dict[str, torch.Tensor], T: int, idx_v: np.ndarray,
                 idx_r: Optional[np.ndarray], units, scale: Optional[float] = None):
    ref = (inp["k_ref"], inp["v_ref"]) if ("k_ref" in inp and idx_r is not None) else None
    dense = (inp["k_dense"], inp["v_dense"]) if "k_dense" in inp else None
    return attend(inp["q"], (inp["k"], inp["v"]), T, idx_v, units, ref=ref, idx_r=idx_r,
                  dense=dense, scale=scale)


def attend_dense_queries(inp: Dict[str, torch.Tensor], q_rows: torch.Tensor, T: int, units,
                         scale: Optional[float] = None):
    """Dense-query rows: q_rows [B, n_rows, H, d] (text, VLM, audio or
    reference tokens as queries) attend to every tile of every segment of the
    problem `inp` -- all video tiles, all reference tiles, every dense token.
    units: (b, h, query tile of q_rows) triples.  Same outputs as attend()."""
    B, n_rows, H, d = q_rows.shape
    n_v = -(-inp["k"].shape[1] // T)
    nq = -(-n_rows // T)
    idx_v = np.ascontiguousarray(np.broadcast_to(np.arange(n_v, dtype=np.int32), (B, H, nq, n_v)))
    ref, idx_r = None, None
    if "k_ref" in inp:
        n_r = -(-inp["k_ref"].shape[1] // T)
        ref = (inp["k_ref"], inp["v_ref"])
        idx_r = np.ascontiguousarray(np.broadcast_to(np.arange(n_r, dtype=np.int32), (B, H, nq, n_r)))
    dense = (inp["k_dense"], inp["v_dense"]) if "k_dense" in inp else None
    return attend(q_rows, (inp["k"], inp["v"]), T, idx_v, units, ref=ref, idx_r=idx_r, dense=dense,
                  scale=scale)
