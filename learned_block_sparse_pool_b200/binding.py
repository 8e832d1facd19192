"""ctypes binding of libveda (include/veda.h): argument marshalling only.

Every step of the computation runs in the CUDA library; this module only
fills the C structs from torch tensors (device pointers, element strides) and
passes the current CUDA stream.  There is no fallback: if libveda.so is
missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libveda.so")

VEDA_OK = 0
VEDA_ERR_INVALID_ARG = -1
VEDA_ERR_UNSUPPORTED = -2
VEDA_ERR_WORKSPACE = -3
VEDA_ERR_CUDA = -4
VEDA_ERR_TIMEOUT = -5
VEDA_ERR_BAD_INDEX = -6
VEDA_ERR_FORMAT = -7
VEDA_ERR_IO = -8
VEDA_F32, VEDA_BF16 = 0, 1
VEDA_FLAG_SIMT_ATTENTION = 1
VEDA_FLAG_TEST_SHORT_WAITS = 2
VEDA_FLAG_UNFUSED_SELECTION = 4
VEDA_FLAG_ONCHIP_SELECTION = 8

EXPORTS = ("veda_workspace_size", "veda_workspace_init", "veda_select_tiles", "veda_block_sparse_attn",
           "veda_attn", "veda_pool_project", "veda_score_tiles", "veda_topk_tiles", "veda_workspace_view",
           "veda_check_status", "veda_status_string", "veda_select_tiles_noalloc", "veda_dense_query_attn",
           "veda_selector_open", "veda_selector_close", "veda_selector_check", "veda_selector_count",
           "veda_selector_find", "veda_selector_info", "veda_selector_metadata", "veda_selector_read",
           "veda_attn_host_buffer_size", "veda_attn_host", "veda_score_topk_tiles")


class VedaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} ({status})")
        self.status = status


class veda_segment(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("n_tokens", ctypes.c_int64),
                ("stride_b", ctypes.c_int64), ("stride_tok", ctypes.c_int64), ("stride_h", ctypes.c_int64),
                ("budget", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class veda_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32), ("tile", ctypes.c_int32),
                ("r", ctypes.c_int32), ("dtype", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("flags", ctypes.c_uint32), ("q", ctypes.c_void_p), ("q_stride_b", ctypes.c_int64),
                ("q_stride_tok", ctypes.c_int64), ("q_stride_h", ctypes.c_int64),
                ("video", veda_segment), ("ref", veda_segment), ("dense", veda_segment)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libveda.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m learned_block_sparse_pool_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(veda_problem)
        vp, sz, i32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p
        L.veda_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
        L.veda_workspace_init.argtypes = [vp, sz, vp]
        L.veda_select_tiles.argtypes = [P, vp, vp, i32p, i32p, vp, sz, vp]
        L.veda_block_sparse_attn.argtypes = [P, i32p, i32p, vp, vp, vp, sz, vp]
        L.veda_attn.argtypes = [P, vp, vp, i32p, i32p, vp, vp, vp, sz, vp]
        i64 = ctypes.c_int64
        L.veda_dense_query_attn.argtypes = [P, vp, i64, i64, i64, i64, vp, vp, vp, sz, vp]
        L.veda_pool_project.argtypes = [P, vp, vp, vp, sz, vp]
        L.veda_score_tiles.argtypes = [P, vp, sz, vp]
        L.veda_topk_tiles.argtypes = [P, i32p, i32p, vp, sz, vp]
        L.veda_score_topk_tiles.argtypes = [P, i32p, i32p, vp, sz, vp]
        L.veda_workspace_view.argtypes = [P, vp, sz, ctypes.c_int, ctypes.POINTER(ctypes.c_void_p),
                                          ctypes.POINTER(ctypes.c_int64)]
        L.veda_check_status.argtypes = [vp, vp]
        L.veda_select_tiles_noalloc.argtypes = [P, vp, vp, i32p, i32p, vp]
        L.veda_status_string.argtypes = [ctypes.c_int]
        L.veda_status_string.restype = ctypes.c_char_p
        L.veda_attn_host_buffer_size.argtypes = [P, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
        L.veda_attn_host.argtypes = [P, vp, vp, i32p, i32p, vp, vp, ctypes.c_int32, vp, sz, vp]
        L.veda_selector_open.argtypes = [ctypes.c_char_p, ctypes.POINTER(vp)]
        L.veda_selector_close.argtypes = [vp]
        L.veda_selector_check.argtypes = [vp, ctypes.c_int32, ctypes.POINTER(ctypes.c_int64), ctypes.c_int32,
                                          ctypes.c_int64, ctypes.c_char_p]
        L.veda_selector_count.argtypes = [vp]
        L.veda_selector_find.argtypes = [vp, ctypes.c_char_p, ctypes.POINTER(ctypes.c_int32)]
        L.veda_selector_info.argtypes = [vp, ctypes.c_int32, ctypes.POINTER(ctypes.c_char_p),
                                         ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_int32),
                                         ctypes.POINTER(ctypes.c_int64)]
        L.veda_selector_metadata.argtypes = [vp, ctypes.c_char_p]
        L.veda_selector_read.argtypes = [vp, ctypes.c_int32, ctypes.c_int, ctypes.c_float, vp, sz]
        for name in EXPORTS:
            if name not in ("veda_status_string", "veda_selector_close", "veda_selector_metadata"):
                getattr(L, name).restype = ctypes.c_int
        L.veda_selector_close.restype = None
        L.veda_selector_metadata.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().veda_status_string(int(s)).decode()


def _check(st: int, where: str) -> None:
    if st != VEDA_OK:
        raise VedaError(st, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return VEDA_BF16
    if t.dtype == torch.float32:
        return VEDA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


class Problem:
    """A veda_problem plus references to the tensors it points at."""

    def __init__(self, q, k, v, *, tile: int, r: int, budget: int, k_ref=None, v_ref=None,
                 budget_ref: int = 0, k_dense=None, v_dense=None, scale: float = 0.0, flags: int = 0):
        B, N, H, d = q.shape
        self.tensors = [q, k, v, k_ref, v_ref, k_dense, v_dense]
        c = veda_problem()
        c.B, c.H, c.d, c.tile, c.r = B, H, d, tile, r
        c.dtype = _dtype_code(q)
        c.softmax_scale = float(scale)
        c.flags = int(flags)
        c.q = q.data_ptr()
        c.q_stride_b, c.q_stride_tok, c.q_stride_h = q.stride(0), q.stride(1), q.stride(2)
        self._seg(c.video, k, v, budget)
        self._seg(c.ref, k_ref, v_ref, budget_ref)
        self._seg(c.dense, k_dense, v_dense, 0)
        self.c = c
        self.B, self.H, self.d, self.tile, self.N = B, H, d, tile, N
        self.n_q_tiles = -(-N // tile)
        self.n_ref_tiles = 0 if k_ref is None else -(-k_ref.shape[1] // tile)
        self.budget, self.budget_ref = budget, budget_ref
        self.dtype = q.dtype
        self.device = q.device

    @staticmethod
    def _seg(seg, k, v, budget):
        if k is None:
            seg.k = seg.v = None
            seg.n_tokens = seg.stride_b = seg.stride_tok = seg.stride_h = 0
            seg.budget = int(budget)
            return
        if k.stride() != v.stride() or k.shape != v.shape:
            raise ValueError("k and v of a segment must share shape and strides")
        seg.k, seg.v = k.data_ptr(), v.data_ptr()
        seg.n_tokens = k.shape[1]
        seg.stride_b, seg.stride_tok, seg.stride_h = k.stride(0), k.stride(1), k.stride(2)
        seg.budget = int(budget)

    @property
    def has_ref(self) -> bool:
        return self.c.ref.n_tokens > 0

    def ref(self):
        return ctypes.byref(self.c)


def workspace_size(p: Problem) -> int:
    n = ctypes.c_size_t()
    _check(lib().veda_workspace_size(p.ref(), ctypes.byref(n)), "veda_workspace_size")
    return n.value


def workspace(p: Problem, stream=None) -> torch.Tensor:
    """Allocate (with torch) and initialise a workspace for `p`."""
    n = workspace_size(p)
    ws = torch.empty(n, dtype=torch.uint8, device=p.device)
    if ws.data_ptr() % 256:
        raise RuntimeError("workspace allocation not 256-byte aligned")
    _check(lib().veda_workspace_init(ws.data_ptr(), n, _stream(stream)), "veda_workspace_init")
    return ws


def alloc_indices(p: Problem) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    iv = torch.empty((p.B, p.H, p.n_q_tiles, p.budget), dtype=torch.int32, device=p.device)
    ir = (torch.empty((p.B, p.H, p.n_q_tiles, p.budget_ref), dtype=torch.int32, device=p.device)
          if p.has_ref else None)
    return iv, ir


def alloc_output(p: Problem, with_lse: bool = False):
    out = torch.empty((p.B, p.N, p.H, p.d), dtype=p.dtype, device=p.device)
    lse = torch.empty((p.B, p.H, p.N), dtype=torch.float32, device=p.device) if with_lse else None
    return out, lse


def select_tiles(p: Problem, w_q, w_k, idx_v, idx_r, ws, stream=None) -> None:
    _check(lib().veda_select_tiles(p.ref(), w_q.data_ptr(), w_k.data_ptr(), _ptr(idx_v), _ptr(idx_r),
                                   ws.data_ptr(), ws.numel(), _stream(stream)), "veda_select_tiles")


def select_tiles_noalloc(p: Problem, w_q, w_k, idx_v, idx_r, stream=None) -> None:
    """veda_select_tiles without a workspace: scratch lives in a static
    per-device array inside the library (see include/veda.h)."""
    _check(lib().veda_select_tiles_noalloc(p.ref(), w_q.data_ptr(), w_k.data_ptr(), _ptr(idx_v), _ptr(idx_r),
                                           _stream(stream)), "veda_select_tiles_noalloc")


def block_sparse_attn(p: Problem, idx_v, idx_r, out, lse, ws, stream=None) -> None:
    _check(lib().veda_block_sparse_attn(p.ref(), _ptr(idx_v), _ptr(idx_r), out.data_ptr(), _ptr(lse),
                                        ws.data_ptr(), ws.numel(), _stream(stream)), "veda_block_sparse_attn")


def dense_query_attn(p: Problem, q_rows, out, lse, ws, stream=None) -> None:
    """q_rows [B, n_rows, H, d] (problem dtype, device) attend to every token
    of every segment of p; out like q_rows, lse [B, H, n_rows] fp32 or None."""
    B, n, H, d = q_rows.shape
    if (B, H, d) != (p.B, p.H, p.d) or q_rows.dtype != p.dtype or q_rows.stride(3) != 1:
        raise ValueError("q_rows must be [B, n_rows, H, d] of the problem's dtype, d contiguous")
    sb, st, sh, _ = q_rows.stride()
    _check(lib().veda_dense_query_attn(p.ref(), q_rows.data_ptr(), n, sb, st, sh, out.data_ptr(), _ptr(lse),
                                       ws.data_ptr(), ws.numel(), _stream(stream)), "veda_dense_query_attn")


def attn_host_buffer(p: Problem, heads_per_group: int, device=None) -> torch.Tensor:
    """The device buffer veda_attn_host needs for problem p (host tensors),
    with its status block initialised."""
    n = ctypes.c_size_t()
    _check(lib().veda_attn_host_buffer_size(p.ref(), heads_per_group, ctypes.byref(n)), "veda_attn_host_buffer_size")
    buf = torch.empty(n.value, dtype=torch.uint8, device=device or torch.device("cuda"))
    _check(lib().veda_workspace_init(buf.data_ptr(), buf.numel(), None), "veda_workspace_init")
    return buf


def attn_host(p: Problem, w_q, w_k, idx_v, idx_r, out, lse, heads_per_group: int, dev_buf, stream=None) -> None:
    """veda_attn on host tensors (p built from host tensors), copies pipelined
    with the compute over head groups."""
    _check(lib().veda_attn_host(p.ref(), w_q.data_ptr(), w_k.data_ptr(), _ptr(idx_v), _ptr(idx_r), out.data_ptr(),
                                _ptr(lse), heads_per_group, dev_buf.data_ptr(), dev_buf.numel(), _stream(stream)),
           "veda_attn_host")


def attn(p: Problem, w_q, w_k, idx_v, idx_r, out, lse, ws, stream=None) -> None:
    _check(lib().veda_attn(p.ref(), w_q.data_ptr(), w_k.data_ptr(), _ptr(idx_v), _ptr(idx_r), out.data_ptr(),
                           _ptr(lse), ws.data_ptr(), ws.numel(), _stream(stream)), "veda_attn")


def pool_project(p: Problem, w_q, w_k, ws, stream=None) -> None:
    _check(lib().veda_pool_project(p.ref(), w_q.data_ptr(), w_k.data_ptr(), ws.data_ptr(), ws.numel(),
                                   _stream(stream)), "veda_pool_project")


def score_tiles(p: Problem, ws, stream=None) -> None:
    _check(lib().veda_score_tiles(p.ref(), ws.data_ptr(), ws.numel(), _stream(stream)), "veda_score_tiles")


def topk_tiles(p: Problem, idx_v, idx_r, ws, stream=None) -> None:
    _check(lib().veda_topk_tiles(p.ref(), _ptr(idx_v), _ptr(idx_r), ws.data_ptr(), ws.numel(),
                                 _stream(stream)), "veda_topk_tiles")


def score_topk_tiles(p: Problem, idx_v, idx_r, ws, stream=None) -> None:
    """Steps 2-3: tensor-core scores, then the top-k (on chip with
    VEDA_FLAG_ONCHIP_SELECTION; SIMT scores with VEDA_FLAG_UNFUSED_SELECTION)."""
    _check(lib().veda_score_topk_tiles(p.ref(), _ptr(idx_v), _ptr(idx_r), ws.data_ptr(), ws.numel(),
                                       _stream(stream)), "veda_score_topk_tiles")


def fallback_rows(p: Problem, ws, ref: bool = False) -> torch.Tensor:
    """Row ids the last fused selection left to the exact step-3 kernel."""
    ptr = ctypes.c_void_p()
    ld = ctypes.c_int64()
    _check(lib().veda_workspace_view(p.ref(), ws.data_ptr(), ws.numel(), 6 if ref else 5, ctypes.byref(ptr),
                                     ctypes.byref(ld)), "veda_workspace_view")
    off = ptr.value - ws.data_ptr()
    count = int(ws[off:off + 4].view(torch.int32).item())
    return ws[off + 4:off + 4 + 4 * count].view(torch.int32).clone()


def workspace_view(p: Problem, ws, which: int) -> torch.Tensor:
    """Copy-free view of a workspace region as a torch tensor (device)."""
    ptr = ctypes.c_void_p()
    ld = ctypes.c_int64()
    _check(lib().veda_workspace_view(p.ref(), ws.data_ptr(), ws.numel(), which, ctypes.byref(ptr),
                                     ctypes.byref(ld)), "veda_workspace_view")
    n_rows_tiles = p.n_ref_tiles if which == 2 else p.n_q_tiles
    shape = (p.B, p.H, n_rows_tiles, ld.value)
    off = ptr.value - ws.data_ptr()
    nbytes = 4 * p.B * p.H * n_rows_tiles * ld.value
    return ws[off:off + nbytes].view(torch.float32).view(shape)


def check_status(ws, stream=None) -> int:
    """Synchronise the stream and return (and clear) the sticky device status."""
    return lib().veda_check_status(ws.data_ptr(), _stream(stream))


# ---------------------------------------------------------------------------
# selector artifacts (host)
# ---------------------------------------------------------------------------

# The published competition layout: 100 float16 tensors (Q and K projections
# of 50 layers), each (56, 384, 128), at most 560,000,000 bytes.
PUBLISHED_LAYOUT = {"n_tensors": 100, "shape": (56, 384, 128), "max_file_bytes": 560_000_000}


class Selector:
    """A selector artifact read by libveda: names, dtypes, shapes, metadata, and
    tensors converted to fp32 or bf16 (host torch tensors)."""

    def __init__(self, path: str):
        h = ctypes.c_void_p()
        _check(lib().veda_selector_open(os.fsencode(path), ctypes.byref(h)), "veda_selector_open")
        self._h = h

    def close(self) -> None:
        if self._h:
            lib().veda_selector_close(self._h)
            self._h = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def check(self, n_tensors: int, shape, max_file_bytes: int = 0, required_meta_key: Optional[str] = None):
        arr = (ctypes.c_int64 * len(shape))(*shape)
        key = required_meta_key.encode() if required_meta_key is not None else None
        _check(lib().veda_selector_check(self._h, n_tensors, arr, len(shape), max_file_bytes, key),
               "veda_selector_check")

    def check_published(self, hotkey_key: Optional[str] = None) -> None:
        """The competition layout (hotkey_key: the metadata key that must name the hotkey)."""
        self.check(PUBLISHED_LAYOUT["n_tensors"], PUBLISHED_LAYOUT["shape"], PUBLISHED_LAYOUT["max_file_bytes"],
                   hotkey_key)

    def __len__(self) -> int:
        return lib().veda_selector_count(self._h)

    def info(self, i: int):
        name, dt, nd = ctypes.c_char_p(), ctypes.c_char_p(), ctypes.c_int32()
        shape = (ctypes.c_int64 * 8)()
        _check(lib().veda_selector_info(self._h, i, ctypes.byref(name), ctypes.byref(dt), ctypes.byref(nd), shape),
               "veda_selector_info")
        return name.value.decode(), dt.value.decode(), tuple(shape[k] for k in range(nd.value))

    def names(self):
        return [self.info(i)[0] for i in range(len(self))]

    def metadata(self, key: str) -> Optional[str]:
        v = lib().veda_selector_metadata(self._h, key.encode())
        return None if v is None else v.decode()

    def read(self, name: str, dtype=torch.bfloat16, scale: float = 1.0) -> torch.Tensor:
        idx = ctypes.c_int32()
        _check(lib().veda_selector_find(self._h, name.encode(), ctypes.byref(idx)), "veda_selector_find")
        _, _, shape = self.info(idx.value)
        if dtype not in (torch.float32, torch.bfloat16):
            raise ValueError("dtype must be float32 or bfloat16")
        out = torch.empty(shape, dtype=dtype)
        _check(lib().veda_selector_read(self._h, idx.value, VEDA_F32 if dtype == torch.float32 else VEDA_BF16,
                                        float(scale), out.data_ptr(), out.numel() * out.element_size()),
               "veda_selector_read")
        return out
