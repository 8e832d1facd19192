"""C-ABI checks that need no GPU: the library loads, exports every function
include/veda.h declares, its structs have the layout a C compiler gives them,
and invalid arguments are rejected on the host with the documented codes."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import learned_block_sparse_pool_b200 as veda
from learned_block_sparse_pool_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "veda.h")


@pytest.fixture(scope="module")
def L():
    from learned_block_sparse_pool_b200 import build
    build.build()
    return veda.lib()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^VEDA_API\s+[\w\s\*]+?\b(veda_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (veda_\w+)", out))
    missing = set(declared_functions()) - exported
    assert not missing, missing
    for name in declared_functions():
        assert hasattr(L, name)


def test_struct_layout_matches_c_compiler(tmp_path):
    prog = tmp_path / "layout.c"
    prog.write_text("""
#include <stdio.h>
#include <stddef.h>
#include "veda.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(veda_segment), sizeof(veda_problem),
         offsetof(veda_problem, q), offsetof(veda_problem, q_stride_h), offsetof(veda_problem, video),
         offsetof(veda_problem, ref), offsetof(veda_problem, dense), offsetof(veda_segment, budget));
  return 0;
}
""")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    P, S = B.veda_problem, B.veda_segment
    want = [ctypes.sizeof(S), ctypes.sizeof(P), P.q.offset, P.q_stride_h.offset, P.video.offset,
            P.ref.offset, P.dense.offset, S.budget.offset]
    assert got == want


def _problem(**over):
    """A valid bf16 problem with fake (never dereferenced) device pointers."""
    p = B.veda_problem()
    p.B, p.H, p.d, p.tile, p.r = 1, 4, 128, 128, 64
    p.dtype = B.VEDA_BF16
    N, H, d = 1000, 4, 128
    p.q = 0x100000
    p.q_stride_b, p.q_stride_tok, p.q_stride_h = N * H * d, H * d, d
    for seg, base, n, budget in ((p.video, 0x200000, N, 3), (p.ref, 0x300000, 300, 2), (p.dense, 0x400000, 77, 0)):
        seg.k, seg.v = base, base + 0x80000
        seg.n_tokens = n
        seg.stride_b, seg.stride_tok, seg.stride_h = n * H * d, H * d, d
        seg.budget = budget
    for k, v in over.items():
        obj = p
        *path, last = k.split(".")
        for part in path:
            obj = getattr(obj, part)
        setattr(obj, last, v)
    return p


def _ws_size(L, p):
    n = ctypes.c_size_t(0)
    return L.veda_workspace_size(ctypes.byref(p), ctypes.byref(n)), n.value


def test_valid_problem_workspace_size(L):
    st, n = _ws_size(L, _problem())
    assert st == B.VEDA_OK
    nq, nr = 8, 3
    ld_v, ld_r = 32, 32
    BH, r = 4, 64
    # status block + qhat + khat + khat_ref + scores + scores_ref + the three
    # bf16 projection planes (q, k, k_ref: 3 x 64 columns) and of the 64
    # sampled key tiles (video, reference) + the two lists of
    # rows left to the exact top-k by the fused selection, each 256-aligned
    expect = 256
    for nbytes in (4 * BH * nq * r, 4 * BH * nq * r, 4 * BH * nr * r, 4 * BH * nq * ld_v, 4 * BH * nq * ld_r,
                   6 * BH * nq * 64, 6 * BH * nq * 64, 6 * BH * nr * 64, 6 * BH * 64 * 64, 6 * BH * 64 * 64,
                   4 * (1 + BH * nq), 4 * (1 + BH * nq)):
        expect += -(-nbytes // 256) * 256
    assert n == expect


@pytest.mark.parametrize("over,code", [
    ({"d": 96}, B.VEDA_ERR_UNSUPPORTED),
    ({"tile": 32}, B.VEDA_ERR_UNSUPPORTED),
    ({"r": 6}, B.VEDA_ERR_UNSUPPORTED),
    ({"r": 132}, B.VEDA_ERR_UNSUPPORTED),
    ({"B": 0}, B.VEDA_ERR_INVALID_ARG),
    ({"dtype": 7}, B.VEDA_ERR_INVALID_ARG),
    ({"flags": 16}, B.VEDA_ERR_INVALID_ARG),
    ({"softmax_scale": -1.0}, B.VEDA_ERR_INVALID_ARG),
    ({"softmax_scale": float("nan")}, B.VEDA_ERR_INVALID_ARG),
    ({"q": 0}, B.VEDA_ERR_INVALID_ARG),
    ({"q": 0x100008}, B.VEDA_ERR_INVALID_ARG),          # not 16-byte aligned
    ({"q_stride_tok": 4 * 128 + 4}, B.VEDA_ERR_INVALID_ARG),  # stride not a multiple of 16 bytes
    ({"video.budget": 0}, B.VEDA_ERR_INVALID_ARG),
    ({"video.budget": 9}, B.VEDA_ERR_INVALID_ARG),       # 1000 tokens = 8 tiles
    ({"video.n_tokens": 0}, B.VEDA_ERR_INVALID_ARG),
    ({"video.k": 0}, B.VEDA_ERR_INVALID_ARG),
    ({"ref.budget": 0}, B.VEDA_ERR_INVALID_ARG),
    ({"ref.budget": 4}, B.VEDA_ERR_INVALID_ARG),          # 300 tokens = 3 tiles
    ({"ref.v": 0}, B.VEDA_ERR_INVALID_ARG),
    ({"dense.budget": 1}, B.VEDA_ERR_INVALID_ARG),
    ({"dense.stride_h": 100}, B.VEDA_ERR_INVALID_ARG),
    ({"ref.n_tokens": 0, "ref.budget": 1}, B.VEDA_ERR_INVALID_ARG),
    ({"video.n_tokens": 128 * 4097, "video.stride_b": 0, "video.budget": 1}, B.VEDA_ERR_UNSUPPORTED),
])
def test_invalid_arguments_rejected_on_host(L, over, code):
    st, _ = _ws_size(L, _problem(**over))
    assert st == code, (over, B.status_string(st))


def test_test_hook_flags_are_accepted(L):
    for flags in (B.VEDA_FLAG_SIMT_ATTENTION, B.VEDA_FLAG_TEST_SHORT_WAITS, B.VEDA_FLAG_UNFUSED_SELECTION,
                  B.VEDA_FLAG_ONCHIP_SELECTION, 15):
        st, _ = _ws_size(L, _problem(flags=flags))
        assert st == B.VEDA_OK


def test_optional_segments_absent_is_valid(L):
    st, _ = _ws_size(L, _problem(**{"ref.n_tokens": 0, "ref.budget": 0, "dense.n_tokens": 0}))
    assert st == B.VEDA_OK


def test_null_problem_and_null_size(L):
    n = ctypes.c_size_t()
    assert L.veda_workspace_size(None, ctypes.byref(n)) == B.VEDA_ERR_INVALID_ARG
    p = _problem()
    assert L.veda_workspace_size(ctypes.byref(p), None) == B.VEDA_ERR_INVALID_ARG


def test_workspace_errors_before_any_launch(L):
    p = _problem()
    st, n = _ws_size(L, p)
    idx = 0x500000
    # NULL, misaligned and too-small workspaces are rejected without touching the device
    assert L.veda_select_tiles(ctypes.byref(p), 0x600000, 0x700000, idx, idx, None, n, None) == B.VEDA_ERR_WORKSPACE
    assert L.veda_select_tiles(ctypes.byref(p), 0x600000, 0x700000, idx, idx, 0x800010, n, None) == \
        B.VEDA_ERR_WORKSPACE
    assert L.veda_select_tiles(ctypes.byref(p), 0x600000, 0x700000, idx, idx, 0x800000, n - 1, None) == \
        B.VEDA_ERR_WORKSPACE
    assert L.veda_attn(ctypes.byref(p), 0x600000, 0x700000, idx, idx, 0x900000, None, None, n, None) == \
        B.VEDA_ERR_WORKSPACE
    assert L.veda_workspace_init(None, 256, None) == B.VEDA_ERR_WORKSPACE
    assert L.veda_check_status(0x800010, None) == B.VEDA_ERR_WORKSPACE


def test_index_and_output_arguments_checked(L):
    p = _problem()
    st, n = _ws_size(L, p)
    ws = 0x800000
    # reference present -> idx_ref required; output must be 16-byte aligned; lse 4-byte aligned
    assert L.veda_topk_tiles(ctypes.byref(p), 0x500000, None, ws, n, None) == B.VEDA_ERR_INVALID_ARG
    assert L.veda_topk_tiles(ctypes.byref(p), None, 0x500000, ws, n, None) == B.VEDA_ERR_INVALID_ARG
    assert L.veda_block_sparse_attn(ctypes.byref(p), 0x500000, 0x510000, 0x900008, None, ws, n, None) == \
        B.VEDA_ERR_INVALID_ARG
    assert L.veda_block_sparse_attn(ctypes.byref(p), 0x500000, 0x510000, 0x900000, 0xA00002, ws, n, None) == \
        B.VEDA_ERR_INVALID_ARG
    assert L.veda_attn(ctypes.byref(p), 0, 0x700000, 0x500000, 0x510000, 0x900000, None, ws, n, None) == \
        B.VEDA_ERR_INVALID_ARG
    q = _problem(**{"ref.n_tokens": 0, "ref.budget": 0})
    assert L.veda_topk_tiles(ctypes.byref(q), 0x500000, 0x510000, ws, n, None) == B.VEDA_ERR_INVALID_ARG


def test_dense_query_arguments_checked(L):
    p = _problem()
    st, n = _ws_size(L, p)
    ws, q, out = 0x800000, 0x900000, 0xA00000
    H, d = 4, 128
    ok = (q, 10, 10 * H * d, H * d, d, out, None, ws, n, None)

    def call(*a):
        return L.veda_dense_query_attn(ctypes.byref(p), *a)
    bad = [
        (0, 10, 10 * H * d, H * d, d, out, None, ws, n, None),            # no query rows
        (q + 8, 10, 10 * H * d, H * d, d, out, None, ws, n, None),        # misaligned rows
        (q, 0, 10 * H * d, H * d, d, out, None, ws, n, None),             # no rows
        (q, 10, 10 * H * d, H * d + 4, d, out, None, ws, n, None),        # stride not 16-byte
        (q, 10, 10 * H * d, H * d, d, out + 8, None, ws, n, None),        # misaligned output
        (q, 10, 10 * H * d, H * d, d, out, 0xB00002, ws, n, None),        # misaligned lse
    ]
    for a in bad:
        assert call(*a) == B.VEDA_ERR_INVALID_ARG, a
    assert call(q, 10, 10 * H * d, H * d, d, out, None, None, n, None) == B.VEDA_ERR_WORKSPACE
    q_bad = _problem(d=96)
    assert L.veda_dense_query_attn(ctypes.byref(q_bad), *ok) == B.VEDA_ERR_UNSUPPORTED


def test_host_call_buffer_and_arguments(L):
    """veda_attn_host: buffer size and the checks made before any CUDA call."""
    p = _problem()                      # packed [B, N, H, d] host layout, reference + dense present
    n1, n4 = B.ctypes.c_size_t(), B.ctypes.c_size_t()
    assert L.veda_attn_host_buffer_size(B.ctypes.byref(p), 1, B.ctypes.byref(n1)) == B.VEDA_OK
    assert L.veda_attn_host_buffer_size(B.ctypes.byref(p), 4, B.ctypes.byref(n4)) == B.VEDA_OK
    assert 256 < n1.value < n4.value    # status block + two slots; a slot grows with the group
    assert L.veda_attn_host_buffer_size(B.ctypes.byref(p), 9, B.ctypes.byref(n1)) == B.VEDA_OK
    assert n1.value == n4.value         # groups are capped at H heads
    assert L.veda_attn_host_buffer_size(B.ctypes.byref(p), 0, B.ctypes.byref(n1)) == B.VEDA_ERR_INVALID_ARG
    unpacked = _problem(q_stride_tok=4 * 128 * 2)
    assert L.veda_attn_host_buffer_size(B.ctypes.byref(unpacked), 2, B.ctypes.byref(n1)) == B.VEDA_ERR_UNSUPPORTED
    buf, w, idx, out = 0x10000000, 0x900000, 0x500000, 0xA00000

    def call(prob, *, dev_bytes=n4.value, dev=buf, o=out, wq=w):
        return L.veda_attn_host(B.ctypes.byref(prob), wq, w, None, None, o, None, 4, dev, dev_bytes, None)
    assert call(p, dev_bytes=n4.value - 1) == B.VEDA_ERR_WORKSPACE
    assert call(p, dev=buf + 16) == B.VEDA_ERR_WORKSPACE
    assert call(p, o=0) == B.VEDA_ERR_INVALID_ARG
    assert call(p, wq=0) == B.VEDA_ERR_INVALID_ARG
    assert call(unpacked) == B.VEDA_ERR_UNSUPPORTED


def test_workspace_view_bounds(L):
    p = _problem(**{"ref.n_tokens": 0, "ref.budget": 0})
    st, n = _ws_size(L, p)
    ptr, ld = ctypes.c_void_p(), ctypes.c_int64()
    assert L.veda_workspace_view(ctypes.byref(p), 0x800000, n, 0, ctypes.byref(ptr), ctypes.byref(ld)) == B.VEDA_OK
    assert ptr.value == 0x800000 + 256 and ld.value == 64
    assert L.veda_workspace_view(ctypes.byref(p), 0x800000, n, 2, ctypes.byref(ptr), ctypes.byref(ld)) == \
        B.VEDA_ERR_INVALID_ARG
    assert L.veda_workspace_view(ctypes.byref(p), 0x800000, n, 5, ctypes.byref(ptr), ctypes.byref(ld)) == B.VEDA_OK
    assert ld.value == 1 and 0x800000 < ptr.value < 0x800000 + n
    assert L.veda_workspace_view(ctypes.byref(p), 0x800000, n, 6, ctypes.byref(ptr), ctypes.byref(ld)) == \
        B.VEDA_ERR_INVALID_ARG
    assert L.veda_workspace_view(ctypes.byref(p), 0x800000, n, 7, ctypes.byref(ptr), ctypes.byref(ld)) == \
        B.VEDA_ERR_INVALID_ARG


def test_status_strings(L):
    for code, name in [(0, "VEDA_OK"), (-1, "VEDA_ERR_INVALID_ARG"), (-2, "VEDA_ERR_UNSUPPORTED"),
                       (-3, "VEDA_ERR_WORKSPACE"), (-4, "VEDA_ERR_CUDA"), (-5, "VEDA_ERR_TIMEOUT"),
                       (-6, "VEDA_ERR_BAD_INDEX"), (-7, "VEDA_ERR_FORMAT"), (-8, "VEDA_ERR_IO"),
                       (-99, "VEDA_ERR_UNKNOWN")]:
        assert B.status_string(code) == name


def test_c_program_uses_the_abi(L, tmp_path):
    """A plain C program linked against libveda.so: validation, sizing, status
    strings and the selector reader, with no Python in between."""
    exe = tmp_path / "abi_from_c"
    src = os.path.join(ROOT, "tests", "c", "abi_from_c.c")
    libdir = os.path.dirname(B.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-O1", "-I", os.path.join(ROOT, "include"), src, "-o", str(exe),
                    "-L", libdir, "-lveda", f"-Wl,-rpath,{libdir}"], check=True)
    res = subprocess.run([str(exe), str(tmp_path / "sel.safetensors")], capture_output=True, text=True)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stderr


NOALLOC_REJECT = r"""
import ctypes, sys
sys.path.insert(0, %r)
import learned_block_sparse_pool_b200 as veda
from learned_block_sparse_pool_b200 import binding as B
p = B.veda_problem()
p.B, p.H, p.d, p.tile, p.r = 1, 1, 128, 128, 64
p.dtype = B.VEDA_BF16
n = 4096 * 128                                    # 4096 key tiles: one head's scores exceed 64 MiB
p.q = 0x100000
p.q_stride_b, p.q_stride_tok, p.q_stride_h = n * 128, 128, 128
p.video.k, p.video.v = 0x200000, 0x300000
p.video.n_tokens = n
p.video.stride_b, p.video.stride_tok, p.video.stride_h = n * 128, 128, 128
p.video.budget = 8
print(veda.lib().veda_select_tiles_noalloc(ctypes.byref(p), 0x400000, 0x500000, 0x600000, None, None))
"""


def test_noalloc_rejects_a_head_that_does_not_fit_without_a_device(L):
    """The static scratch array holds 64 MiB; a single head with 4096 key
    tiles needs more, and the call must refuse it on the host.  Run with no
    device visible, so the fake pointers can never reach a kernel."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "-c", NOALLOC_REJECT % ROOT], env=env, capture_output=True, text=True,
                         check=True, timeout=300)
    assert int(res.stdout.strip().splitlines()[-1]) == B.VEDA_ERR_WORKSPACE
