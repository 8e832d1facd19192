"""veda_select_tiles_noalloc: tile selection for callers that cannot
allocate device memory at call time (a serving engine with a pre-planned
memory pool, a plugin enqueue hook that must not allocate, a loop that cannot
take cudaMalloc's device synchronisation).  Its scratch is a static per-device
array inside the library, so the caller passes only inputs and outputs.

Checked through the C ABI against veda_select_tiles (the workspace entry
point) running the same kernels (VEDA_FLAG_UNFUSED_SELECTION): the kept tiles
must be identical, on two calls in a row (the static
array keeps the previous call's contents, which must not leak into the next
result).  pytest collects this file last (its name sorts last), so a run that
stops at the first failure has run every other test before this one; the
tests pass either way, alone in a fresh process or after the others.
"""
import pytest
import torch

import learned_block_sparse_pool_b200 as veda
import workloads
from learned_block_sparse_pool_b200 import binding as B

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from learned_block_sparse_pool_b200 import build
    build.build()
    return torch.device("cuda:0")


def _problem(w, g, flags=0):
    return veda.Problem(g["q"], g["k"], g["v"], tile=w.T, r=w.r, budget=w.budget_video,
                        k_ref=g.get("k_ref"), v_ref=g.get("v_ref"),
                        budget_ref=w.budget_ref if "k_ref" in g else 0,
                        k_dense=g.get("k_dense"), v_dense=g.get("v_dense"), flags=flags)


def _compare_two_calls(w, g):
    # the workspace entry point on the same kernels (fp32 SIMT scores, then
    # the warp-per-row top-k), so the kept tiles must be identical
    p = _problem(w, g, flags=B.VEDA_FLAG_UNFUSED_SELECTION)
    ws = veda.workspace(p)
    iv, ir = veda.alloc_indices(p)
    veda.select_tiles(p, g["w_q"], g["w_k"], iv, ir, ws)
    assert veda.check_status(ws) == 0
    for call in range(2):
        jv, jr = veda.alloc_indices(p)
        jv.fill_(-7)
        if jr is not None:
            jr.fill_(-7)
        veda.select_tiles_noalloc(p, g["w_q"], g["w_k"], jv, jr)
        torch.cuda.synchronize()
        assert torch.equal(jv, iv), f"call {call}: video tiles differ"
        if ir is not None:
            assert torch.equal(jr, ir), f"call {call}: reference tiles differ"


def test_noalloc_matches_workspace_entry_full_clip(dev):
    """5.17 s clip (32 heads, 977 tiles): one head needs 4,376,960 bytes of
    scratch (q-hat, k-hat and the 977 x 992 score rows), so the 64 MiB array
    holds 15 heads and the call runs in three head groups (15 + 15 + 2)."""
    w = workloads.get("t2v_5.17s")
    _compare_two_calls(w, workloads.make_inputs(w, device=dev))


def test_noalloc_matches_workspace_entry_batch_and_reference(dev):
    w = workloads.small("r2va_5.17s", B=2, frames=3, Y=16, X=21, H=4, ref_frames=1, budget_video=3,
                        budget_ref=2, dense=(("text", 200),))
    _compare_two_calls(w, {k: v.to(dev) for k, v in workloads.make_inputs(w).items()})


def test_noalloc_rejects_a_head_that_does_not_fit(dev):
    """4096 key tiles: one head's scores alone exceed the static array, so the
    call returns VEDA_ERR_WORKSPACE before launching anything.  The problem
    points at real device tensors of its full size, so even a call that went
    further would read valid memory."""
    n = 4096 * 128
    q = torch.zeros((1, n, 1, 128), dtype=torch.bfloat16, device=dev)
    k = torch.zeros_like(q)
    v = torch.zeros_like(q)
    w = torch.zeros((1, 128, 64), dtype=torch.bfloat16, device=dev)
    p = veda.Problem(q, k, v, tile=128, r=64, budget=8)
    iv, _ = veda.alloc_indices(p)
    st = veda.lib().veda_select_tiles_noalloc(p.ref(), w.data_ptr(), w.data_ptr(), iv.data_ptr(), None,
                                              torch.cuda.current_stream().cuda_stream)
    assert st == B.VEDA_ERR_WORKSPACE
