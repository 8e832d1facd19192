"""veda_attn_host (host buffers, copies pipelined over head groups) against
the device-resident veda_attn on the same inputs: every head is independent,
so the outputs, LSE and kept tiles must match bit for bit, for any grouping
of the heads (one head per group, a short last group, all heads in one)."""
import pytest
import torch

import learned_block_sparse_pool_b200 as veda
import workloads
from test_gpu_parity import REDUCED, make_problem, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from learned_block_sparse_pool_b200 import build
    build.build()
    return torch.device("cuda:0")


def run_both(w, inp, dev, groups):
    g = to_dev(inp, dev)
    p = make_problem(w, g)
    ws = veda.workspace(p)
    iv, ir = veda.alloc_indices(p)
    out, lse = veda.alloc_output(p, with_lse=True)
    veda.attn(p, g["w_q"], g["w_k"], iv, ir, out, lse, ws)
    assert veda.check_status(ws) == 0
    host = {k: v.contiguous().pin_memory() for k, v in inp.items()}
    ph = make_problem(w, host)
    res = []
    for hpg in groups:
        buf = veda.attn_host_buffer(ph, hpg, dev)
        o_h = torch.full(out.shape, float("nan"), dtype=out.dtype).pin_memory()
        l_h = torch.full(lse.shape, float("nan"), dtype=torch.float32).pin_memory()
        iv_h = torch.full(iv.shape, -1, dtype=torch.int32).pin_memory()
        ir_h = torch.full(ir.shape, -1, dtype=torch.int32).pin_memory() if ir is not None else None
        veda.attn_host(ph, host["w_q"], host["w_k"], iv_h, ir_h, o_h, l_h, hpg, buf)
        torch.cuda.synchronize()
        assert veda.check_status(buf) == 0
        assert torch.equal(iv_h, iv.cpu()), hpg
        if ir is not None:
            assert torch.equal(ir_h, ir.cpu()), hpg
        assert torch.equal(o_h.view(torch.int16) if o_h.dtype == torch.bfloat16 else o_h,
                           out.cpu().view(torch.int16) if out.dtype == torch.bfloat16 else out.cpu()), hpg
        assert torch.equal(l_h, lse.cpu()), hpg
        res.append(hpg)
    return res


@pytest.mark.parametrize("name", ["t2v_ragged", "r2va_ragged"])
def test_host_call_matches_device_call(dev, name):
    w = REDUCED[name]()                      # 4 heads
    inp = workloads.make_inputs(w)
    assert run_both(w, inp, dev, [1, 3, 4, 16]) == [1, 3, 4, 16]


def test_host_call_batch_two(dev):
    """B = 2 with a reference segment: the head-range copies of every batch
    entry land in the right place, in and out."""
    w = REDUCED["r2va_ragged"]()
    w = workloads.small(w.name, **{**{f: getattr(w, f) for f in ("frames", "Y", "X", "dense", "budget_video",
                                                                  "ref_frames", "budget_ref")}, "H": 3, "B": 2})
    inp = workloads.make_inputs(w)
    assert run_both(w, inp, dev, [1, 2]) == [1, 2]


def test_host_call_full_size(dev):
    w = workloads.get("t2v_5.17s")
    inp = {k: v.cpu() for k, v in workloads.make_inputs(w, device=dev).items()}
    assert run_both(w, inp, dev, [8]) == [8]


def test_host_call_rejects_unpacked_inputs(dev):
    w = REDUCED["t2v_ragged"]()
    inp = workloads.make_inputs(w)
    bad = dict(inp)
    bad["q"] = inp["q"].permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)   # [B, N, H, d] view, not packed
    p = make_problem(w, bad)
    with pytest.raises(veda.VedaError) as e:
        veda.attn_host_buffer(p, 2, dev)
    assert e.value.status == veda.binding.VEDA_ERR_UNSUPPORTED
