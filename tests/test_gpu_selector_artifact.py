"""Selector artifact -> tile selection, on the GPU.

The trained selector projections ship as a safetensors file of float16
tensors (tao.media, "Affine launches MiniMax-H3 video studio...", section
"How the SN120 Competition Works"); the R2VA predictor is stored in FP8 and
dequantised to BF16 at load (veyrul.com, "Veda R2VA for MiniMax-H3", second
paragraph).  Here an F16 artifact and an FP8 (E4M3, with a stated per-tensor
scale) artifact holding per-head [H, d, r] query and key projections are
written byte by byte, read back with the library's reader (veda_selector_*),
and the weights it returns drive veda_select_tiles; the kept tiles are
compared with the oracle's on the same dequantised weights.
"""
import numpy as np
import pytest
import torch

import learned_block_sparse_pool_b200 as veda
import workloads
from parity import assert_selection, compare_selection
from test_selector_io import write_st

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from learned_block_sparse_pool_b200 import build
    build.build()
    return torch.device("cuda:0")


def _workload():
    # 6 frames of 48 x 84 = 24,192 tokens = 189 tiles, 4 heads, 20 kept
    return workloads.small("t2v_5.17s", frames=6, Y=48, X=84, H=4, budget_video=20, dense=(("text", 128),))


def _select_and_compare(oracle_mod, w, inp, wq, wk, dev, what):
    g = {k: v.to(dev) for k, v in inp.items()}
    p = veda.Problem(g["q"], g["k"], g["v"], tile=w.T, r=w.r, budget=w.budget_video,
                     k_dense=g["k_dense"], v_dense=g["v_dense"])
    ws = veda.workspace(p)
    iv, _ = veda.alloc_indices(p)
    veda.select_tiles(p, wq.to(dev), wk.to(dev), iv, None, ws)
    assert veda.check_status(ws) == 0
    ref = dict(inp, w_q=wq, w_k=wk)
    sel = oracle_mod.select_tiles(ref, w.T, w.budget_video)
    rep = compare_selection(oracle_mod, iv.cpu().numpy(), sel["idx_v"], sel["kth_v"], sel["qhat"], sel["khat"])
    assert_selection(rep, what)


def test_f16_artifact_drives_selection(dev, oracle_mod, tmp_path):
    w = _workload()
    inp = workloads.make_inputs(w)
    shape = tuple(inp["w_q"].shape)                      # (H, d, r) = (4, 128, 64)
    q16 = inp["w_q"].float().numpy().astype(np.float16)  # the weights as an fp16 artifact
    k16 = inp["w_k"].float().numpy().astype(np.float16)
    path = write_st(tmp_path / "selector.safetensors",
                    [("layers.0.q_proj", "F16", shape, q16.tobytes()), ("layers.0.k_proj", "F16", shape, k16.tobytes())],
                    meta={"hotkey": "5FtestHotkey"})
    with veda.Selector(str(path)) as s:
        s.check(2, shape, max_file_bytes=0, required_meta_key="hotkey")
        wq = s.read("layers.0.q_proj", torch.bfloat16)
        wk = s.read("layers.0.k_proj", torch.bfloat16)
    # the reader's fp16 -> bf16 conversion: exact widening, then round to nearest even
    for got, a16 in ((wq, q16), (wk, k16)):
        want = torch.from_numpy(a16.astype(np.float32)).to(torch.bfloat16)
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    _select_and_compare(oracle_mod, w, inp, wq, wk, dev, "F16 artifact")


def test_fp8_artifact_with_scale_drives_selection(dev, oracle_mod, tmp_path):
    w = _workload()
    inp = workloads.make_inputs(w)
    shape = tuple(inp["w_q"].shape)
    scale = 2.0 ** -6          # stated per-tensor scale: stored code x scale = weight
    q8 = (inp["w_q"].float() / scale).to(torch.float8_e4m3fn)
    k8 = (inp["w_k"].float() / scale).to(torch.float8_e4m3fn)
    path = write_st(tmp_path / "predictor_fp8.safetensors",
                    [("q_proj", "F8_E4M3", shape, q8.view(torch.uint8).numpy().tobytes()),
                     ("k_proj", "F8_E4M3", shape, k8.view(torch.uint8).numpy().tobytes())])
    with veda.Selector(str(path)) as s:
        wq = s.read("q_proj", torch.bfloat16, scale=scale)
        wk = s.read("k_proj", torch.bfloat16, scale=scale)
    # e4m3 codes times a power of two are bf16 values: dequantisation is exact
    assert torch.equal(wq, (q8.float() * scale).to(torch.bfloat16))
    assert torch.equal(wk, (k8.float() * scale).to(torch.bfloat16))
    _select_and_compare(oracle_mod, w, inp, wq, wk, dev, "FP8 artifact")
