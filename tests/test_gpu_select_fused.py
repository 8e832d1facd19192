"""Tile selection on the tensor cores against the CPU oracle, in both of its
forms: tensor-core scores written out and selected by the warp-per-row top-k
(the default of veda_select_tiles), and the on-chip selection that writes no
score matrix (VEDA_FLAG_ONCHIP_SELECTION).

  * reduced workloads with several 64-tile chunks per row (ragged last chunk
    and last block of query tiles, a reference segment), budgets 1, ~10 %,
    n - 1 and n;
  * crafted integer scores through the whole pipeline (exact in every
    precision): heavy ties, constant rows, sorted rows, a single winner;
  * rows the on-chip selection cannot finish (all scores equal) go to the
    exact step-3 kernel and still match;
  * the tensor-core and the fp32 SIMT score paths agree outside the tie band,
    and few rows of a realistic problem need the on-chip fallback.
"""
import numpy as np
import pytest
import torch

import learned_block_sparse_pool_b200 as veda
import workloads
from learned_block_sparse_pool_b200 import binding as B
from parity import assert_selection, compare_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from learned_block_sparse_pool_b200 import build
    build.build()
    return torch.device("cuda:0")


def _problem(w, g, budget=None, budget_ref=None, flags=0):
    return veda.Problem(g["q"], g["k"], g["v"], tile=w.T, r=w.r,
                        budget=w.budget_video if budget is None else budget,
                        k_ref=g.get("k_ref"), v_ref=g.get("v_ref"),
                        budget_ref=(w.budget_ref if budget_ref is None else budget_ref) if "k_ref" in g else 0,
                        k_dense=g.get("k_dense"), v_dense=g.get("v_dense"), flags=flags)


def _select(p, g, flags_problem=None):
    ws = veda.workspace(p)
    iv, ir = veda.alloc_indices(p)
    veda.select_tiles(p, g["w_q"], g["w_k"], iv, ir, ws)
    assert veda.check_status(ws) == 0
    return ws, iv, ir


# 10 frames of 48 x 84 = 40,320 tokens = 315 tiles (3 chunks, the last of 59);
# reference 5 frames = 158 tiles; 4 heads
MULTI = dict(frames=10, Y=48, X=84, H=4, dense=(("text", 200),))


ONCHIP = B.VEDA_FLAG_ONCHIP_SELECTION


@pytest.mark.parametrize("flags", [0, ONCHIP], ids=["tensor_scores", "onchip"])
@pytest.mark.parametrize("budget", [1, 32, 314, 315])
def test_fused_selection_several_chunks(dev, oracle_mod, budget, flags):
    w = workloads.small("r2va_5.17s", ref_frames=5, budget_video=budget, budget_ref=min(budget, 158), **MULTI)
    inp = workloads.make_inputs(w)
    g = {k: v.to(dev) for k, v in inp.items()}
    p = _problem(w, g, flags=flags)
    ws, iv, ir = _select(p, g)
    sel = oracle_mod.select_tiles(inp, w.T, w.budget_video, w.budget_ref)
    rep = compare_selection(oracle_mod, iv.cpu().numpy(), sel["idx_v"], sel["kth_v"], sel["qhat"], sel["khat"])
    assert_selection(rep, f"fused k={budget} video")
    rep = compare_selection(oracle_mod, ir.cpu().numpy(), sel["idx_r"], sel["kth_r"], sel["qhat"], sel["khat_r"])
    assert_selection(rep, f"fused k={budget} reference")
    n_rows = w.B * w.H * w.n_q_tiles
    fb = len(veda.fallback_rows(p, ws))
    if flags == 0:
        assert fb == 0
    else:   # very small budgets give narrow bands that pass A's approximate scores can miss
        assert fb <= (n_rows // 6 if budget <= 2 else max(2, n_rows // 50)), fb


def _crafted(dev, x, y, a, H=2, T=128):
    """Q, K whose projections are q_i = (1, a_i, 0, ...) and k_j = (x_j, y_j, 0, ...)
    exactly (every token of a tile equal, W = identity on the first 64
    channels), so s_ij = x_j + a_i y_j: small integers, exact in every
    precision."""
    n = len(x)
    d, r = 128, 64
    qt = torch.zeros(1, n, H, d)
    qt[:, :, :, 0] = 1.0
    qt[0, :, :, 1] = torch.tensor(a, dtype=torch.float32)[:, None]
    kt = torch.zeros(1, n, H, d)
    kt[0, :, :, 0] = torch.tensor(x, dtype=torch.float32)[:, None]
    kt[0, :, :, 1] = torch.tensor(y, dtype=torch.float32)[:, None]
    q = qt.repeat_interleave(T, dim=1).to(torch.bfloat16)
    k = kt.repeat_interleave(T, dim=1).to(torch.bfloat16)
    v = torch.randn(1, n * T, H, d).to(torch.bfloat16)
    wmat = torch.zeros(H, d, r)
    wmat[:, :r, :] = torch.eye(r)
    wmat = wmat.to(torch.bfloat16)
    return {"q": q, "k": k, "v": v, "w_q": wmat, "w_k": wmat.clone()}


@pytest.mark.parametrize("flags", [0, ONCHIP], ids=["tensor_scores", "onchip"])
@pytest.mark.parametrize("case", ["ties", "constant", "sorted", "single_winner"])
def test_fused_selection_crafted_integer_scores(dev, oracle_mod, case, flags):
    rng = np.random.default_rng(3)
    n = 300
    if case == "ties":
        x, y = rng.integers(-3, 4, n), rng.integers(-2, 3, n)
    elif case == "constant":
        x, y = np.full(n, 5), np.zeros(n, int)
    elif case == "sorted":
        x, y = np.arange(n) % 97, np.arange(n) // 97
    else:
        x, y = np.zeros(n, int), np.zeros(n, int)
        x[137] = 9
    a = rng.integers(-2, 3, n)
    inp = _crafted(dev, x, y, a)
    g = {k_: v_.to(dev) for k_, v_ in inp.items()}
    for k in (1, 7, 30, 150, 299):
        p = veda.Problem(g["q"], g["k"], g["v"], tile=128, r=64, budget=k, flags=flags)
        ws, iv, _ = _select(p, g)
        qhat = oracle_mod.project(oracle_mod.pool(inp["q"], 128), inp["w_q"])
        khat = oracle_mod.project(oracle_mod.pool(inp["k"], 128), inp["w_k"])
        idx, _, _ = oracle_mod.select(qhat, khat, k)
        assert np.array_equal(iv.cpu().numpy(), idx), (case, k)


def test_rows_left_to_the_exact_kernel(dev, oracle_mod):
    """All query projections zero: every score is 0, no band can be narrowed,
    and every row goes to the step-3 kernel; the kept tiles are 0 .. k-1."""
    w = workloads.small("t2v_5.17s", budget_video=20, **MULTI)
    inp = workloads.make_inputs(w)
    inp["q"] = torch.zeros_like(inp["q"])
    g = {k: v.to(dev) for k, v in inp.items()}
    p = _problem(w, g, flags=ONCHIP)
    ws, iv, _ = _select(p, g)
    fb = veda.fallback_rows(p, ws)
    assert len(fb) == w.B * w.H * w.n_q_tiles
    assert (iv.cpu().numpy() == np.arange(20)).all()


def test_tensor_simt_and_onchip_paths_agree(dev, oracle_mod):
    w = workloads.small("portrait_10.13s", frames=12, Y=84, X=48, H=4, budget_video=40, dense=())
    inp = workloads.make_inputs(w)
    g = {k: v.to(dev) for k, v in inp.items()}
    _, iv_t, _ = _select(_problem(w, g), g)
    _, iv_s, _ = _select(_problem(w, g, flags=B.VEDA_FLAG_UNFUSED_SELECTION), g)
    _, iv_o, _ = _select(_problem(w, g, flags=ONCHIP), g)
    sel = oracle_mod.select_tiles(inp, w.T, w.budget_video)
    for iv, what in ((iv_t, "tensor scores"), (iv_s, "simt scores"), (iv_o, "on-chip")):
        rep = compare_selection(oracle_mod, iv.cpu().numpy(), sel["idx_v"], sel["kth_v"], sel["qhat"], sel["khat"])
        assert_selection(rep, what)
    # the same scores, bit for bit: the two tensor-core paths keep the same tiles
    assert torch.equal(iv_t, iv_o)
    differ = (iv_t != iv_s).any(dim=-1).sum().item()
    assert differ <= 5, differ
