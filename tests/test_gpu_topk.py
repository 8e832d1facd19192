"""GPU parity of the fixed-budget top-k on crafted score rows.

The selector projections in the workspace are overwritten with small
integers, so every tile score q̂_i·k̂_j is an exact integer in fp32 and in the
oracle's fp64; the device scores and keeps tiles (veda_score_tiles +
veda_topk_tiles) and the kept sets must equal the oracle's bit for bit.  The
rows are chosen to reach every branch of the selection: heavy ties at the
k-th score (lowest index wins), rows sorted up and down, rows whose strided
sample sits far below or far above the rest of the row (so the bracketed
candidate list overflows or comes up short and the whole-row select runs),
short rows that are not sampled, budget 1 and budget = every tile, and row
lengths with a ragged tail past each 1024-key chunk.
"""
import numpy as np
import pytest
import torch

import learned_block_sparse_pool_b200 as veda

pytestmark = pytest.mark.gpu

T, D, R, H = 64, 64, 4, 2


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from learned_block_sparse_pool_b200 import build
    build.build()
    return torch.device("cuda:0")


def sample_positions(n):
    # the strided positions the device samples a row at (256 of them)
    return np.array([(m * n) // 256 for m in range(256)], np.int64)


def columns(kind, n):
    """(s, t): per key tile integers; the score of row i is s + a_i * t."""
    j = np.arange(n)
    if kind == "ties":
        return j % 3, (j * 7) % 5
    if kind == "sorted":
        return j, -2 * j
    if kind == "sample_low":            # sampled keys far below the rest
        s = np.full(n, 1000)
        s[sample_positions(n)] = 0
        return s, j % 2
    if kind == "sample_high":           # sampled keys far above the rest
        s = np.zeros(n, np.int64)
        s[sample_positions(n)] = 1000
        return s, j % 2
    if kind == "equal":
        return np.zeros(n, np.int64), np.zeros(n, np.int64)
    if kind == "random":
        rng = np.random.default_rng(n)
        return rng.integers(-500, 500, n), rng.integers(-3, 4, n)
    raise ValueError(kind)


def run_case(dev, oracle_mod, n, k, kind):
    N = n * T
    x = torch.empty((1, N, H, D), dtype=torch.float32, device=dev)
    p = veda.Problem(x, x, x, tile=T, r=R, budget=k)
    ws = veda.workspace(p)
    s, t = columns(kind, n)
    nq = p.n_q_tiles
    assert nq == n
    a = (np.arange(nq) % 4) - 1                          # row multipliers -1, 0, 1, 2
    qhat = np.zeros((1, H, nq, R))
    khat = np.zeros((1, H, n, R))
    for h in range(H):
        qhat[0, h, :, 0] = 1.0
        qhat[0, h, :, 1] = a if h == 0 else a[::-1]
        khat[0, h, :, 0] = s
        khat[0, h, :, 1] = t
    veda.workspace_view(p, ws, 0)[..., :R].copy_(torch.from_numpy(qhat).float())
    veda.workspace_view(p, ws, 1)[..., :R].copy_(torch.from_numpy(khat).float())
    veda.score_tiles(p, ws)
    iv, _ = veda.alloc_indices(p)
    veda.topk_tiles(p, iv, None, ws)
    assert veda.check_status(ws) == 0
    want, _, _ = oracle_mod.select(qhat, khat, k)
    got = iv.cpu().numpy()
    bad = np.argwhere((got != want).any(axis=-1))
    assert bad.size == 0, f"{kind} n={n} k={k}: {len(bad)} rows differ, first {bad[0]}: " \
                          f"got {got[tuple(bad[0])][:12]} want {want[tuple(bad[0])][:12]}"


@pytest.mark.parametrize("kind", ["ties", "sorted", "sample_low", "sample_high", "equal", "random"])
@pytest.mark.parametrize("n,k", [(977, 98), (2741, 138), (1922, 193), (300, 8), (200, 17), (1025, 300)])
def test_topk_crafted_rows(dev, oracle_mod, kind, n, k):
    run_case(dev, oracle_mod, n, k, kind)


@pytest.mark.parametrize("n", [63, 977, 2741])
@pytest.mark.parametrize("kind", ["ties", "random"])
def test_topk_budget_extremes(dev, oracle_mod, n, kind):
    for k in (1, n - 1, n):
        run_case(dev, oracle_mod, n, k, kind)
