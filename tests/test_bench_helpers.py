"""Host-side helpers of bench.py (CPU): the measured attention DRAM traffic
is keyed by real workload shapes, and the oracle baseline's fixed sample of
(b, h, query tile) units covers the first and the last (padded) tile."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def test_attention_traffic_is_keyed_by_real_workloads():
    assert bench.ATTN_TRAFFIC, "no measured traffic"
    for (name, heads, budget), traffic in bench.ATTN_TRAFFIC.items():
        w = workloads.get(name)
        assert (w.H, w.budget_video) == (heads, budget), name
        # DRAM traffic of a launch whose inputs exceed L2 cannot fall below
        # reading Q, K, V once and writing O once
        algorithmic = 4 * w.B * w.n_video * w.H * w.d * 2
        assert traffic >= 0.9 * algorithmic, (name, traffic, algorithmic)


def test_oracle_sample_covers_first_and_last_tile():
    for name in ("t2v_5.17s", "t2v_14.38s", "r2va_5.17s", "tiny"):
        w = workloads.get(name)
        units = bench.oracle_units(w)
        total = w.B * w.H * w.n_q_tiles
        assert len(units) >= min(64, total)
        assert len(set(units)) == len(units)
        assert units[0] == (0, 0, 0)
        assert units[1] == (w.B - 1, w.H - 1, w.n_q_tiles - 1)
        for b, h, i in units:
            assert 0 <= b < w.B and 0 <= h < w.H and 0 <= i < w.n_q_tiles
        assert bench.oracle_units(w) == units   # fixed: both arms time the same sample


def test_head_split_covers_every_head_once():
    for H in (2, 32, 40):
        for n in range(1, 9):
            if n > H:
                continue
            ranges = [bench.head_range(H, n, r) for r in range(n)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            for (a0, a1), (b0, _) in zip(ranges, ranges[1:]):
                assert a1 == b0            # contiguous, no gap, no overlap
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_head_slice_is_a_strided_view():
    import torch
    B, N, H, d, r = 1, 6, 4, 8, 2
    g = {"q": torch.randn(B, N, H, d), "k": torch.randn(B, N, H, d), "w_q": torch.randn(H, d, r)}
    s = bench.head_slice(g, 1, 3)
    assert s["q"].shape == (B, N, 2, d) and s["w_q"].shape == (2, d, r)
    assert s["q"].data_ptr() == g["q"][:, :, 1].data_ptr()      # a view, no copy
    assert s["q"].stride() == g["q"].stride()                    # token stride H * d kept
    assert torch.equal(s["k"], g["k"][:, :, 1:3]) and torch.equal(s["w_q"], g["w_q"][1:3])
