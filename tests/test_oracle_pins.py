"""Pins for the CPU oracle: checks against what the mathematics fixes, not
against the oracle itself.

  * a hand-derived worked example (tests/golden/hand_example.json),
  * closed forms (tile means of arithmetic series; unit projection matrices),
  * invariants (pooling commutes with a linear projection; softmax of
    all-ones values is 1; every kept score >= every dropped score),
  * brute force over all k-subsets on tiny integer-score rows,
  * special cases that reduce to textbook routines: at a budget of every tile
    the restricted attention is dense softmax attention, and for any budget it
    equals dense attention under the boolean mask built from the kept tiles
    (torch's fp64 scaled_dot_product_attention / logsumexp / softmax).

All of these run on the CPU (no GPU marker).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bnhd(rows, dtype=torch.float32):
    """[[...d], ...] tokens of one head -> [1, N, 1, d] tensor."""
    return torch.tensor(rows, dtype=torch.float64).to(dtype)[None, :, None, :].contiguous()


# ---------------------------------------------------------------------------
# the hand-worked example
# ---------------------------------------------------------------------------

def _hand():
    with open(os.path.join(GOLDEN, "hand_example.json")) as f:
        return json.load(f)


def _eval(expr):
    if expr == "nan":
        return float("nan")
    return eval(expr, {"E": math.e, "log": math.log})  # expressions from the fixture


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_hand_example_selection(oracle_mod, dtype):
    g = _hand()
    T = g["shape"]["T"]
    inp = {k: _bnhd(v, dtype) for k, v in g["inputs"].items() if k.startswith(("q", "k", "v"))}
    w_q = torch.tensor(g["inputs"]["w_q"], dtype=torch.float64).to(dtype)[None]
    w_k = torch.tensor(g["inputs"]["w_k"], dtype=torch.float64).to(dtype)[None]
    pq = oracle_mod.pool(inp["q"], T)
    pk = oracle_mod.pool(inp["k"], T)
    np.testing.assert_array_equal(pq[0, 0], np.array(g["expected"]["pooled_q"], float))
    np.testing.assert_array_equal(pk[0, 0], np.array(g["expected"]["pooled_k"], float))
    qhat = oracle_mod.project(pq, w_q)
    khat = oracle_mod.project(pk, w_k)
    np.testing.assert_array_equal(khat[0, 0], np.array(g["expected"]["khat"], float))
    s = oracle_mod.scores(qhat, khat, rows=[0, 1, 2])
    np.testing.assert_array_equal(s, np.array(g["expected"]["scores"], float))
    idx, kth, nxt = oracle_mod.select(qhat, khat, g["shape"]["budget"])
    np.testing.assert_array_equal(idx[0, 0], np.array(g["expected"]["idx"]))
    np.testing.assert_array_equal(kth[0, 0], np.array(g["expected"]["kth"], float))
    np.testing.assert_array_equal(nxt[0, 0], np.array(g["expected"]["next"], float))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_hand_example_attention(oracle_mod, dtype):
    g = _hand()
    T = g["shape"]["T"]
    t = {k: _bnhd(v, dtype) for k, v in g["inputs"].items() if not k.startswith("w")}
    idx = np.array(g["expected"]["idx"], np.int32)[None, None]
    units = [(0, 0, i) for i in range(3)]
    out, lse = oracle_mod.attend(t["q"], (t["k"], t["v"]), T, idx, units,
                                 dense=(t["k_dense"], t["v_dense"]), scale=g["shape"]["scale"])
    want = np.array([[_eval(e) for e in row] for row in g["expected"]["out_expr"]])
    want_lse = np.array([_eval(e) for e in g["expected"]["lse_expr"]])
    got = out.reshape(-1, 2)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13, equal_nan=True)
    np.testing.assert_allclose(lse.reshape(-1), want_lse, rtol=1e-13, atol=1e-13, equal_nan=True)


# ---------------------------------------------------------------------------
# pooling
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,T", [(11, 4), (12, 4), (1, 4), (130, 64)])
def test_pool_closed_form(oracle_mod, dtype, N, T):
    """x[b,t,h,e] = a[b,h,e] + c[e]*t (small integers, exact in bf16 too):
    the mean over tokens t0..t1-1 is a + c*(t0 + t1 - 1)/2, whatever the
    tile's length (a short last tile included)."""
    B, H, d = 2, 3, 5
    gen = torch.Generator().manual_seed(7)
    a = torch.randint(-20, 20, (B, H, d), generator=gen).double()
    c = torch.randint(-1, 2, (d,), generator=gen).double()
    t = torch.arange(N).double()
    x = a[:, None, :, :] + c[None, None, None, :] * t[None, :, None, None]   # [B,N,H,d]
    # store as [B,H,N,d] and view as [B,N,H,d]: non-packed strides
    xs = x.permute(0, 2, 1, 3).contiguous().to(dtype).permute(0, 2, 1, 3)
    got = oracle_mod.pool(xs, T)
    n = -(-N // T)
    want = np.empty((B, H, n, d))
    for i in range(n):
        t0, t1 = i * T, min(N, (i + 1) * T)
        want[:, :, i, :] = (a + c * (t0 + t1 - 1) / 2.0).numpy()
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------------------
# projection
# ---------------------------------------------------------------------------

def test_project_unit_matrices(oracle_mod):
    """W[h] = e_a e_b^T moves pooled channel a of head h to output b, and
    nothing else (catches a transposed or head-mixed weight index)."""
    B, H, n, d, r = 2, 3, 4, 6, 5
    pooled = np.random.default_rng(0).standard_normal((B, H, n, d))
    pairs = [(1, 4), (5, 0), (2, 2)]
    w = torch.zeros(H, d, r)
    for h, (a, b) in enumerate(pairs):
        w[h, a, b] = 1.0
    out = oracle_mod.project(pooled, w)
    for h, (a, b) in enumerate(pairs):
        want = np.zeros((B, n, r))
        want[:, :, b] = pooled[:, h, :, a]
        np.testing.assert_array_equal(out[:, h], want)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_project_commutes_with_pool(oracle_mod, dtype):
    """mean_t(x_t) W == mean_t(x_t W): projecting each token first and then
    averaging (plain numpy, other order of operations) gives the same."""
    B, N, H, d, r, T = 1, 37, 2, 8, 3, 8
    gen = torch.Generator().manual_seed(3)
    x = torch.randn(B, N, H, d, generator=gen).to(dtype)
    w = torch.randn(H, d, r, generator=gen).to(dtype)
    got = oracle_mod.project(oracle_mod.pool(x, T), w)
    xd = x.double().numpy()
    wd = w.double().numpy()
    n = -(-N // T)
    want = np.empty((B, H, n, r))
    for h in range(H):
        per_token = xd[:, :, h, :] @ wd[h]           # [B, N, r]
        for i in range(n):
            want[:, h, i] = per_token[:, i * T:(i + 1) * T].mean(axis=1)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------

def _planted(scores_rows):
    """qhat = e_0, khat_j = s_j e_0, so s_ij = s_j exactly (integers)."""
    s = np.asarray(scores_rows, float)
    R, n = s.shape
    # each row needs its own key scores: one batch entry per row
    qhat = np.zeros((R, 1, 1, 2))
    qhat[:, 0, 0, 0] = 1.0
    khat = np.zeros((R, 1, n, 2))
    khat[:, 0, :, 0] = s
    return qhat, khat


def test_select_planted_ties(oracle_mod):
    s = [[5, 1, 9, 9, 3, 9, 2, 0]]
    qhat, khat = _planted(s)
    want = {1: [2], 2: [2, 3], 3: [2, 3, 5], 4: [0, 2, 3, 5], 8: list(range(8))}
    for k, exp in want.items():
        idx, kth, nxt = oracle_mod.select(qhat, khat, k)
        assert idx.reshape(-1).tolist() == exp, (k, idx)
    idx, kth, nxt = oracle_mod.select(qhat, khat, 2)
    assert kth.item() == 9 and nxt.item() == 9
    idx, kth, nxt = oracle_mod.select(qhat, khat, 4)
    assert kth.item() == 5 and nxt.item() == 3
    idx, kth, nxt = oracle_mod.select(qhat, khat, 8)
    assert kth.item() == 0 and math.isnan(nxt.item())


def test_select_bruteforce_subsets(oracle_mod):
    """The kept set is the k-subset with the largest score sum, and among
    those the smallest index sum (ties go to the lowest indices)."""
    rng = np.random.default_rng(11)
    for trial in range(60):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, n + 1))
        s = rng.integers(-3, 4, size=n).astype(float)
        qhat, khat = _planted([s])
        idx, _, _ = oracle_mod.select(qhat, khat, k)
        best = max(itertools.combinations(range(n), k),
                   key=lambda c: (sum(s[j] for j in c), -sum(c)))
        assert idx.reshape(-1).tolist() == list(best), (s, k)


def test_select_planted_per_head(oracle_mod):
    """Several heads with their own planted integer scores (q-hat = e_0 in
    every head, k-hat_j = s_hj e_0): each head's kept set is its own
    brute-force best k-subset, so a score or selection that mixes heads
    (or batch entries) fails."""
    rng = np.random.default_rng(23)
    B, H, n = 2, 3, 7
    s = rng.integers(-4, 5, size=(B, H, n)).astype(float)
    s[0, 1] = s[0, 0][::-1]                 # heads with permuted scores: a head mix-up changes the set
    qhat = np.zeros((B, H, 1, 2))
    qhat[..., 0] = 1.0
    khat = np.zeros((B, H, n, 2))
    khat[..., 0] = s
    for k in (1, 3, 6):
        idx, kth, _ = oracle_mod.select(qhat, khat, k)
        for b, h in itertools.product(range(B), range(H)):
            best = max(itertools.combinations(range(n), k),
                       key=lambda c: (sum(s[b, h, j] for j in c), -sum(c)))
            assert idx[b, h, 0].tolist() == list(best), (b, h, k)
            assert kth[b, h, 0] == sorted(s[b, h])[::-1][k - 1]


def test_select_properties_random(oracle_mod):
    rng = np.random.default_rng(5)
    B, H, nq, nk, r = 2, 3, 9, 23, 4
    qhat = rng.standard_normal((B, H, nq, r))
    khat = rng.standard_normal((B, H, nk, r))
    khat[:, :, 7] = khat[:, :, 3]          # exact duplicate tiles -> exact ties
    for k in (1, 5, 11, 22, 23):
        idx, kth, nxt = oracle_mod.select(qhat, khat, k)
        rows = np.arange(B * H * nq)
        s = oracle_mod.scores(qhat, khat, rows).reshape(B, H, nq, nk)
        for b, h, i in itertools.product(range(B), range(H), range(nq)):
            kept = idx[b, h, i].tolist()
            assert len(kept) == k and all(0 <= j < nk for j in kept)
            assert all(a < c for a, c in zip(kept, kept[1:]))
            dropped = sorted(set(range(nk)) - set(kept))
            srow = s[b, h, i]
            if dropped:
                lo = min(srow[kept])
                hi = max(srow[dropped])
                assert lo >= hi
                # equal scores across the boundary: every kept index is lower
                for j in dropped:
                    for m in kept:
                        if srow[j] == srow[m]:
                            assert m < j
            order = np.sort(srow)[::-1]
            assert kth[b, h, i] == order[k - 1]
            if k < nk:
                assert nxt[b, h, i] == order[k]


def test_select_duplicate_tiles_through_pipeline(oracle_mod):
    """Key tiles 3 and 6 hold identical tokens, so they score identically in
    any precision; at the budget boundary the lower index must win."""
    T, d = 4, 3
    u = np.array([1.0, 2.0, -1.0])
    coeff = [1, 2, 7, 5, 0, 3, 5, -2]            # per key tile: every token = coeff * u
    kt = []
    for c in coeff:
        kt += [list(c * u)] * T
    k = _bnhd(kt)
    q = _bnhd([list(u)] * (2 * T))
    eye = torch.eye(d)[None]
    qhat = oracle_mod.project(oracle_mod.pool(q, T), eye)
    khat = oracle_mod.project(oracle_mod.pool(k, T), eye)
    idx, kth, nxt = oracle_mod.select(qhat, khat, 2)
    assert idx[0, 0].tolist() == [[2, 3], [2, 3]]
    assert kth[0, 0, 0] == nxt[0, 0, 0]          # a tie sits on the boundary
    idx, _, _ = oracle_mod.select(qhat, khat, 3)
    assert idx[0, 0, 0].tolist() == [2, 3, 6]


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def _sdpa(q, keys, vals, mask=None, scale=None):
    """Textbook dense softmax attention in fp64 via torch: q [Nq, d], keys [Nk, d]."""
    o = F.scaled_dot_product_attention(q[None, None], keys[None, None], vals[None, None],
                                       attn_mask=None if mask is None else mask[None, None],
                                       scale=scale)
    return o[0, 0]


def _problem(seed, B, H, d, T, n_video, n_ref=0, n_dense=0, dtype=torch.float32):
    gen = torch.Generator().manual_seed(seed)

    def r(n):
        return torch.randn(B, n, H, d, generator=gen).to(dtype)

    p = {"q": r(n_video), "k": r(n_video), "v": r(n_video)}
    if n_ref:
        p["k_ref"], p["v_ref"] = r(n_ref), r(n_ref)
    if n_dense:
        p["k_dense"], p["v_dense"] = r(n_dense), r(n_dense)
    return p


def _mask_from_idx(idx_row, T, n_video, n_ref=0, idx_r_row=None, n_dense=0):
    """Boolean key mask (video | ref | dense) for one query tile."""
    m = torch.zeros(n_video + n_ref + n_dense, dtype=torch.bool)
    for j in idx_row:
        m[j * T:min(n_video, (j + 1) * T)] = True
    if n_ref:
        for j in idx_r_row:
            m[n_video + j * T:n_video + min(n_ref, (j + 1) * T)] = True
    m[n_video + n_ref:] = True
    return m


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_attend_full_budget_is_dense_attention(oracle_mod, dtype):
    B, H, d, T, N, Nd = 2, 2, 16, 8, 45, 11        # ragged video and dense tails
    p = _problem(1, B, H, d, T, N, n_dense=Nd, dtype=dtype)
    nq = -(-N // T)
    idx = np.broadcast_to(np.arange(nq, dtype=np.int32), (B, H, nq, nq)).copy()
    units = [(b, h, i) for b in range(B) for h in range(H) for i in range(nq)]
    out, lse = oracle_mod.attend(p["q"], (p["k"], p["v"]), T, idx, units,
                                 dense=(p["k_dense"], p["v_dense"]))
    for u, (b, h, i) in enumerate(units):
        qs = p["q"][b, i * T:min(N, (i + 1) * T), h].double()
        keys = torch.cat([p["k"][b, :, h], p["k_dense"][b, :, h]]).double()
        vals = torch.cat([p["v"][b, :, h], p["v_dense"][b, :, h]]).double()
        want = _sdpa(qs, keys, vals).numpy()
        c = qs.shape[0]
        np.testing.assert_allclose(out[u, :c], want, rtol=1e-11, atol=1e-12)
        assert np.isnan(out[u, c:]).all()
        want_lse = torch.logsumexp((qs @ keys.T) / math.sqrt(d), dim=1).numpy()
        np.testing.assert_allclose(lse[u, :c], want_lse, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("via", ["attend", "attend_units"])
def test_attend_masked_dense_equivalence_with_reference_segment(oracle_mod, via):
    """Through attend() and through attend_units(), the composition the GPU
    parity tests call with a problem's tensors."""
    B, H, d, T = 1, 2, 8, 4
    N, Nr, Nd = 30, 13, 6
    p = _problem(2, B, H, d, T, N, n_ref=Nr, n_dense=Nd)
    nq, nr = -(-N // T), -(-Nr // T)
    rng = np.random.default_rng(2)
    k_v, k_r = 3, 2
    idx_v = np.sort(np.stack([rng.choice(nq, k_v, replace=False)
                              for _ in range(B * H * nq)]).reshape(B, H, nq, k_v), -1).astype(np.int32)
    idx_r = np.sort(np.stack([rng.choice(nr, k_r, replace=False)
                              for _ in range(B * H * nq)]).reshape(B, H, nq, k_r), -1).astype(np.int32)
    # make sure the short last tiles (video 7, reference 3) are picked somewhere
    idx_v[0, 0, 0] = [0, 5, 7]
    idx_r[0, 0, 0] = [1, 3]
    units = [(0, h, i) for h in range(H) for i in range(nq)]
    if via == "attend":
        out, lse = oracle_mod.attend(p["q"], (p["k"], p["v"]), T, idx_v, units,
                                     ref=(p["k_ref"], p["v_ref"]), idx_r=idx_r,
                                     dense=(p["k_dense"], p["v_dense"]), scale=0.3)
    else:
        out, lse = oracle_mod.attend_units(p, T, idx_v, idx_r, units, scale=0.3)
    for u, (b, h, i) in enumerate(units):
        qs = p["q"][b, i * T:min(N, (i + 1) * T), h].double()
        keys = torch.cat([p["k"][b, :, h], p["k_ref"][b, :, h], p["k_dense"][b, :, h]]).double()
        vals = torch.cat([p["v"][b, :, h], p["v_ref"][b, :, h], p["v_dense"][b, :, h]]).double()
        m = _mask_from_idx(idx_v[b, h, i], T, N, Nr, idx_r[b, h, i], Nd)
        want = _sdpa(qs, keys, vals, m.expand(qs.shape[0], -1), scale=0.3).numpy()
        c = qs.shape[0]
        np.testing.assert_allclose(out[u, :c], want, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dense_query_rows_are_dense_attention(oracle_mod, dtype):
    """Non-video query rows attending to every tile (reference present, ragged
    query, video, reference and dense tails) equal textbook dense attention
    over the concatenated keys."""
    B, H, d, T = 2, 2, 16, 8
    N, Nr, Nd, Nq = 29, 13, 6, 21
    p = _problem(5, B, H, d, T, N, n_ref=Nr, n_dense=Nd, dtype=dtype)
    gen = torch.Generator().manual_seed(55)
    q_rows = torch.randn(B, Nq, H, d, generator=gen).to(dtype)
    nq = -(-Nq // T)
    units = [(b, h, i) for b in range(B) for h in range(H) for i in range(nq)]
    out, lse = oracle_mod.attend_dense_queries(p, q_rows, T, units, scale=0.4)
    for u, (b, h, i) in enumerate(units):
        qs = q_rows[b, i * T:min(Nq, (i + 1) * T), h].double()
        keys = torch.cat([p["k"][b, :, h], p["k_ref"][b, :, h], p["k_dense"][b, :, h]]).double()
        vals = torch.cat([p["v"][b, :, h], p["v_ref"][b, :, h], p["v_dense"][b, :, h]]).double()
        c = qs.shape[0]
        np.testing.assert_allclose(out[u, :c], _sdpa(qs, keys, vals, scale=0.4).numpy(), rtol=1e-11, atol=1e-12)
        assert np.isnan(out[u, c:]).all()
        want_lse = torch.logsumexp((qs @ keys.T) * 0.4, dim=1).numpy()
        np.testing.assert_allclose(lse[u, :c], want_lse, rtol=1e-12, atol=1e-12)


def test_attend_all_ones_values(oracle_mod):
    """Softmax weights sum to one: with V = 1 every output is exactly 1."""
    B, H, d, T, N, Nd = 1, 2, 8, 4, 23, 5
    p = _problem(3, B, H, d, T, N, n_dense=Nd)
    p["v"] = torch.ones_like(p["v"])
    p["v_dense"] = torch.ones_like(p["v_dense"])
    p["q"] = p["q"] * 6.0                               # peaked softmax
    nq = -(-N // T)
    idx = np.tile(np.array([1, 5], np.int32), (B, H, nq, 1))
    units = [(0, h, i) for h in range(H) for i in range(nq)]
    out, _ = oracle_mod.attend(p["q"], (p["k"], p["v"]), T, idx, units,
                               dense=(p["k_dense"], p["v_dense"]))
    valid = ~np.isnan(out)
    assert np.abs(out[valid] - 1.0).max() < 1e-13


def test_attend_single_tile_is_t_key_softmax(oracle_mod):
    B, H, d, T, N = 1, 1, 8, 4, 16
    p = _problem(4, B, H, d, T, N)
    idx = np.array([[[[2], [0], [3], [1]]]], np.int32)
    units = [(0, 0, i) for i in range(4)]
    out, _ = oracle_mod.attend(p["q"], (p["k"], p["v"]), T, idx, units)
    for i in range(4):
        j = int(idx[0, 0, i, 0])
        qs = p["q"][0, i * T:(i + 1) * T, 0].double()
        ks = p["k"][0, j * T:(j + 1) * T, 0].double()
        vs = p["v"][0, j * T:(j + 1) * T, 0].double()
        w = torch.softmax(qs @ ks.T / math.sqrt(d), dim=1)
        np.testing.assert_allclose(out[i], (w @ vs).numpy(), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# the tiny workload end to end
# ---------------------------------------------------------------------------

def test_tiny_workload_full_budget_equals_dense(oracle_mod):
    """Tiny config (fp32, 4096 video tokens, 64 tiles, 128 dense text keys):
    at a budget of all 64 tiles, selection keeps every tile and attention is
    plain dense attention."""
    w = workloads.get("tiny")
    inp = workloads.make_inputs(w)
    sel = oracle_mod.select_tiles(inp, w.T, w.n_q_tiles)
    assert (sel["idx_v"] == np.arange(w.n_q_tiles)).all()
    units = [(0, h, i) for h in range(w.H) for i in (0, 17, 63)]
    out, _ = oracle_mod.attend_units(inp, w.T, sel["idx_v"], None, units)
    for u, (b, h, i) in enumerate(units):
        qs = inp["q"][b, i * w.T:(i + 1) * w.T, h].double()
        keys = torch.cat([inp["k"][b, :, h], inp["k_dense"][b, :, h]]).double()
        vals = torch.cat([inp["v"][b, :, h], inp["v_dense"][b, :, h]]).double()
        np.testing.assert_allclose(out[u], _sdpa(qs, keys, vals).numpy(), rtol=1e-11, atol=1e-12)


def test_tiny_workload_selection_shape_and_budget(oracle_mod):
    w = workloads.get("tiny")
    inp = workloads.make_inputs(w)
    sel = oracle_mod.select_tiles(inp, w.T, w.budget_video)
    idx = sel["idx_v"]
    assert idx.shape == (1, 2, 64, 8)
    assert (np.diff(idx, axis=-1) > 0).all() and idx.min() >= 0 and idx.max() < 64


def test_select_tiles_reference_segment_hand_case(oracle_mod):
    """The reference segment's key tiles are projected with W_k (the same key
    projection as the video tiles) and ranked against the query tiles'
    qhat independently of the video tiles, with their own budget (veyrul.com,
    "Veda R2VA for MiniMax-H3", second paragraph: reference and video tiles
    are selected independently with fixed budgets).

    Hand derivation (d = r = 2, T = 2, every token of a tile equal, so the
    pooled vector is that token):
      W_q = [[1, 0], [0, 2]]  ->  qhat = pooled q W_q;  W_k = [[0, 1], [1, 0]]
      (swaps the two channels).
      query tile: (1, 1) -> qhat = (1, 2).
      video tiles  (0, 5), (1, 0), (2, 2) -> khat (5, 0), (0, 1), (2, 2)
                   -> scores 5, 2, 6 -> budget 1 keeps {2}.
      reference    (3, 0), (0, 2), (1, 1) -> khat (0, 3), (2, 0), (1, 1)
                   -> scores 6, 2, 3 -> budget 2 keeps {0, 2}.
    Projecting the reference with W_q instead would give khat (3, 0), (0, 4),
    (1, 2) and scores 3, 8, 5 (keeps {1, 2}); ranking the reference against
    the video's khat, or with the video's budget, gives {0, 2} -> [2] or [0]."""
    T = 2

    def tiles(vals):
        rows = []
        for v in vals:
            rows += [v] * T
        return _bnhd(rows)

    inp = {
        "q": tiles([(1, 1)]),
        "k": tiles([(0, 5), (1, 0), (2, 2)]),
        "k_ref": tiles([(3, 0), (0, 2), (1, 1)]),
        "w_q": torch.tensor([[[1.0, 0.0], [0.0, 2.0]]]),
        "w_k": torch.tensor([[[0.0, 1.0], [1.0, 0.0]]]),
    }
    sel = oracle_mod.select_tiles(inp, T, 1, 2)
    np.testing.assert_array_equal(sel["qhat"].reshape(-1), [1.0, 2.0])
    np.testing.assert_array_equal(sel["khat_r"].reshape(3, 2), [[0, 3], [2, 0], [1, 1]])
    assert sel["idx_v"].reshape(-1).tolist() == [2]
    assert sel["idx_r"].reshape(-1).tolist() == [0, 2]
    assert sel["kth_r"].item() == 3.0 and sel["next_r"].item() == 2.0
