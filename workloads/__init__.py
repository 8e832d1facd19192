"""Seeded synthetic inputs shaped like the Veda / MiniMax-H3 video workloads.

This module is shared by the CPU oracle tests and the CUDA path.  It holds only
shapes, budgets and random-number recipes: no pooling, projection, scoring,
selection or attention arithmetic lives here.

Workload shapes follow the pages:
  * 1344x768 landscape at 24 fps, clip lengths 5.17 / 10.13 / 14.38 s
    (tao.media "Affine launches MiniMax-H3 video studio...", section
    "Inside the MiniMax-H3 Studio"); 124 frames per 5.17 s clip and the
    32 reference + 32 video tile budgets (veyrul.com record "Veda R2VA for
    MiniMax-H3", second and third paragraphs).
  * 90% / 95% sparsity (tao.media article, section "Training the Selector,
    Not the Generator"); block budgets 16 / 32 / 64 (same article, section
    "How the SN120 Competition Works").
  * R2VA at 1:1 and 4:3 and at 10.1 s and 14.4 s (veyrul.com record "Veda
    R2VA for MiniMax-H3", third paragraph; square and 4:3 formats also in the
    tao.media article, section "Inside the MiniMax-H3 Studio").  The pages
    give no resolution for 1:1 and 4:3: they keep about the 1344x768 pixel
    count at multiples of 16 pixels (1024x1024 -> 64 x 64 latent tokens,
    1152x864 -> 54 x 72).

The latent grids (31 x 48 x 84 tokens for 5.17 s, 87 x 48 x 84 for 14.38 s,
61 x 84 x 48 for the 10.13 s portrait clip) and the value recipes below are
synthetic stand-ins: i.i.d. N(0,1) values plus either a per-frame offset
vector (tiny case) or a smooth sum of 8 low-frequency sinusoids over
(t, y, x), so that pooled tiles carry structure and scores have locality.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Tuple

import torch

__all__ = ["Workload", "WORKLOADS", "get", "make_inputs", "ceil_div", "budget_for_sparsity"]


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def budget_for_sparsity(n_tiles: int, sparsity: float) -> int:
    """Kept tiles for a sparsity ratio: ceil((1 - s) * n), at least 1.

    Computed in exact rational arithmetic (percent steps) so that 0.10 * 977
    cannot round the wrong way."""
    keep_pct = round((1.0 - sparsity) * 10000)  # basis points
    return max(1, ceil_div(n_tiles * keep_pct, 10000))


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    T: int               # tile size (query tile == key tile)
    r: int               # selector projection width
    dtype: str           # "f32" | "bf16"
    frames: int          # latent frames of the generated video
    Y: int               # latent rows per frame
    X: int               # latent columns per frame
    budget_video: int
    ref_frames: int = 0  # latent frames of visual reference (0: no reference segment)
    budget_ref: int = 0
    dense: Tuple[Tuple[str, int], ...] = ()   # always-attended segments, concatenated
    seed: int = 0
    values: str = "sinusoid"   # "frame_offset" | "sinusoid"
    boost_frac: float = 0.0    # fraction of video key tiles given a +3 mean boost
    sweep: Tuple[int, ...] = ()

    # ---- derived sizes -------------------------------------------------
    @property
    def n_video(self) -> int:
        return self.frames * self.Y * self.X

    @property
    def n_ref(self) -> int:
        return self.ref_frames * self.Y * self.X

    @property
    def n_dense(self) -> int:
        return sum(n for _, n in self.dense)

    @property
    def n_q_tiles(self) -> int:
        return ceil_div(self.n_video, self.T)

    @property
    def n_ref_tiles(self) -> int:
        return ceil_div(self.n_ref, self.T)

    @property
    def n_dense_tiles(self) -> int:
        return ceil_div(self.n_dense, self.T)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_budget(self, budget_video: int, budget_ref: Optional[int] = None) -> "Workload":
        return replace(self, budget_video=budget_video,
                       budget_ref=self.budget_ref if budget_ref is None else budget_ref)

    def kept_pairs(self) -> int:
        """(batch, head, query tile, key tile) pairs one attention call touches."""
        per_q = self.budget_video + (self.budget_ref if self.n_ref else 0) + self.n_dense_tiles
        return self.B * self.H * self.n_q_tiles * per_q

    def kept_flops(self) -> float:
        """Algorithmic FLOPs of one attention call: 4*T*T*d per kept block pair
        (Q K^T and P V, two flops per multiply-add), full tiles counted."""
        return 4.0 * self.T * self.T * self.d * self.kept_pairs()

    def describe(self) -> Dict[str, object]:
        return {
            "workload": self.name, "B": self.B, "H": self.H, "head_dim": self.d,
            "tile": self.T, "selector_dim": self.r, "video_tokens": self.n_video,
            "ref_tokens": self.n_ref, "dense_tokens": self.n_dense,
            "budget_video": self.budget_video, "budget_ref": self.budget_ref,
            "q_tiles": self.n_q_tiles, "seed": self.seed,
        }


def _tiny() -> Workload:
    return Workload(name="tiny", B=1, H=2, d=64, T=64, r=32, dtype="f32",
                    frames=4, Y=32, X=32, budget_video=8,
                    dense=(("text", 128),), seed=0, values="frame_offset")


def _t2v_517() -> Workload:
    return Workload(name="t2v_5.17s", B=1, H=32, d=128, T=128, r=64, dtype="bf16",
                    frames=31, Y=48, X=84, budget_video=budget_for_sparsity(977, 0.90),
                    dense=(("text", 512), ("audio", 256)), seed=1)


def _t2v_1438() -> Workload:
    n = ceil_div(87 * 48 * 84, 128)
    return Workload(name="t2v_14.38s", B=1, H=32, d=128, T=128, r=64, dtype="bf16",
                    frames=87, Y=48, X=84, budget_video=budget_for_sparsity(n, 0.95),
                    dense=(("text", 512), ("audio", 512)), seed=2,
                    sweep=tuple(budget_for_sparsity(n, s) for s in (0.80, 0.90, 0.95, 0.98)))


def _r2va() -> Workload:
    return Workload(name="r2va_5.17s", B=1, H=32, d=128, T=128, r=64, dtype="bf16",
                    frames=31, Y=48, X=84, budget_video=32, ref_frames=2, budget_ref=32,
                    dense=(("text", 512), ("vlm", 256), ("audio", 256)), seed=3)


def _portrait() -> Workload:
    n = ceil_div(61 * 84 * 48, 128)
    return Workload(name="portrait_10.13s", B=1, H=40, d=128, T=128, r=64, dtype="bf16",
                    frames=61, Y=84, X=48, budget_video=budget_for_sparsity(n, 0.90),
                    dense=(("text", 512),), seed=4, boost_frac=0.05,
                    sweep=(budget_for_sparsity(n, 0.90), n))


def _competition_budgets() -> Tuple[Workload, ...]:
    """t2v 5.17 s at the competition's fixed block budgets 16 / 32 / 64."""
    base = _t2v_517()
    return tuple(replace(base, name=f"t2v_5.17s_k{k}", budget_video=k) for k in (16, 32, 64))


def _r2va_variants() -> Tuple[Workload, ...]:
    """R2VA at 1:1 and 4:3 (5.17 s) and at 10.1 s / 14.4 s (16:9)."""
    base = _r2va()
    return (replace(base, name="r2va_5.17s_1x1", Y=64, X=64, seed=5),
            replace(base, name="r2va_5.17s_4x3", Y=54, X=72, seed=6),
            replace(base, name="r2va_10.13s", frames=61, seed=7),
            replace(base, name="r2va_14.38s", frames=87, seed=8))


WORKLOADS: Dict[str, Workload] = {w.name: w for w in
                                  (_tiny(), _t2v_517(), _t2v_1438(), _r2va(), _portrait())
                                  + _competition_budgets() + _r2va_variants()}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def small(name: str, **kw) -> Workload:
    """A reduced workload for parity tests (same recipe, fewer frames/heads)."""
    return replace(WORKLOADS[name], **kw)


# ---------------------------------------------------------------------------
# value recipes
# ---------------------------------------------------------------------------

def _xavier(g: torch.Generator, H: int, d: int, r: int, device) -> torch.Tensor:
    a = math.sqrt(6.0 / (d + r))
    return (torch.rand((H, d, r), generator=g, device=device, dtype=torch.float32) * 2.0 - 1.0) * a


@dataclass
class _Smooth:
    """Parameters of a smooth spatio-temporal component: 8 sinusoids over
    (t, y, x), integer frequencies 0..2 per axis (not all zero), one phase per
    (sinusoid, head, channel)."""
    freqs: torch.Tensor    # [8, 3]
    phases: torch.Tensor   # [8, H, d]


def _smooth_params(seed: int, tag: int, H: int, d: int) -> _Smooth:
    g = torch.Generator(device="cpu").manual_seed(seed * 1000 + tag)
    rows = []
    while len(rows) < 8:
        f = torch.randint(0, 3, (3,), generator=g)
        if int(f.abs().sum()) > 0:
            rows.append(f)
    freqs = torch.stack(rows).to(torch.float32)
    phases = torch.rand((8, H, d), generator=g, dtype=torch.float32) * (2.0 * math.pi)
    return _Smooth(freqs, phases)


def _add_smooth(x: torch.Tensor, sp: _Smooth, F: int, Y: int, X: int) -> None:
    """x: [B, F*Y*X, H, d] fp32, modified in place (one frame at a time)."""
    B, N, H, d = x.shape
    dev = x.device
    freqs = sp.freqs.to(dev)
    # sin(a + p) = sin a cos p + cos a sin p  ->  basis [tokens, 16] @ coef [16, H*d]
    coef = torch.cat([torch.cos(sp.phases), torch.sin(sp.phases)], 0).reshape(16, H * d).to(dev)
    coef = coef * (1.0 / math.sqrt(8.0))
    yy, xx = torch.meshgrid(torch.arange(Y, device=dev, dtype=torch.float32),
                            torch.arange(X, device=dev, dtype=torch.float32), indexing="ij")
    yy = yy.reshape(-1) / Y
    xx = xx.reshape(-1) / X
    for t in range(F):
        ang = 2.0 * math.pi * (freqs[:, 0][None, :] * (t / F) + freqs[:, 1][None, :] * yy[:, None]
                               + freqs[:, 2][None, :] * xx[:, None])            # [Y*X, 8]
        basis = torch.cat([torch.sin(ang), torch.cos(ang)], 1)                  # [Y*X, 16]
        comp = (basis @ coef).reshape(Y * X, H, d)
        x[:, t * Y * X:(t + 1) * Y * X] += comp[None]


def _video_tensor(g, w: Workload, F: int, tag: int, device, smooth_tag: Optional[int]) -> torch.Tensor:
    N = F * w.Y * w.X
    x = torch.randn((w.B, N, w.H, w.d), generator=g, device=device, dtype=torch.float32)
    if w.values == "frame_offset":
        off = torch.randn((w.B, F, w.H, w.d), generator=g, device=device, dtype=torch.float32) * 0.5
        x.view(w.B, F, w.Y * w.X, w.H, w.d).add_(off[:, :, None])
    elif w.values == "sinusoid":
        _add_smooth(x, _smooth_params(w.seed, smooth_tag if smooth_tag is not None else tag, w.H, w.d),
                    F, w.Y, w.X)
    else:
        raise ValueError(w.values)
    return x


def boosted_tiles(w: Workload) -> torch.Tensor:
    """Seeded set of video key tiles that receive the +3 mean boost."""
    n = w.n_q_tiles
    cnt = ceil_div(int(round(w.boost_frac * 10000)) * n, 10000) if w.boost_frac > 0 else 0
    g = torch.Generator(device="cpu").manual_seed(w.seed * 1000 + 99)
    return torch.sort(torch.randperm(n, generator=g)[:cnt]).values


def make_inputs(w: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    """All tensors of one problem, in the layout the library takes:
    q, k, v, k_ref, v_ref, k_dense, v_dense: [B, N, H, d] (d contiguous), dtype w.dtype;
    w_q, w_k: [H, d, r], dtype w.dtype."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(w.seed)
    out: Dict[str, torch.Tensor] = {}
    for i, name in enumerate(("q", "k", "v")):
        x = _video_tensor(g, w, w.frames, tag=i, device=device, smooth_tag=i)
        if name == "k" and w.boost_frac > 0:
            T = w.T
            for j in boosted_tiles(w).tolist():
                x[:, j * T:min((j + 1) * T, x.shape[1])] += 3.0
        out[name] = x.to(w.torch_dtype)
        del x
    if w.ref_frames:
        for i, name in enumerate(("k_ref", "v_ref")):
            x = _video_tensor(g, w, w.ref_frames, tag=10 + i, device=device, smooth_tag=10 + i)
            out[name] = x.to(w.torch_dtype)
            del x
    if w.dense:
        parts_k, parts_v = [], []
        for _, n in w.dense:
            parts_k.append(torch.randn((w.B, n, w.H, w.d), generator=g, device=device))
            parts_v.append(torch.randn((w.B, n, w.H, w.d), generator=g, device=device))
        out["k_dense"] = torch.cat(parts_k, 1).to(w.torch_dtype)
        out["v_dense"] = torch.cat(parts_v, 1).to(w.torch_dtype)
    out["w_q"] = _xavier(g, w.H, w.d, w.r, device).to(w.torch_dtype)
    out["w_k"] = _xavier(g, w.H, w.d, w.r, device).to(w.torch_dtype)
    return out
