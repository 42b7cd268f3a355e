"""Seeded synthetic visual-KV workloads (inputs only; no codec arithmetic here).

The TACT-KV pages evaluate on real CT / video KV caches that are not available here, so every
input is a synthetic stand-in with the structure the method relies on: a visual K or V tensor of
one layer, laid out on its (S, H, W) token grid ("Methodology in Plain English", stage 1 of the
TACT-KV summary page), correlated along each of the three axes (the same section names this
as the redundancy the 3D transform removes) and heavy-tailed ("Main Findings", gain-shape
bullet: post-DCT absmax/std 4.81 versus 3.01 for a Gaussian).

Field recipe (per channel): iid innovations e, filtered along S, then H, then W by a stationary
AR(1) recursion y[0] = e[0], y[t] = rho * y[t-1] + sqrt(1 - rho^2) * e[t]; innovations are
Gaussian or Student-t(nu) rescaled to unit variance by sqrt((nu - 2) / nu); the field is then
multiplied by a per-channel scale.  K and V of a layer are independent draws.

Both the CUDA path and the oracle receive exactly the tensors produced here (generated once,
copied to wherever they are consumed), so this module is the only code the two sides share.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator, List, Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One benchmark configuration: a batch of independent units of the same shape."""
    name: str
    S: int
    H: int
    W: int
    heads: int
    head_dim: int
    layers: int
    kv: Tuple[int, ...]            # which of K (0) / V (1) are present
    sequences: int
    bits: Tuple[int, ...]          # nominal bits per element exercised
    rho: Tuple[float, float, float]
    nu: Optional[float]            # None -> Gaussian innovations
    scale: str                     # "one" | "lognormal0.5" | "outlier1pct_x10"
    dtype: torch.dtype
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.S * self.H * self.W

    @property
    def channels(self) -> int:
        return self.heads * self.head_dim

    @property
    def n_units(self) -> int:
        return self.sequences * self.layers * len(self.kv)

    @property
    def elements_per_unit(self) -> int:
        return self.tokens * self.channels

    def units(self) -> Iterator[Tuple[int, int, int]]:
        """(sequence, layer, kv) of every unit, in the order units are laid out in a batch."""
        for q in range(self.sequences):
            for layer in range(self.layers):
                for kv in self.kv:
                    yield q, layer, kv


WORKLOADS = {
    # 1 layer, K only, 1 head x 64, 8x8x8 grid, fp32 Gaussian AR(1) rho=0.9, LogNormal(0,0.5) scales
    "tiny": Workload("tiny", 8, 8, 8, 1, 64, 1, (0,), 1, (2,), (0.9, 0.9, 0.9), None,
                     "lognormal0.5", torch.float32, seed=0),
    # 4B-class medical VLM: 34 layers, 4 KV heads x 256, K and V, 64x16x16 grid, t(4), 1 bit
    "med4b": Workload("med4b", 64, 16, 16, 4, 256, 34, (0, 1), 1, (1,), (0.85, 0.9, 0.9), 4.0,
                      "one", torch.bfloat16, seed=2),
    # same layout, batch 8 with independent seeds, 1/2/4 bits
    "med4b_b8": Workload("med4b_b8", 64, 16, 16, 4, 256, 34, (0, 1), 8, (1, 2, 4),
                         (0.85, 0.9, 0.9), 4.0, "one", torch.bfloat16, seed=3),
    # 32B-class: 64 layers, 8 KV heads x 128, 32x24x24 grid, t(4), 1% channels x10, batch 4
    "med32b": Workload("med32b", 32, 24, 24, 8, 128, 64, (0, 1), 4, (1,), (0.85, 0.9, 0.9), 4.0,
                       "outlier1pct_x10", torch.bfloat16, seed=4),
    # video VLM: 28 layers, 4 KV heads x 128, 64 frames x 14 x 14, rho_T=.95 rho_HW=.8, t(5), batch 16
    "video": Workload("video", 64, 14, 14, 4, 128, 28, (0, 1), 16, (1,), (0.95, 0.8, 0.8), 5.0,
                      "one", torch.bfloat16, seed=5),
}


def unit_seed(w: Workload, seq: int, layer: int, kv: int) -> int:
    """Deterministic seed of one unit: distinct per (workload seed, sequence, layer, K|V)."""
    return (w.seed * 1_000_003 + seq * 10_007 + layer * 101 + kv * 7 + 12345) & 0x7FFFFFFF


def _innovations(shape, nu: Optional[float], gen: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if nu is None:
        return z
    k = int(round(nu))
    if abs(k - nu) > 1e-9 or k < 3:
        raise ValueError("Student-t innovations need an integer nu >= 3 (chi-square by sums of squares)")
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(k):
        g = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        chi2.addcmul_(g, g)
    t = z / torch.sqrt(chi2 / k)
    return t * math.sqrt((k - 2) / k)


def _ar1_(y: torch.Tensor, axis: int, rho: float) -> None:
    """In place: y <- stationary AR(1) filter of its own values along `axis` (unit variance kept)."""
    c = math.sqrt(1.0 - rho * rho)
    y_t = y.movedim(axis, 0)
    for t in range(1, y_t.shape[0]):
        y_t[t].mul_(c).add_(y_t[t - 1], alpha=rho)


def _channel_scale(kind: str, n: int, gen: torch.Generator, device) -> torch.Tensor:
    if kind == "one":
        return torch.ones(n, device=device)
    if kind == "lognormal0.5":
        return torch.exp(0.5 * torch.randn(n, generator=gen, device=device))
    if kind == "outlier1pct_x10":
        s = torch.ones(n, device=device)
        k = max(1, int(round(0.01 * n)))
        idx = torch.randperm(n, generator=gen, device=device)[:k]
        s[idx] = 10.0
        return s
    raise ValueError(kind)


def make_unit(S: int, H: int, W: int, heads: int, head_dim: int, *, rho=(0.9, 0.9, 0.9),
              nu: Optional[float] = None, scale: str = "one", dtype=torch.bfloat16,
              seed: int = 0, device="cpu") -> torch.Tensor:
    """One synthetic visual K or V: tensor [S*H*W tokens, heads, head_dim], token t = (s*H + h)*W + w."""
    n = heads * head_dim
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    y = _innovations((S, H, W, n), nu, gen, device)
    for axis, r in enumerate(rho):
        _ar1_(y, axis, float(r))
    y.mul_(_channel_scale(scale, n, gen, device))
    return y.reshape(S * H * W, heads, head_dim).to(dtype)


def make_workload_unit(w: Workload, seq: int, layer: int, kv: int, device="cpu") -> torch.Tensor:
    return make_unit(w.S, w.H, w.W, w.heads, w.head_dim, rho=w.rho, nu=w.nu, scale=w.scale,
                     dtype=w.dtype, seed=unit_seed(w, seq, layer, kv), device=device)


def make_batch(w: Workload, device="cpu", out: Optional[torch.Tensor] = None,
               units: Optional[List[int]] = None) -> torch.Tensor:
    """All (or the listed) units of a workload stacked as [units, tokens, heads, head_dim]."""
    all_units = list(w.units())
    pick = range(len(all_units)) if units is None else units
    if out is None:
        out = torch.empty((len(pick), w.tokens, w.heads, w.head_dim), dtype=w.dtype, device=device)
    for j, u in enumerate(pick):
        q, layer, kv = all_units[u]
        out[j].copy_(make_workload_unit(w, q, layer, kv, device=device))
    return out
