"""Seeded synthetic inputs shaped like the pages' long-context prefill workloads.

This module only draws random tensors and budgets; it holds none of the
method's arithmetic.  The CUDA tests, the benchmark and the oracle's tests all
take their inputs from here.

Workloads (a Llama-3-8B-like attention layer: 32 query heads, 8 KV heads,
head dim 128, contexts up to 128K tokens; the tiny fp32 case is for exhaustive
checks):

* ``tiny_fp32_L256``       B=1, 4 heads (MHA), L=256, d=64, fp32, N(0,1), W=16, K=64.
* ``gqa_bf16_L8192``       B=1, 32/8 heads, d=128, L=8192, bf16, N(0, 0.5^2), W=64, keep 0.5.
* ``gqa_bf16_L32768``      as above at L=32768, keep 0.25, 128 planted salient keys per KV head.
* ``gqa_bf16_L131072``     as above at L=131072, keep 0.1, planted keys plus 4 attention sinks.
* ``ragged_bf16_L131072``  the L=131072 data with per-KV-head budgets drawn in [0.05 L, 0.5 L].

Planted salient keys: for every KV head g a random unit vector u_g and 128
distinct positions in [0, L - W) drawn from the seed; the bias 3 * sigma * sqrt(d) * u_g
(per-coordinate RMS 3 sigma) is added to those keys and to the W window
queries of every query head of group g, which makes their logits stand out
by about 9 sigma^2 sqrt(d) and the scores peaked.  Sinks add the same bias to
keys 0..3.
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    D: int
    dtype: str  # "f32" or "bf16"
    W: int
    keep: float  # fraction of L kept per KV head (ignored when budgets are ragged)
    sigma: float
    planted: int = 0
    sinks: int = 0
    ragged: tuple | None = None  # (lo_frac, hi_frac) for per-head budgets

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def budgets(self, seed: int = 0) -> list[int]:
        """Per-(batch, KV head) budgets, length B * Hkv."""
        n = self.B * self.Hkv
        if self.ragged is None:
            k = max(1, int(math.floor(self.keep * self.L)))
            return [k] * n
        lo = int(math.floor(self.ragged[0] * self.L))
        hi = int(math.floor(self.ragged[1] * self.L))
        g = torch.Generator(device="cpu").manual_seed(1_000_003 + seed)
        return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_fp32_L256", 1, 4, 4, 256, 64, "f32", 16, 0.25, 1.0),
        Workload("gqa_bf16_L8192", 1, 32, 8, 8192, 128, "bf16", 64, 0.5, 0.5),
        Workload("gqa_bf16_L32768", 1, 32, 8, 32768, 128, "bf16", 64, 0.25, 0.5, planted=128),
        Workload("gqa_bf16_L131072", 1, 32, 8, 131072, 128, "bf16", 64, 0.1, 0.5, planted=128, sinks=4),
        Workload("ragged_bf16_L131072", 1, 32, 8, 131072, 128, "bf16", 64, 0.1, 0.5, planted=128, sinks=4,
                 ragged=(0.05, 0.5)),
    ]
}

# Uniform budgets of the sparsity sweep at L=131072: K = floor((1 - tau) L).
SWEEP_TAUS = (0.5, 0.75, 0.9, 0.95)


def sweep_budget(tau: float, L: int) -> int:
    return max(1, int(math.floor((1.0 - tau) * L)))


def custom(name: str = "custom", **kw) -> Workload:
    base = dict(B=1, Hq=4, Hkv=4, L=256, D=64, dtype="f32", W=16, keep=0.25, sigma=1.0)
    base.update(kw)
    return Workload(name, **base)


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def make_qkv(w: Workload, seed: int = 0, device: str | torch.device = "cpu"):
    """Return (q, k, v) with layouts [B,Hq,L,D], [B,Hkv,L,D], [B,Hkv,L,D] in the workload dtype.

    Values are drawn in fp32 from a seeded generator on ``device`` and then
    rounded (round-to-nearest-even) to bf16 for the bf16 workloads.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(seed)
    dt = torch_dtype(w)
    shp_q = (w.B, w.Hq, w.L, w.D)
    shp_kv = (w.B, w.Hkv, w.L, w.D)
    q = torch.randn(shp_q, generator=g, device=dev, dtype=torch.float32).mul_(w.sigma)
    k = torch.randn(shp_kv, generator=g, device=dev, dtype=torch.float32).mul_(w.sigma)
    v = torch.randn(shp_kv, generator=g, device=dev, dtype=torch.float32).mul_(w.sigma)
    if w.planted or w.sinks:
        gc = torch.Generator(device="cpu").manual_seed(7_919 + seed)
        hi = w.L - w.W
        for b in range(w.B):
            for kv in range(w.Hkv):
                u = torch.randn(w.D, generator=gc)
                u = u / u.norm()
                bias = (3.0 * w.sigma * math.sqrt(w.D) * u).to(dev)
                pos = []
                if w.planted:
                    n = min(w.planted, hi)
                    pos.append(torch.randperm(hi, generator=gc)[:n])
                if w.sinks:
                    pos.append(torch.arange(min(w.sinks, w.L)))
                p = torch.unique(torch.cat(pos)).to(dev)
                k[b, kv, p] += bias
                q[b, kv * w.G:(kv + 1) * w.G, w.L - w.W:, :] += bias
    return q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous()


def make_scores(B: int, Hkv: int, L: int, seed: int = 0, kind: str = "random") -> torch.Tensor:
    """Synthetic fp32 score tensors [B, Hkv, L] for select tests (CPU).

    kind: "random"  uniform(0,1) values;
          "ties"    values from a small set, so many ties sit at any threshold;
          "equal"   all equal;
          "zeros"   mix of +0.0 and -0.0 with a few positive values;
          "denorm"  subnormal and tiny normal values;
          "peaked"  log-normal exp(3 N(0,1)) values scaled to sum to 256 per
                    head, like window scores (G * W = 256 probability rows)
                    concentrated on a few keys.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    if kind == "random":
        return torch.rand((B, Hkv, L), generator=g)
    if kind == "ties":
        return torch.randint(0, 5, (B, Hkv, L), generator=g).float() * 0.25
    if kind == "equal":
        return torch.full((B, Hkv, L), 0.5)
    if kind == "zeros":
        s = torch.zeros((B, Hkv, L))
        sign = torch.randint(0, 2, (B, Hkv, L), generator=g).bool()
        s[sign] = -0.0
        pos = torch.rand((B, Hkv, L), generator=g) < 0.05
        s[pos] = torch.rand((B, Hkv, L), generator=g)[pos]
        return s
    if kind == "denorm":
        e = torch.randint(-149, -120, (B, Hkv, L), generator=g).float()
        return torch.pow(2.0, e)
    if kind == "peaked":
        x = torch.exp(3.0 * torch.randn((B, Hkv, L), generator=g, dtype=torch.float64))
        return (256.0 * x / x.sum(-1, keepdim=True)).float()
    raise ValueError(kind)


# --- hidden states for the representation-drift metric ------------------------------------
#
# Two [B, L, hidden] tensors shaped like a Llama-3-8B layer's residual stream
# (hidden = 32 heads * 128 = 4096): h_before has N(0, 1) entries times a
# log-normal per-row scale (exp(N(0, 0.5^2))) and 4 outlier channels at 20x;
# h_after = h_before + delta * (fresh N(0, 1) noise at the same row scale).
# Without the outliers the row cosine would be about 1 / sqrt(1 + delta^2);
# with them the drift for the default delta = 0.3 is about 0.03, below the
# 0.05-0.1 stability thresholds the skill page recommends.

DRIFT_WORKLOAD = {"name": "drift_bf16_L131072_h4096", "B": 1, "L": 131072, "hidden": 4096, "dtype": "bf16",
                  "delta": 0.3}


def make_hidden(B: int, L: int, hidden: int, dtype: str = "bf16", delta: float = 0.3, seed: int = 0,
                device: str | torch.device = "cpu", chunk_rows: int = 8192):
    """Seeded (h_before, h_after), each [B, L, hidden] in ``dtype``; generated in row chunks on ``device``."""
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = torch.Generator(device=device).manual_seed(seed)
    before = torch.empty((B * L, hidden), dtype=td, device=device)
    after = torch.empty_like(before)
    outliers = torch.randperm(hidden, generator=torch.Generator().manual_seed(seed + 1))[:4].to(device)
    for r0 in range(0, B * L, chunk_rows):
        n = min(chunk_rows, B * L - r0)
        scale = torch.exp(0.5 * torch.randn((n, 1), generator=g, device=device))
        x = torch.randn((n, hidden), generator=g, device=device)
        x[:, outliers] *= 20.0
        x *= scale
        before[r0:r0 + n] = x.to(td)
        after[r0:r0 + n] = (x + delta * scale * torch.randn((n, hidden), generator=g, device=device)).to(td)
    return before.view(B, L, hidden), after.view(B, L, hidden)
