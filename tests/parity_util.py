"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same inputs, and compare with the stated tolerances.

Tolerances (the target the library is held to):
* scores:    |gpu - oracle| <= 1e-4 * |oracle| + 1e-35 per element (the
             absolute floor covers float32 flush-to-zero of probabilities
             below 2^-126, summed over at most 256 window rows);
* select:    bit-exact permutation given the same float32 score tensor;
* attention: bf16 -- max |gpu - oracle| <= 2e-2 and per-row relative L2
             error <= 5e-3;  fp32 -- both <= 1e-5;
* dropped rows: exactly +0.0 in every column (bit pattern 0).
"""

from __future__ import annotations

import numpy as np
import torch

import long_context_tsa_b200 as T
from long_context_tsa_b200 import inputs as I
from oracle import tsa_oracle as O

SCORE_RTOL = 1e-4
SCORE_ATOL = 1e-35
ATOL = {"bf16": 2e-2, "f32": 1e-5}
RTOL_ROW = {"bf16": 5e-3, "f32": 1e-5}


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


class Run:
    """Device buffers and a workspace for one workload shape."""

    def __init__(self, w: I.Workload, q, k, v, window=None, scale=0.0):
        self.w = w
        self.q, self.k, self.v = q, k, v
        self.window = w.W if window is None else window
        self.desc = T.desc_for(q, k, scale)
        self.ws = T.alloc_workspace(self.desc, self.window, device=q.device)
        dev = q.device
        self.scores = torch.empty((w.B, w.Hkv, w.L), dtype=torch.float32, device=dev)
        self.perm = torch.empty((w.B, w.Hkv, w.L), dtype=torch.int32, device=dev)
        self.out = torch.empty_like(q)

    def status(self) -> int:
        return T.tsa_check_status(self.ws)

    def score(self):
        T.tsa_score(self.desc, self.q, self.k, self.window, self.scores, self.ws)
        assert self.status() == 0
        return self.scores

    def select(self, scores, budgets):
        T.tsa_select(self.desc, scores, budgets, self.perm, self.ws)
        assert self.status() == 0
        return self.perm

    def attend(self, perm, budgets):
        self.out.fill_(float("nan"))  # every element must be written
        T.tsa_attend(self.desc, self.q, self.k, self.v, perm, budgets, self.out, self.ws)
        assert self.status() == 0
        return self.out

    def forward(self, budgets):
        self.out.fill_(float("nan"))
        T.tsa_forward(self.desc, self.q, self.k, self.v, self.window, budgets, self.out, self.ws,
                      scores=self.scores, perm=self.perm)
        assert self.status() == 0
        return self.scores, self.perm, self.out


def assert_scores_close(gpu: np.ndarray, ora: np.ndarray):
    err = np.abs(gpu.astype(np.float64) - ora)
    bound = SCORE_RTOL * np.abs(ora) + SCORE_ATOL
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} score elements out of tolerance; worst rel "
                           f"{(err / np.maximum(np.abs(ora), 1e-300)).max():.3e}")


def assert_rows_close(gpu_rows: np.ndarray, ora_rows: np.ndarray, dtype: str, what: str = ""):
    """gpu_rows, ora_rows: [n, D]."""
    assert np.all(np.isfinite(gpu_rows)), f"{what}: non-finite output"
    diff = gpu_rows.astype(np.float64) - ora_rows
    mx = np.abs(diff).max() if diff.size else 0.0
    rel = np.linalg.norm(diff, axis=1) / np.maximum(np.linalg.norm(ora_rows, axis=1), 1e-30)
    assert mx <= ATOL[dtype], f"{what}: max abs {mx:.3e} > {ATOL[dtype]}"
    assert rel.max(initial=0.0) <= RTOL_ROW[dtype], f"{what}: row rel L2 {rel.max():.3e} > {RTOL_ROW[dtype]}"
    return mx, rel.max(initial=0.0)


def assert_dropped_rows_zero(out: torch.Tensor, perm: torch.Tensor, budgets, G: int):
    """Bit-exact +0 at every dropped position (checked on the device, by bit pattern)."""
    B, Hq, L, D = out.shape
    Hkv = perm.shape[1]
    bits = out.view(torch.int16) if out.dtype == torch.bfloat16 else out.view(torch.int32)
    for b in range(B):
        for g in range(Hkv):
            K = min(int(budgets[b * Hkv + g]), L)
            if K == L:
                continue
            drop = perm[b, g, K:].long()
            sl = bits[b, g * G:(g + 1) * G].index_select(1, drop)
            assert int(sl.abs().max()) == 0, f"dropped rows not +0 at b={b} g={g}"


def compare_attend(out: torch.Tensor, q, k, v, perm_np: np.ndarray, budgets, dtype: str, rows_per_head=None,
                   seed: int = 0):
    """Compare kept rows of ``out`` with the oracle (all rows, or a seeded sample per head)."""
    B, Hq, L, D = out.shape
    Hkv = perm_np.shape[1]
    G = Hq // Hkv
    kept = O.clamp_budgets(budgets, L)
    rng = np.random.default_rng(seed)
    worst = (0.0, 0.0)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            K = int(kept[b * Hkv + g])
            if rows_per_head is None or rows_per_head >= K:
                rows = np.arange(K)
            else:
                pick = rng.choice(K, size=rows_per_head, replace=False)
                rows = np.unique(np.concatenate([pick, np.arange(min(4, K)), [K - 1]]))  # first rows hold kept sinks
            ora = O.attend_rows(q, k, v, perm_np[b, g], K, b, h, G, rows)
            pos = torch.from_numpy(perm_np[b, g, rows].astype(np.int64)).to(out.device)
            gpu = host(out[b, h].index_select(0, pos))
            mx, rel = assert_rows_close(gpu, ora, dtype, f"b={b} h={h}")
            worst = (max(worst[0], mx), max(worst[1], rel))
    return worst
