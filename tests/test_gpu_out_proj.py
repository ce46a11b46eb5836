"""Output projection + residual (tsa_out_proj) against the oracle.

Both sides get the same inputs: the residual x, the full-length attention
output (zeros at every row a head's group dropped, as tsa_attend writes it)
and the projection weight.  Rows kept by some group are compared with the
oracle's fp64 value within a bound derived from the arithmetic (one rounding
of the result to the output dtype, 2^-8 relative for bf16, plus fp32
accumulation over at most Hq*D products, 2^-12 of the sum of the terms'
magnitudes); rows no group kept must come back bit for bit.
"""

import numpy as np
import pytest
import torch

import long_context_tsa_b200 as T
from long_context_tsa_b200 import inputs as I
from oracle import tsa_oracle as O

from .parity_util import Run, host

pytestmark = pytest.mark.gpu

DEV = "cuda"
ROUND = {"bf16": 2.0 ** -8, "f32": 2.0 ** -23}


def _inputs(w, hidden, budgets, seed, perm=None, dropped_fill=0.0):
    gen = torch.Generator(device=DEV).manual_seed(seed)
    dt = I.torch_dtype(w)
    if perm is None:
        sc = torch.rand((w.B, w.Hkv, w.L), generator=torch.Generator().manual_seed(seed))
        perm = O.select(sc.numpy(), budgets)
    attn = (0.5 * torch.randn((w.B, w.Hq, w.L, w.D), generator=gen, device=DEV)).to(dt)
    kept = O.clamp_budgets(budgets, w.L)
    for b in range(w.B):
        for g in range(w.Hkv):
            drop = torch.from_numpy(perm[b, g, int(kept[b * w.Hkv + g]):]).to(DEV)
            attn[b, g * w.G:(g + 1) * w.G].index_fill_(1, drop, dropped_fill)
    x = torch.randn((w.B, w.L, hidden), generator=gen, device=DEV).to(dt)
    wo = (torch.randn((hidden, w.Hq * w.D), generator=gen, device=DEV) / np.sqrt(w.Hq * w.D)).to(dt)
    return perm, attn, x, wo


def _kept_any(perm, budgets, B, Hkv, L):
    kept = O.clamp_budgets(budgets, L)
    m = np.zeros((B, L), bool)
    for b in range(B):
        for g in range(Hkv):
            m[b, perm[b, g, :int(kept[b * Hkv + g])]] = True
    return m


def _run(w, perm, budgets, attn, x, wo):
    desc = T.desc_for(attn, torch.empty((w.B, w.Hkv, 1, w.D)))
    ws = T.alloc_out_proj_workspace(desc, device=DEV)
    y = x.clone()
    T.tsa_out_proj(desc, attn, torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets, wo, y, ws)
    assert T.tsa_check_status(ws) == 0
    return y


def _compare(w, y, x, attn, wo, perm, budgets, rows_per_batch=None, seed=0, attn_oracle=None):
    an = host(attn if attn_oracle is None else attn_oracle)
    xn, wn, yn = host(x), host(wo), host(y)
    kept_any = _kept_any(perm, budgets, w.B, w.Hkv, w.L)
    rng = np.random.default_rng(seed)
    for b in range(w.B):
        rows = np.nonzero(kept_any[b])[0]
        if rows_per_batch is not None and rows.size > rows_per_batch:
            rows = np.unique(np.concatenate([rng.choice(rows, rows_per_batch, replace=False), rows[:2], rows[-2:]]))
        ora = O.out_proj_residual(xn, an, wn, b=b, rows=rows)
        mag = O.out_proj_residual(np.abs(xn), np.abs(an), np.abs(wn), b=b, rows=rows)
        err = np.abs(yn[b, rows].astype(np.float64) - ora)
        bound = ROUND[w.dtype] * np.abs(ora) + 2.0 ** -12 * mag + 1e-30
        assert np.all(np.isfinite(yn[b, rows]))
        assert np.all(err <= bound), f"b={b}: {int((err > bound).sum())} elements out, worst {(err / bound).max():.2f}x"
        rel = np.linalg.norm(yn[b, rows] - ora, axis=1) / np.maximum(np.linalg.norm(ora, axis=1), 1e-30)
        assert rel.max() <= (5e-3 if w.dtype == "bf16" else 1e-5), f"b={b}: row rel L2 {rel.max():.2e}"
        # Rows no group kept: the residual, bit for bit.
        untouched = torch.from_numpy(np.nonzero(~kept_any[b])[0]).to(DEV)
        assert torch.equal(y[b].index_select(0, untouched), x[b].index_select(0, untouched))


@pytest.mark.parametrize("cfg", [
    dict(B=1, Hq=8, Hkv=2, L=2000, D=128, dtype="bf16", hidden=512, budgets=[300, 1500]),
    dict(B=2, Hq=8, Hkv=8, L=777, D=64, dtype="bf16", hidden=256, budgets=[1, 50, 777, 200, 3, 9, 400, 700] * 2),
    dict(B=1, Hq=16, Hkv=1, L=300, D=128, dtype="bf16", hidden=768, budgets=[300]),
    dict(B=1, Hq=32, Hkv=8, L=4096, D=128, dtype="bf16", hidden=1024, budgets=[410] * 8),
    dict(B=2, Hq=4, Hkv=4, L=256, D=64, dtype="f32", hidden=128, budgets=[64, 1, 256, 100, 7, 80, 3, 200]),
    dict(B=1, Hq=6, Hkv=3, L=130, D=128, dtype="f32", hidden=64, budgets=[129, 2, 64]),
])
def test_out_proj_small_all_rows(cfg):
    c = dict(cfg)
    hidden, budgets = c.pop("hidden"), c.pop("budgets")
    w = I.custom("op", W=1, sigma=1.0, **c)
    perm, attn, x, wo = _inputs(w, hidden, budgets, seed=hidden)
    y = _run(w, perm, budgets, attn, x, wo)
    _compare(w, y, x, attn, wo, perm, budgets)


def test_out_proj_does_not_read_dropped_rows():
    # NaN at every dropped row of attn_out: the result must not see them.
    w = I.custom("op_nan", B=1, Hq=8, Hkv=2, L=1000, D=128, dtype="bf16", W=1, sigma=1.0)
    budgets = [100, 600]
    perm, attn, x, wo = _inputs(w, 512, budgets, seed=5, dropped_fill=float("nan"))
    y = _run(w, perm, budgets, attn, x, wo)
    clean = torch.nan_to_num(attn, nan=0.0)
    _compare(w, y, x, clean, wo, perm, budgets)


def test_out_proj_after_attend_at_128k():
    # The bench layer: tsa_forward's output projected with a seeded 4096 x 4096 weight;
    # 512 sampled kept rows (plus the first and last two) against the oracle on the
    # same bf16 attention output, and every untouched row checked.
    w = I.WORKLOADS["gqa_bf16_L131072"]
    q, k, v = I.make_qkv(w, seed=0, device=DEV)
    budgets = w.budgets()
    r = Run(w, q, k, v)
    _, perm_d, out = r.forward(budgets)
    perm = host(perm_d).astype(np.int64)
    gen = torch.Generator(device=DEV).manual_seed(31)
    hidden = w.Hq * w.D
    x = torch.randn((w.B, w.L, hidden), generator=gen, device=DEV).to(torch.bfloat16)
    wo = (torch.randn((hidden, hidden), generator=gen, device=DEV) / np.sqrt(hidden)).to(torch.bfloat16)
    y = _run(w, perm, budgets, out, x, wo)
    _compare(w, y, x, out, wo, perm, budgets, rows_per_batch=512, seed=3)


def test_out_proj_rejects_bad_shapes():
    w = I.custom("op_bad", B=1, Hq=4, Hkv=4, L=64, D=64, dtype="bf16", W=1, sigma=1.0)
    perm, attn, x, wo = _inputs(w, 256, [8] * 4, seed=1)
    desc = T.desc_for(attn, torch.empty((1, 4, 1, 64)))
    ws = T.alloc_out_proj_workspace(desc, device=DEV)
    bad_x = torch.zeros((1, 64, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(T.TsaError):  # hidden 128 is not a multiple of 256 on the tensor-core path
        T.tsa_out_proj(desc, attn, torch.from_numpy(perm.astype(np.int32)).to(DEV), [8] * 4,
                       torch.zeros((128, 256), dtype=torch.bfloat16, device=DEV), bad_x, ws)
    with pytest.raises(T.TsaError):
        T.tsa_out_proj(desc, attn, torch.from_numpy(perm.astype(np.int32)).to(DEV), [0] * 4, wo, x, ws)
