"""tsa_forward_host: host inputs and output, two transfer paths, one result.

With pinned (device-mapped) q and v the library copies K and the window rows of
Q, then reads only the kept rows of Q and V in place after the selection; with
pageable inputs it copies everything.  Either way out_host equals the device
forward on the same inputs bit for bit (the same kernels run on the same
values), and the attention output matches the oracle through that equality.
"""

import numpy as np
import pytest
import torch

import long_context_tsa_b200 as T
from long_context_tsa_b200 import inputs as I

pytestmark = pytest.mark.gpu

DEV = "cuda"

SHAPES = [
    I.custom("host_bf16_L1000_G4_D128", Hq=8, Hkv=2, L=1000, D=128, dtype="bf16", W=64, keep=0.3, sigma=0.5),
    I.custom("host_bf16_L777_G1_D64", Hq=3, Hkv=3, L=777, D=64, dtype="bf16", W=20, keep=0.6, sigma=1.0),
    I.custom("host_bf16_L2050_G8_D128_B2", B=2, Hq=16, Hkv=2, L=2050, D=128, dtype="bf16", W=32, keep=0.27,
             sigma=0.5, planted=16),
    I.custom("host_f32_L513_G2_D128", Hq=4, Hkv=2, L=513, D=128, dtype="f32", W=40, keep=0.5, sigma=1.0),
]


def _device_forward(w, q, k, v, budgets):
    desc = T.desc_for(q, k)
    ws = T.alloc_workspace(desc, w.W, device=DEV)
    out = torch.empty_like(q)
    T.tsa_forward(desc, q, k, v, w.W, budgets, out, ws)
    assert T.tsa_check_status(ws) == 0
    return out


def _host_forward(w, qh, kh, vh, budgets, fill):
    desc = T.make_desc(w.B, w.Hq, w.Hkv, w.L, w.D, qh.dtype)
    ws = T.alloc_workspace(desc, w.W, device=DEV)
    qd = torch.full(qh.shape, fill, dtype=qh.dtype, device=DEV)
    kd = torch.empty(kh.shape, dtype=kh.dtype, device=DEV)
    vd = torch.full(vh.shape, fill, dtype=vh.dtype, device=DEV)
    od = torch.empty(qh.shape, dtype=qh.dtype, device=DEV)
    oh = torch.empty(qh.shape, dtype=qh.dtype).pin_memory()
    T.tsa_forward_host(desc, qh, kh, vh, w.W, budgets, oh, qd, kd, vd, od, ws)
    assert T.tsa_check_status(ws) == 0
    return oh, qd, T.tsa_forward_host_h2d_bytes(desc, w.W, budgets, qh, vh)


def _full_bytes(w, esz):
    return (w.B * w.Hq + 2 * w.B * w.Hkv) * w.L * w.D * esz


def _sparse_bytes(w, esz, budgets):
    kept = sum(min(int(x), w.L) for x in budgets)
    return (w.B * w.Hkv * w.L + w.B * w.Hq * w.W + kept * (w.G + 1)) * w.D * esz


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_host_forward_pinned_reads_only_kept_rows(w):
    q, k, v = I.make_qkv(w, seed=5, device=DEV)
    budgets = w.budgets()
    ref = _device_forward(w, q, k, v, budgets)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh, qd, nbytes = _host_forward(w, qh, kh, vh, budgets, fill=7.0)
    assert torch.equal(oh, ref.cpu()), "host-buffer forward differs from the device forward"
    esz = 4 if w.dtype == "f32" else 2
    assert nbytes == _sparse_bytes(w, esz, budgets)
    # A row neither kept by its group nor in the score window was never written.
    perm = torch.empty((w.B, w.Hkv, w.L), dtype=torch.int32, device=DEV)
    desc = T.desc_for(q, k)
    ws = T.alloc_workspace(desc, w.W, device=DEV)
    scores = torch.empty((w.B, w.Hkv, w.L), dtype=torch.float32, device=DEV)
    T.tsa_forward(desc, q, k, v, w.W, budgets, torch.empty_like(q), ws, scores=scores, perm=perm)
    kb = [min(int(x), w.L) for x in budgets]
    untouched = 0
    for b in range(w.B):
        for g in range(w.Hkv):
            K = kb[b * w.Hkv + g]
            for p in perm[b, g, K:].tolist()[:8]:
                if p < w.L - w.W:
                    assert torch.all(qd[b, g * w.G, p].float() == 7.0), (b, g, p)
                    untouched += 1
    assert untouched > 0 or all(K == w.L for K in kb)


@pytest.mark.parametrize("w", SHAPES[:2], ids=lambda w: w.name)
def test_host_forward_pageable_copies_everything(w):
    q, k, v = I.make_qkv(w, seed=6, device=DEV)
    budgets = w.budgets()
    ref = _device_forward(w, q, k, v, budgets)
    qh, kh, vh = (t.cpu() for t in (q, k, v))  # pageable: not mapped into the device
    oh, _, nbytes = _host_forward(w, qh, kh, vh, budgets, fill=0.0)
    assert torch.equal(oh, ref.cpu())
    assert nbytes == _full_bytes(w, 4 if w.dtype == "f32" else 2)


def test_host_forward_pinned_32768_layer():
    w = I.WORKLOADS["gqa_bf16_L32768"]
    q, k, v = I.make_qkv(w, seed=0, device=DEV)
    budgets = w.budgets()
    ref = _device_forward(w, q, k, v, budgets)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh, _, nbytes = _host_forward(w, qh, kh, vh, budgets, fill=0.0)
    assert torch.equal(oh, ref.cpu())
    assert nbytes == _sparse_bytes(w, 2, budgets)
    assert nbytes < _full_bytes(w, 2) / 2


def test_host_forward_ragged_budgets_pinned():
    w = SHAPES[2]
    q, k, v = I.make_qkv(w, seed=7, device=DEV)
    rng = np.random.default_rng(8)
    budgets = [int(x) for x in rng.integers(1, w.L + 200, size=w.B * w.Hkv)]  # some above L (clamped)
    ref = _device_forward(w, q, k, v, budgets)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh, _, nbytes = _host_forward(w, qh, kh, vh, budgets, fill=0.0)
    assert torch.equal(oh, ref.cpu())
    assert nbytes == _sparse_bytes(w, 2, budgets)
