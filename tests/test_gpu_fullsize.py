"""Parity at the workloads' full sizes, in the launch configuration bench.py times.

Scores are compared in full (the oracle's window scoring is cheap); the
selection bit for bit on a shared float32 score tensor; attention on a seeded
sample of kept rows per head (always including the first and last kept rows),
computed one by one by the oracle on the same permutation; dropped rows in full.
"""

import numpy as np
import pytest
import torch

import long_context_tsa_b200 as T
from long_context_tsa_b200 import inputs as I
from oracle import tsa_oracle as O

from .parity_util import Run, assert_dropped_rows_zero, assert_rows_close, assert_scores_close, compare_attend, host

pytestmark = pytest.mark.gpu

DEV = "cuda"
ROWS = 512  # sampled kept rows per query head (plus the first four -- kept sinks sit there -- and the last)


def _setup(name, seed=0):
    w = I.WORKLOADS[name]
    q, k, v = I.make_qkv(w, seed=seed, device=DEV)
    return w, q, k, v, host(q), host(k), host(v)


@pytest.mark.parametrize("name", ["gqa_bf16_L8192", "gqa_bf16_L32768", "gqa_bf16_L131072"])
def test_forward_full_size(name):
    w, q, k, v, qn, kn, vn = _setup(name)
    budgets = w.budgets()
    r = Run(w, q, k, v)
    scores, perm, out = r.forward(budgets)  # the path bench.py times
    perm = perm.clone()  # r.select below reuses the run's permutation buffer
    assert_dropped_rows_zero(out, perm, budgets, w.G)
    ora_s = O.score(qn, kn, w.W)
    sg = host(scores)
    assert_scores_close(sg, ora_s)
    np.testing.assert_allclose(sg.sum(-1), w.W * w.G, rtol=1e-4)
    # Selection: bit-exact given the same float32 score tensor.
    np.testing.assert_array_equal(host(perm).astype(np.int64), O.select(sg, budgets))
    s32 = ora_s.astype(np.float32)
    ora_perm = O.select(s32, budgets)
    np.testing.assert_array_equal(host(r.select(torch.from_numpy(s32).to(DEV), budgets)), ora_perm)
    # Attention on the oracle's permutation, sampled rows.
    out = r.attend(torch.from_numpy(ora_perm.astype(np.int32)).to(DEV), budgets)
    compare_attend(out, qn, kn, vn, ora_perm, budgets, w.dtype, rows_per_head=ROWS, seed=1)
    assert_dropped_rows_zero(out, torch.from_numpy(ora_perm).to(DEV), budgets, w.G)


def test_ragged_budgets_and_sparsity_sweep_131072():
    w, q, k, v, qn, kn, vn = _setup("ragged_bf16_L131072")
    r = Run(w, q, k, v)
    s32 = O.score(qn, kn, w.W).astype(np.float32)
    sweeps = [w.budgets(seed=0)] + [[I.sweep_budget(t, w.L)] * (w.B * w.Hkv) for t in I.SWEEP_TAUS]
    for budgets in sweeps:
        perm = O.select(s32, budgets)
        np.testing.assert_array_equal(host(r.select(torch.from_numpy(s32).to(DEV), budgets)), perm)
        out = r.attend(torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets)
        compare_attend(out, qn, kn, vn, perm, budgets, w.dtype, rows_per_head=ROWS, seed=2)
        assert_dropped_rows_zero(out, torch.from_numpy(perm).to(DEV), budgets, w.G)


def test_dense_keep_all_131072():
    # K = L through the same library: identity permutation, ordinary causal attention.
    w, q, k, v, qn, kn, vn = _setup("gqa_bf16_L131072", seed=3)
    budgets = [w.L] * (w.B * w.Hkv)
    perm = np.broadcast_to(np.arange(w.L, dtype=np.int64), (w.B, w.Hkv, w.L)).copy()
    r = Run(w, q, k, v)
    out = r.attend(torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets)
    compare_attend(out, qn, kn, vn, perm, budgets, w.dtype, rows_per_head=ROWS, seed=3)


def test_block_sparse_131072():
    # Block-sparse composition at the bench size: diagonal blocks, the first block
    # column (sinks) and a seeded half of the other causal blocks.
    w, q, k, v, qn, kn, vn = _setup("gqa_bf16_L131072", seed=4)
    budgets = w.budgets()
    perm = O.select(O.score(qn, kn, w.W).astype(np.float32), budgets)
    nb = -(-w.L // 128)
    rng = np.random.default_rng(5)
    bm = (rng.random((w.B, w.Hkv, nb, nb)) < 0.5).astype(np.uint8)
    bm[:, :, np.arange(nb), np.arange(nb)] = 1
    bm[:, :, :, 0] = 1
    r = Run(w, q, k, v)
    r.out.fill_(float("nan"))
    T.tsa_attend_block_sparse(r.desc, q, k, v, torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets,
                              torch.from_numpy(bm).to(DEV), r.out, r.ws)
    assert r.status() == 0
    kept = O.clamp_budgets(budgets, w.L)
    rs = np.random.default_rng(6)
    for h in range(w.Hq):
        g = h // w.G
        K = int(kept[g])
        rows = np.unique(np.concatenate([rs.choice(K, ROWS, replace=False), np.arange(4), [K - 1]]))
        ora = O.attend_rows(qn, kn, vn, perm[0, g], K, 0, h, w.G, rows, block_mask_bg=bm[0, g])
        pos = torch.from_numpy(perm[0, g, rows]).to(DEV)
        assert_rows_close(host(r.out[0, h].index_select(0, pos)), ora, w.dtype, f"h={h}")
    assert_dropped_rows_zero(r.out, torch.from_numpy(perm).to(DEV), budgets, w.G)


def test_accumulate_8192_many_items_per_cta():
    # 512 work items on at most 148 persistent CTAs: every kept row must be added
    # exactly once (a repeated item would add its rows twice), dropped rows untouched.
    w, q, k, v, qn, kn, vn = _setup("gqa_bf16_L8192", seed=6)
    budgets = w.budgets()
    perm = O.select(np.random.default_rng(7).random((w.B, w.Hkv, w.L)).astype(np.float32), budgets)
    base = torch.randn(q.shape, generator=torch.Generator().manual_seed(8)).to(q.dtype).to(DEV)
    out = base.clone()
    r = Run(w, q, k, v)
    T.tsa_attend_accumulate(r.desc, q, k, v, torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets, out, r.ws)
    assert r.status() == 0
    kept = O.clamp_budgets(budgets, w.L)
    bn = host(base)
    rs = np.random.default_rng(9)
    for h in range(w.Hq):
        g = h // w.G
        K = int(kept[g])
        rows = np.unique(np.concatenate([rs.choice(K, ROWS, replace=False), np.arange(4), [K - 1]]))
        ora = bn[0, h, perm[0, g, rows]] + O.attend_rows(qn, kn, vn, perm[0, g], K, 0, h, w.G, rows)
        pos = torch.from_numpy(perm[0, g, rows]).to(DEV)
        assert_rows_close(host(out[0, h].index_select(0, pos)), ora, w.dtype, f"h={h}")
        drop = torch.from_numpy(perm[0, g, K:]).to(DEV)
        assert torch.equal(out[0, h].index_select(0, drop), base[0, h].index_select(0, drop))


@pytest.mark.parametrize("name", ["tiny_fp32_L256", "gqa_bf16_L131072", "ragged_bf16_L131072"])
def test_zero_dropped_standalone(name):
    # The scatter's zero rows on their own: +0 at every dropped row of every query
    # head, kept rows left exactly as they were.
    w = I.WORKLOADS[name]
    q, k, _ = I.make_qkv(w, seed=0, device=DEV)
    budgets = w.budgets(seed=1)
    perm = O.select(np.random.default_rng(11).random((w.B, w.Hkv, w.L)).astype(np.float32), budgets)
    perm_d = torch.from_numpy(perm.astype(np.int32)).to(DEV)
    base = torch.randn(q.shape, generator=torch.Generator(device=DEV).manual_seed(12), device=DEV).to(q.dtype)
    out = base.clone()
    desc = T.desc_for(q, k)
    ws = T.alloc_workspace(desc, w.W, device=DEV)
    T.tsa_zero_dropped(desc, perm_d, budgets, out, ws)
    assert T.tsa_check_status(ws) == 0
    assert_dropped_rows_zero(out, perm_d, budgets, w.G)
    kept = O.clamp_budgets(budgets, w.L)
    for g in range(w.Hkv):
        keep = torch.from_numpy(perm[0, g, :int(kept[g])]).to(DEV)
        hs = slice(g * w.G, (g + 1) * w.G)
        assert torch.equal(out[0, hs].index_select(1, keep), base[0, hs].index_select(1, keep))
