"""Coverage-driven budgets on the GPU vs the oracle: the chosen K per KV head
and the permutation, bit for bit on the same float32 scores; and the forward
path that uses them."""

import numpy as np
import pytest
import torch

import long_context_tsa_b200 as T
from long_context_tsa_b200 import inputs as I
from oracle import tsa_oracle as O

from .parity_util import Run, assert_dropped_rows_zero, compare_attend, host

pytestmark = pytest.mark.gpu

DEV = "cuda"
TAUS = [0.0, 0.005, 0.1, 0.5, 0.9, 1.0]


def _select_coverage(scores, tau):
    B, Hkv, L = scores.shape
    w = I.custom(B=B, Hq=Hkv, Hkv=Hkv, L=L, D=64, dtype="f32", W=1)
    z = torch.zeros((B, Hkv, 1, 64), device=DEV)
    desc = T.make_desc(B, Hkv, Hkv, L, 64, T.TSA_F32)
    ws = T.alloc_workspace(desc, 1, device=DEV)
    perm = torch.full((B, Hkv, L), -1, dtype=torch.int32, device=DEV)
    kout = torch.full((B * Hkv,), -1, dtype=torch.int32, device=DEV)
    T.tsa_select_coverage(desc, scores.to(DEV), tau, perm, kout, ws)
    assert T.tsa_check_status(ws) == 0
    del w, z
    return host(kout).astype(np.int64), host(perm).astype(np.int64)


@pytest.mark.parametrize("L", [1, 2, 7, 1000, 8193, 131072])
@pytest.mark.parametrize("kind", ["random", "ties", "equal", "zeros", "denorm", "peaked"])
def test_select_coverage_bit_exact(L, kind):
    s = I.make_scores(1, 3, L, seed=L + 1, kind=kind)
    sn = s.numpy()
    for tau in TAUS:
        k_gpu, p_gpu = _select_coverage(s, tau)
        k_ora = O.coverage_budgets(sn, tau)
        np.testing.assert_array_equal(k_gpu, k_ora, err_msg=f"tau={tau}")
        np.testing.assert_array_equal(p_gpu, O.select(sn, k_ora.tolist()), err_msg=f"tau={tau}")


def test_select_coverage_batches_and_heads():
    s = I.make_scores(2, 8, 20000, seed=3, kind="peaked")
    k_gpu, p_gpu = _select_coverage(s, 0.005)
    k_ora = O.coverage_budgets(s.numpy(), 0.005)
    np.testing.assert_array_equal(k_gpu, k_ora)
    np.testing.assert_array_equal(p_gpu, O.select(s.numpy(), k_ora.tolist()))


def test_select_coverage_rejects_bad_tau():
    s = I.make_scores(1, 1, 64, kind="random").to(DEV)
    desc = T.make_desc(1, 1, 1, 64, 64, T.TSA_F32)
    ws = T.alloc_workspace(desc, 1, device=DEV)
    perm = torch.empty((1, 1, 64), dtype=torch.int32, device=DEV)
    kout = torch.empty(1, dtype=torch.int32, device=DEV)
    for tau in (-0.1, 1.5, float("nan")):
        with pytest.raises(T.TsaError):
            T.tsa_select_coverage(desc, s, tau, perm, kout, ws)


@pytest.mark.parametrize("name,tau", [("gqa_bf16_L8192", 0.005), ("gqa_bf16_L32768", 0.05)])
def test_forward_coverage(name, tau):
    w = I.WORKLOADS[name]
    q, k, v = I.make_qkv(w, seed=5, device=DEV)
    qn, kn, vn = host(q), host(k), host(v)
    r = Run(w, q, k, v)
    r.out.fill_(float("nan"))
    budgets = T.tsa_forward_coverage(r.desc, q, k, v, w.W, tau, r.out, r.ws, scores=r.scores, perm=r.perm)
    assert r.status() == 0
    sg = host(r.scores)
    # The budgets and the permutation are the oracle's on the GPU's own float32 scores.
    np.testing.assert_array_equal(np.array(budgets), O.coverage_budgets(sg, tau))
    perm = host(r.perm).astype(np.int64)
    np.testing.assert_array_equal(perm, O.select(sg, budgets))
    assert 1 <= min(budgets) and max(budgets) < w.L  # peaked scores: coverage drops tokens
    assert_dropped_rows_zero(r.out, r.perm, budgets, w.G)
    compare_attend(r.out, qn, kn, vn, perm, budgets, w.dtype, rows_per_head=512, seed=7)
