"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Stage-wise: scores (same q, k), selection (same float32 score tensor, produced
by the input generator or by the oracle), attention (same permutation, produced
by the oracle).  End to end: tsa_forward vs the oracle's forward.
"""

import numpy as np
import pytest
import torch

import long_context_tsa_b200 as T
from long_context_tsa_b200 import inputs as I
from oracle import tsa_oracle as O

from .parity_util import (Run, assert_dropped_rows_zero, assert_rows_close, assert_scores_close, compare_attend,
                          host)

pytestmark = pytest.mark.gpu

DEV = "cuda"

# Small shapes the oracle finishes in seconds, spanning several tiles with ragged tails.
SMALL = [
    I.WORKLOADS["tiny_fp32_L256"],
    I.custom("bf16_L1000_G4_D128", Hq=8, Hkv=2, L=1000, D=128, dtype="bf16", W=64, keep=0.333, sigma=0.5),
    I.custom("bf16_L777_G1_D64", Hq=3, Hkv=3, L=777, D=64, dtype="bf16", W=20, keep=0.6, sigma=1.0),
    I.custom("bf16_L2050_G8_D128_B2", B=2, Hq=16, Hkv=2, L=2050, D=128, dtype="bf16", W=32, keep=0.27, sigma=0.5,
             planted=16),
    I.custom("f32_L513_G2_D128", Hq=4, Hkv=2, L=513, D=128, dtype="f32", W=40, keep=0.5, sigma=1.0),
    I.custom("bf16_L300_G16_D64", Hq=16, Hkv=1, L=300, D=64, dtype="bf16", W=16, keep=0.9, sigma=0.5),
]


def _inputs(w, seed=0):
    q, k, v = I.make_qkv(w, seed=seed, device=DEV)
    return q, k, v, host(q), host(k), host(v)


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_score_matches_oracle(w):
    q, k, v, qn, kn, vn = _inputs(w)
    r = Run(w, q, k, v)
    gpu = host(r.score())
    ora = O.score(qn, kn, w.W)
    assert_scores_close(gpu, ora)
    np.testing.assert_allclose(gpu.sum(-1), w.W * w.G, rtol=1e-5)


@pytest.mark.parametrize("L", [1, 2, 7, 256, 1000, 8193, 131072])
@pytest.mark.parametrize("kind", ["random", "ties", "equal", "zeros", "denorm"])
def test_select_bit_exact_on_same_scores(L, kind):
    Hkv = 3
    s = I.make_scores(1, Hkv, L, seed=L, kind=kind)
    budgets = [1, max(1, L - 1), max(1, (L * 3) // 7)]
    w = I.custom(Hq=Hkv, Hkv=Hkv, L=L, D=64, dtype="f32", W=1)
    z = torch.zeros((1, Hkv, L, 64), device=DEV)
    r = Run(w, z, z, z)
    perm = host(r.select(s.to(DEV), budgets))
    ora = O.select(s.numpy(), budgets)
    np.testing.assert_array_equal(perm, ora)


def test_select_clamps_and_keeps_everything():
    L = 5000
    s = I.make_scores(2, 2, L, seed=1, kind="ties")
    w = I.custom(B=2, Hq=2, Hkv=2, L=L, D=64, dtype="f32", W=1)
    z = torch.zeros((2, 2, L, 64), device=DEV)
    r = Run(w, z, z, z)
    budgets = [L, 10 * L, 1, 4999]
    np.testing.assert_array_equal(host(r.select(s.to(DEV), budgets)), O.select(s.numpy(), budgets))


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_select_on_oracle_scores(w):
    q, k, v, qn, kn, vn = _inputs(w, seed=1)
    s32 = O.score(qn, kn, w.W).astype(np.float32)
    budgets = w.budgets()
    r = Run(w, q, k, v)
    perm = host(r.select(torch.from_numpy(s32).to(DEV), budgets))
    np.testing.assert_array_equal(perm, O.select(s32, budgets))


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_attend_matches_oracle_all_rows(w):
    q, k, v, qn, kn, vn = _inputs(w, seed=2)
    budgets = w.budgets()
    perm = O.select(O.score(qn, kn, w.W).astype(np.float32), budgets)
    r = Run(w, q, k, v)
    out = r.attend(torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets)
    compare_attend(out, qn, kn, vn, perm, budgets, w.dtype)
    assert_dropped_rows_zero(out, torch.from_numpy(perm).to(DEV), budgets, w.G)


@pytest.mark.parametrize("w", SMALL[:4], ids=lambda w: w.name)
def test_attend_ragged_budgets_and_random_subsets(w):
    q, k, v, qn, kn, vn = _inputs(w, seed=3)
    rng = np.random.default_rng(5)
    budgets = [int(x) for x in rng.integers(1, w.L + 1, size=w.B * w.Hkv)]
    budgets[0] = 1
    perm = O.select(rng.random((w.B, w.Hkv, w.L)).astype(np.float32), budgets)
    r = Run(w, q, k, v)
    out = r.attend(torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets)
    compare_attend(out, qn, kn, vn, perm, budgets, w.dtype)
    assert_dropped_rows_zero(out, torch.from_numpy(perm).to(DEV), budgets, w.G)


@pytest.mark.parametrize("w", SMALL[:3], ids=lambda w: w.name)
def test_attend_keep_all_is_dense_causal(w):
    q, k, v, qn, kn, vn = _inputs(w, seed=4)
    budgets = [w.L] * (w.B * w.Hkv)
    perm = np.broadcast_to(np.arange(w.L, dtype=np.int64), (w.B, w.Hkv, w.L)).copy()
    r = Run(w, q, k, v)
    out = r.attend(torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets)
    compare_attend(out, qn, kn, vn, perm, budgets, w.dtype)


def _first_disagreement(p_gpu, p_ora, K):
    a, b = np.sort(p_gpu[:K]), np.sort(p_ora[:K])
    if np.array_equal(a, b):
        return None
    sa, sb = set(a.tolist()), set(b.tolist())
    return min(sa ^ sb)


def check_forward(w, q, k, v, qn, kn, vn, budgets, rows_per_head=None):
    r = Run(w, q, k, v)
    scores, perm, out = r.forward(budgets)
    ora_s = O.score(qn, kn, w.W)
    assert_scores_close(host(scores), ora_s)
    ora_s32 = ora_s.astype(np.float32)
    ora_perm = O.select(ora_s32, budgets)
    gp = host(perm).astype(np.int64)
    # The selection from the GPU's own float32 scores must be the oracle's
    # selection of those same scores, bit for bit.
    np.testing.assert_array_equal(gp, O.select(host(scores), budgets))
    kept = O.clamp_budgets(budgets, w.L)
    assert_dropped_rows_zero(out, perm, budgets, w.G)
    rng = np.random.default_rng(11)
    for b in range(w.B):
        for g in range(w.Hkv):
            K = int(kept[b * w.Hkv + g])
            first = _first_disagreement(gp[b, g], ora_perm[b, g], K)
            if first is not None:
                # Differences may only involve near-ties at the K-th score.
                thr = np.sort(ora_s[b, g])[::-1][K - 1]
                diff = set(gp[b, g, :K].tolist()) ^ set(ora_perm[b, g, :K].tolist())
                for j in diff:
                    assert abs(ora_s[b, g, j] - thr) <= 2 * 1e-4 * thr, (b, g, j)
            # Compare rows whose visible key set is identical on both sides.
            limit = K if first is None else int(np.searchsorted(gp[b, g, :K], first))
            if limit == 0:
                continue
            rows = np.arange(limit)
            if rows_per_head is not None and limit > rows_per_head:
                rows = np.unique(np.concatenate([rng.choice(limit, rows_per_head, replace=False), [0, limit - 1]]))
            for h in range(g * w.G, (g + 1) * w.G):
                ora = O.attend_rows(qn, kn, vn, ora_perm[b, g], K, b, h, w.G, rows)
                pos = torch.from_numpy(ora_perm[b, g, rows]).to(DEV)
                assert_rows_close(host(out[b, h].index_select(0, pos)), ora, w.dtype, f"b={b} h={h}")


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_forward_matches_oracle(w):
    q, k, v, qn, kn, vn = _inputs(w, seed=6)
    check_forward(w, q, k, v, qn, kn, vn, w.budgets())


def test_edge_shapes():
    # L = 1 (one token, K = 1), window = L, budget above L (clamped).
    for (L, W, Kb) in [(1, 1, 1), (5, 5, 100), (64, 64, 64), (129, 1, 2)]:
        w = I.custom(Hq=4, Hkv=2, L=L, D=128, dtype="bf16", W=W, sigma=0.5)
        q, k, v, qn, kn, vn = _inputs(w, seed=L)
        check_forward(w, q, k, v, qn, kn, vn, [Kb, max(1, Kb // 2)])


@pytest.mark.parametrize("spikes", [[0], [40], [128 + 40], [128 + 100, 256 + 5], [384 + 70, 640 + 127]])
def test_attend_logit_spikes_force_rescales(spikes):
    # A kept key whose logit jumps far above the running row max (q.k = 4 * 40 = 160,
    # i.e. ~20 in log2 units after the 1/sqrt(128) scale, far above the rescale
    # threshold of 8) makes every later query row move its softmax reference
    # mid-tile, including after earlier 32-column chunks of the tile were written.
    w = I.custom("spikes", Hq=8, Hkv=2, L=900, D=128, dtype="bf16", W=16, sigma=0.3)
    q, k, v = I.make_qkv(w, seed=7, device="cpu")
    u = torch.randn(128, generator=torch.Generator().manual_seed(3))
    u = u / u.norm()
    q = (q.float() + 4.0 * u).to(torch.bfloat16)  # every query leans on u
    budgets = [800, 777]
    perm = O.select(np.random.default_rng(4).random((1, 2, 900)).astype(np.float32), budgets)
    k = k.float()
    for g in range(2):
        for c in spikes:
            if c < budgets[g]:
                k[0, g, perm[0, g, c]] += 40.0 * u
    k = k.to(torch.bfloat16)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    r = Run(w, qd, kd, vd)
    out = r.attend(torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets)
    compare_attend(out, host(q), host(k), host(v), perm, budgets, "bf16")
    assert_dropped_rows_zero(out, torch.from_numpy(perm).to(DEV), budgets, w.G)


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_attend_accumulate_scatter_adds(w):
    # Scatter-add into an existing output: kept rows gain their attention row,
    # dropped rows keep their previous value bit for bit.
    q, k, v, qn, kn, vn = _inputs(w, seed=8)
    rng = np.random.default_rng(9)
    budgets = [int(x) for x in rng.integers(1, w.L + 1, size=w.B * w.Hkv)]
    perm = O.select(rng.random((w.B, w.Hkv, w.L)).astype(np.float32), budgets)
    base = torch.randn(q.shape, generator=torch.Generator().manual_seed(10)).to(q.dtype).to(DEV)
    out = base.clone()
    r = Run(w, q, k, v)
    T.tsa_attend_accumulate(r.desc, q, k, v, torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets, out, r.ws)
    assert r.status() == 0
    ora = O.attend_accumulate(host(base), qn, kn, vn, perm, budgets)
    got = host(out)
    kept = O.clamp_budgets(budgets, w.L)
    for b in range(w.B):
        for h in range(w.Hq):
            g = h // w.G
            K = int(kept[b * w.Hkv + g])
            rows = perm[b, g, :K]
            assert_rows_close(got[b, h, rows], ora[b, h, rows], w.dtype, f"b={b} h={h}")
            drop = torch.from_numpy(perm[b, g, K:]).to(DEV)
            assert torch.equal(out[b, h].index_select(0, drop), base[b, h].index_select(0, drop)), (b, h)


def _block_mask(w, density, seed, kill_first_diag=False):
    nb = -(-w.L // 128)
    rng = np.random.default_rng(seed)
    bm = (rng.random((w.B, w.Hkv, nb, nb)) < density).astype(np.uint8)
    idx = np.arange(nb)
    bm[:, :, idx, idx] = 1  # the diagonal on ...
    if kill_first_diag:
        bm[:, 0, 0, 0] = 0  # ... except block 0 of group 0: its rows see no key at all
    return bm


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("density", [0.0, 0.4, 1.0])
def test_attend_block_sparse_matches_oracle(w, density):
    q, k, v, qn, kn, vn = _inputs(w, seed=12)
    rng = np.random.default_rng(13)
    budgets = [int(x) for x in rng.integers(1, w.L + 1, size=w.B * w.Hkv)]
    perm = O.select(rng.random((w.B, w.Hkv, w.L)).astype(np.float32), budgets)
    bm = _block_mask(w, density, seed=14, kill_first_diag=density == 0.4)
    r = Run(w, q, k, v)
    r.out.fill_(float("nan"))
    T.tsa_attend_block_sparse(r.desc, q, k, v, torch.from_numpy(perm.astype(np.int32)).to(DEV), budgets,
                              torch.from_numpy(bm).to(DEV), r.out, r.ws)
    assert r.status() == 0
    ora = O.attend_block_sparse(qn, kn, vn, perm, budgets, bm)
    got = host(r.out)
    kept = O.clamp_budgets(budgets, w.L)
    for b in range(w.B):
        for h in range(w.Hq):
            g = h // w.G
            rows = perm[b, g, :int(kept[b * w.Hkv + g])]
            assert_rows_close(got[b, h, rows], ora[b, h, rows], w.dtype, f"b={b} h={h}")
    assert_dropped_rows_zero(r.out, torch.from_numpy(perm).to(DEV), budgets, w.G)
    if density == 0.4:  # rows with no visible key are exact zeros
        rows0 = perm[0, 0, :min(128, int(kept[0]))]
        assert np.all(got[0, :w.G][:, rows0] == 0.0)


def test_attend_block_sparse_full_mask_equals_attend():
    w = SMALL[3]
    q, k, v, qn, kn, vn = _inputs(w, seed=15)
    budgets = w.budgets()
    perm_t = torch.from_numpy(O.select(O.score(qn, kn, w.W).astype(np.float32), budgets).astype(np.int32)).to(DEV)
    r = Run(w, q, k, v)
    dense = r.attend(perm_t, budgets).clone()
    nb = -(-w.L // 128)
    ones = torch.ones((w.B, w.Hkv, nb, nb), dtype=torch.uint8, device=DEV)
    T.tsa_attend_block_sparse(r.desc, q, k, v, perm_t, budgets, ones, r.out, r.ws)
    assert r.status() == 0
    assert torch.equal(r.out, dense)  # the same kernel path, bit for bit


@pytest.mark.parametrize("spike_pos", [700, 1500, 2900])
def test_score_logit_far_above_the_running_max(spike_pos):
    # One key whose logit exceeds every earlier key of the window rows by ~200 in
    # log2 units (q.k = 40 * 40 = 1600, x scale * log2(e) ~ 0.1275): in the row-
    # statistics pass the tile holding it starts far above the running reference,
    # the sum leaves the safe range (or saturates at 2^127 in the FMA-pipe lanes)
    # and the tile is redone against its own maximum.
    w = I.custom("score_spike", Hq=4, Hkv=1, L=3000, D=128, dtype="bf16", W=32, sigma=0.3)
    q, k, v = I.make_qkv(w, seed=21, device="cpu")
    u = torch.randn(128, generator=torch.Generator().manual_seed(22))
    u = u / u.norm()
    q = q.float()
    q[0, :, w.L - w.W:] += 40.0 * u  # every window row points along u
    k = k.float()
    k[0, 0, spike_pos] += 40.0 * u
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    r = Run(w, q.to(DEV), k.to(DEV), v.to(DEV))
    gpu = host(r.score())
    ora = O.score(host(q), host(k), w.W)
    assert_scores_close(gpu, ora)
    assert gpu[0, 0, spike_pos] > 0.99 * w.W * w.G  # the spike takes nearly all of the mass
