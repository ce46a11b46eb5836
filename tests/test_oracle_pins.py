"""Pins for the fp64 oracle: each check is fixed by the pages or by mathematics,
never by the oracle itself.

Sources: "Token Sparse Attention Long Context" (skillsdirectory skill page),
Step 1 (``score_tokens`` "entropy", ``select_top_k``), Step 2 (``gather_tokens``,
``scatter_attention_output``), Step 3 (``SparseAttentionHead.forward``);
"Token Sparse Attention: Efficient Long-Context Inference with Interleaved
Token Selection" (sciencestack), Figure 3.

The pages print no worked numeric example; the fixed values below are closed
forms derived by hand, exhaustive enumeration on tiny inputs, and PyTorch's own
scaled-dot-product attention (an independent library routine).
"""

import itertools
import math

import numpy as np
import pytest
import torch

from oracle import tsa_oracle as O

rng = np.random.default_rng(1234)


# ----------------------------------------------------------------------------- score


def test_score_total_mass_is_window_times_group():
    # Every window query's softmax sums to 1, so a KV group's scores sum to W * G.
    B, Hq, Hkv, L, D, W = 2, 4, 2, 40, 8, 5
    q = rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    s = O.score(q, k, W)
    assert s.shape == (B, Hkv, L)
    np.testing.assert_allclose(s.sum(-1), W * (Hq // Hkv), rtol=0, atol=1e-12)
    assert np.all(s >= 0)


@pytest.mark.parametrize("W", [1, 3, 17, 24])
def test_score_zero_queries_harmonic_closed_form(W):
    # q = 0 makes every visible logit 0: the window query at position p spreads
    # 1/(p+1) over keys 0..p.  So score_g[j] = G * sum_{p >= max(j, L-W)} 1/(p+1).
    # Dropping the causal mask would give the flat value W*G/L instead.
    B, Hq, Hkv, L, D = 1, 2, 1, 24, 4
    q = np.zeros((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    s = O.score(q, k, W)
    G = Hq // Hkv
    want = np.array([G * sum(1.0 / (p + 1) for p in range(max(j, L - W), L)) for j in range(L)])
    np.testing.assert_allclose(s[0, 0], want, rtol=1e-13, atol=1e-15)


def test_score_two_token_hand_worked():
    # L=2, W=2, d=4, scale 1/sqrt(4) = 1/2.  Query 0 sees only key 0 (prob 1).
    # Query 1 = (2,0,0,0) against k0 = (1,0,0,0), k1 = 0: logits (1, 0), so
    # prob(k0) = sigmoid(1).  score = (1 + sigmoid(1), 1 - sigmoid(1)).
    q = np.zeros((1, 1, 2, 4))
    q[0, 0, 0] = [0.3, -1.0, 2.0, 0.5]
    q[0, 0, 1] = [2.0, 0.0, 0.0, 0.0]
    k = np.zeros((1, 1, 2, 4))
    k[0, 0, 0] = [1.0, 0.0, 0.0, 0.0]
    sig1 = 0.7310585786300049  # 1 / (1 + e^-1)
    s = O.score(q, k, 2)
    np.testing.assert_allclose(s[0, 0], [1.0 + sig1, 1.0 - sig1], rtol=1e-14)
    # An explicit scale of 1 doubles the logit: prob(k0) = sigmoid(2).
    sig2 = 0.8807970779778823
    s = O.score(q, k, 2, scale=1.0)
    np.testing.assert_allclose(s[0, 0], [1.0 + sig2, 1.0 - sig2], rtol=1e-14)


def test_score_gqa_groups_sum_their_own_query_heads():
    # Hq=4, Hkv=2 (G=2): query heads 0,1 use KV head 0 and heads 2,3 use KV head 1.
    # Keys are one-hot e_j; the last query of head h is a * e_{t_h}.  With W=1
    # the only window query sees all 8 keys, logits a*s at t_h and 0 elsewhere:
    # prob = e^{as}/(e^{as}+7) at t_h and 1/(e^{as}+7) elsewhere.
    L, D, a = 8, 8, 5.0
    t = [1, 2, 5, 6]
    q = np.zeros((1, 4, L, D))
    for h in range(4):
        q[0, h, L - 1, t[h]] = a
    k = np.zeros((1, 2, L, D))
    k[0, :, np.arange(L), np.arange(L)] = 1.0
    s = O.score(q, k, 1)
    e = math.exp(a / math.sqrt(D))
    hi, lo = e / (e + 7.0), 1.0 / (e + 7.0)
    for g in range(2):
        want = np.full(L, 2 * lo)
        for h in (2 * g, 2 * g + 1):
            want[t[h]] += hi - lo
        np.testing.assert_allclose(s[0, g], want, rtol=1e-14)


def test_score_only_window_queries_matter():
    B, Hq, Hkv, L, D, W = 1, 2, 2, 30, 6, 7
    q = rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    s0 = O.score(q, k, W)
    q2 = q.copy()
    q2[:, :, : L - W] = rng.standard_normal((B, Hq, L - W, D))
    np.testing.assert_array_equal(O.score(q2, k, W), s0)
    q3 = q.copy()
    q3[:, :, L - 1] += 1.0
    assert not np.allclose(O.score(q3, k, W), s0)


# ----------------------------------------------------------------------------- select


def _brute_force_topk(vals, K):
    # The max-sum K-subset; among equal sums the lexicographically smallest
    # sorted index tuple (= ties broken toward lower indices).
    best = None
    for c in itertools.combinations(range(len(vals)), K):
        key = (-sum(vals[i] for i in c), c)
        if best is None or key < best:
            best = key
    return list(best[1])


@pytest.mark.parametrize("L", range(1, 10))
def test_select_matches_exhaustive_enumeration(L):
    for trial in range(4):
        vals = rng.integers(0, 4, size=L).astype(np.float64)  # many ties
        for K in range(1, L + 1):
            perm = O.select(vals[None, None, :], [K])[0, 0]
            assert list(perm[:K]) == _brute_force_topk(list(vals), K)
            assert sorted(perm.tolist()) == list(range(L))


def test_select_invariants_random_and_ragged():
    B, Hkv, L = 2, 3, 1000
    s = rng.integers(0, 50, size=(B, Hkv, L)).astype(np.float32)
    budgets = [1, 10, 999, 1000, 5000, 333]
    perm = O.select(s, budgets)
    for i, (b, g) in enumerate(itertools.product(range(B), range(Hkv))):
        K = min(budgets[i], L)
        p = perm[b, g]
        assert sorted(p.tolist()) == list(range(L))
        sel, rest = p[:K], p[K:]
        assert np.all(np.diff(sel) > 0) and np.all(np.diff(rest) > 0)
        if K < L:
            thr = s[b, g, sel].min()
            assert thr >= s[b, g, rest].max()
            tied_sel = sel[s[b, g, sel] == thr]
            tied_rest = rest[s[b, g, rest] == thr]
            if tied_rest.size:
                assert tied_sel.max() < tied_rest.min()


def test_select_clamps_budget_to_length_and_rejects_nonpositive():
    s = rng.random((1, 1, 12)).astype(np.float32)
    np.testing.assert_array_equal(O.select(s, [99])[0, 0], np.arange(12))
    with pytest.raises(ValueError):
        O.select(s, [0])


def test_select_signed_zero_ties_and_last_bit():
    s = np.array([[[-0.0, 0.0, 1.0, -0.0, 0.0]]], dtype=np.float32)
    assert O.select(s, [3])[0, 0, :3].tolist() == [0, 1, 2]
    a = np.float32(0.1)
    b = np.nextafter(a, np.float32(1.0))  # one ulp larger in float32
    s = np.array([[[a, a, b, a]]], dtype=np.float32)
    assert O.select(s, [1])[0, 0, :1].tolist() == [2]
    assert O.select(s, [2])[0, 0, :2].tolist() == [0, 2]


# ----------------------------------------------------------------------------- attend


def _sdpa64(q, k, v, mask=None, causal=False, scale=None):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))  # noqa: E731
    G = q.shape[1] // k.shape[1]
    out = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=None if mask is None else torch.from_numpy(mask),
        is_causal=causal, scale=scale, enable_gqa=G > 1)
    return out.numpy()


def test_attend_keep_all_is_dense_causal_attention():
    # K = L: gather and scatter are identities and the op is ordinary causal
    # attention (Step 3 on the full token set), checked against PyTorch SDPA,
    # whose grouped-query mode maps query head h to KV head h // G.
    B, Hq, Hkv, L, D = 2, 4, 2, 50, 16
    q = rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    perm = np.broadcast_to(np.arange(L), (B, Hkv, L))
    out = O.attend(q, k, v, perm, [L] * (B * Hkv))
    np.testing.assert_allclose(out, _sdpa64(q, k, v, causal=True), rtol=0, atol=1e-12)


def test_attend_equals_full_length_masked_attention():
    # Attention on the compressed tensors equals full-length attention with the
    # mask M[p, r] = kept[r] and r <= p, read at the kept rows; dropped rows are 0.
    B, Hq, Hkv, L, D = 1, 4, 2, 40, 8
    q = rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    budgets = [13, 29]
    perm = O.select(rng.random((B, Hkv, L)), budgets)
    out = O.attend(q, k, v, perm, budgets)
    G = Hq // Hkv
    for g in range(Hkv):
        kept = np.zeros(L, bool)
        kept[perm[0, g, : budgets[g]]] = True
        mask = kept[None, :] & (np.arange(L)[None, :] <= np.arange(L)[:, None])
        hs = slice(g * G, (g + 1) * G)
        ref = _sdpa64(q[:, hs], k[:, g:g + 1], v[:, g:g + 1], mask=mask)
        np.testing.assert_allclose(out[0, hs][:, kept], ref[0][:, kept], rtol=0, atol=1e-12)
        assert np.all(out[0, hs][:, ~kept] == 0.0)


def test_attend_first_kept_row_copies_its_value_row():
    B, Hq, Hkv, L, D = 1, 2, 1, 20, 4
    q = rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    perm = O.select(rng.random((B, Hkv, L)), [7])
    out = O.attend(q, k, v, perm, [7])
    p0 = perm[0, 0, 0]
    for h in range(Hq):
        np.testing.assert_array_equal(out[0, h, p0], v[0, 0, p0])


def test_attend_zero_queries_give_prefix_means():
    B, Hq, Hkv, L, D, K = 1, 1, 1, 30, 5, 11
    q = np.zeros((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    perm = O.select(rng.random((B, Hkv, L)), [K])
    out = O.attend(q, k, v, perm, [K])
    vh = v[0, 0, perm[0, 0, :K]]
    want = np.cumsum(vh, axis=0) / np.arange(1, K + 1)[:, None]
    np.testing.assert_allclose(out[0, 0, perm[0, 0, :K]], want, rtol=1e-13, atol=1e-14)


def test_attend_rows_within_convex_hull_and_subset_agrees():
    B, Hq, Hkv, L, D, K = 1, 2, 1, 64, 8, 33
    q = 3.0 * rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    perm = O.select(rng.random((B, Hkv, L)), [K])
    out = O.attend(q, k, v, perm, [K])
    vh = v[0, 0, perm[0, 0, :K]]
    for i in range(K):
        row = out[0, 1, perm[0, 0, i]]
        assert np.all(row <= vh[: i + 1].max(0) + 1e-12)
        assert np.all(row >= vh[: i + 1].min(0) - 1e-12)
    rows = np.array([0, 5, 32])
    sub = O.attend_rows(q, k, v, perm[0, 0], K, 0, 1, 2, rows)
    np.testing.assert_allclose(sub, out[0, 1, perm[0, 0, rows]], rtol=0, atol=1e-14)


def test_forward_preserves_shape_and_composes():
    B, Hq, Hkv, L, D, W = 1, 4, 2, 48, 8, 6
    q = rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    sc, perm, out = O.forward(q, k, v, W, [12, 20])
    assert out.shape == (B, Hq, L, D)
    np.testing.assert_array_equal(perm, O.select(O.score(q, k, W).astype(np.float32), [12, 20]))
    np.testing.assert_array_equal(out, O.attend(q, k, v, perm, [12, 20]))


def test_attend_budget_above_length_is_clamped():
    # Step 3 of the skill page clamps the kept count to the sequence length.
    B, Hq, Hkv, L, D = 1, 2, 1, 16, 4
    q = rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    perm = np.broadcast_to(np.arange(L), (B, Hkv, L))
    np.testing.assert_array_equal(O.attend(q, k, v, perm, [10 * L]), O.attend(q, k, v, perm, [L]))
    assert O.clamp_budgets([10 * L, 3], L).tolist() == [L, 3]


def test_attend_accumulate_adds_at_kept_rows_only():
    # Step 2's scatter_add: base + attention at the kept rows; with a zero base it
    # is exactly the scatter into zeros; dropped rows keep the base bit for bit.
    B, Hq, Hkv, L, D = 1, 4, 2, 30, 8
    q = rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    budgets = [9, 17]
    perm = O.select(rng.random((B, Hkv, L)), budgets)
    zero = np.zeros((B, Hq, L, D))
    np.testing.assert_array_equal(O.attend_accumulate(zero, q, k, v, perm, budgets), O.attend(q, k, v, perm, budgets))
    base = rng.standard_normal((B, Hq, L, D))
    acc = O.attend_accumulate(base, q, k, v, perm, budgets)
    att = O.attend(q, k, v, perm, budgets)
    for g, K in enumerate(budgets):
        hs = slice(2 * g, 2 * g + 2)
        kept, drop = perm[0, g, :K], perm[0, g, K:]
        np.testing.assert_array_equal(acc[0, hs][:, drop], base[0, hs][:, drop])
        np.testing.assert_allclose(acc[0, hs][:, kept], base[0, hs][:, kept] + att[0, hs][:, kept], rtol=0, atol=1e-14)


# --- representation drift (skill page, Step 4) -------------------------------------------


def _rows(seed, shape):
    return np.random.default_rng(seed).standard_normal(shape)


def test_drift_identical_negated_and_rescaled_states():
    a = _rows(30, (2, 17, 96))
    assert abs(O.drift(a, a)) <= 1e-15
    assert abs(O.drift(a, -a) - 2.0) <= 1e-15
    # Cosine ignores each row's positive scale, however large or small (above eps).
    s = np.exp(np.random.default_rng(31).uniform(-12, 12, size=(2, 17, 1)))
    assert abs(O.drift(a, s * a)) <= 1e-14
    np.testing.assert_allclose(O.row_cosine(a, s * a), 1.0, rtol=0, atol=1e-14)


def test_drift_orthogonal_rows_is_one():
    qm, _ = np.linalg.qr(_rows(32, (64, 64)))
    a = qm[:, :32].T.reshape(1, 32, 64)  # 32 orthonormal rows
    b = qm[:, 32:].T.reshape(1, 32, 64)  # orthogonal to every row of a
    assert abs(O.drift(a, b) - 1.0) <= 1e-14


def test_drift_known_angles():
    # before = e1, after = cos(t) e1 + sin(t) e2: the row cosine is cos(t) exactly.
    t = np.linspace(0.0, np.pi, 11)
    a = np.zeros((1, 11, 8))
    b = np.zeros((1, 11, 8))
    a[0, :, 0] = 1.0
    b[0, :, 0] = np.cos(t)
    b[0, :, 1] = np.sin(t)
    np.testing.assert_allclose(O.row_cosine(a, b)[0], np.cos(t), rtol=0, atol=1e-15)
    assert abs(O.drift(a, b) - (1.0 - np.cos(t).mean())) <= 1e-15


def test_drift_matches_scipy_cosine_distance():
    from scipy.spatial.distance import cosine
    a = _rows(33, (3, 9, 40))
    b = a + 0.7 * _rows(34, (3, 9, 40))
    ref = np.mean([cosine(x, y) for x, y in zip(a.reshape(-1, 40), b.reshape(-1, 40))])
    assert abs(O.drift(a, b) - ref) <= 1e-14


def test_drift_mean_weights_every_row_equally():
    # Batch 0: identical rows (cosine 1); batch 1: negated rows (cosine -1) in 3 of 4 rows.
    a = _rows(35, (2, 4, 16))
    b = a.copy()
    b[1, :3] = -a[1, :3]
    np.testing.assert_allclose(O.row_cosine(a, b), [[1, 1, 1, 1], [-1, -1, -1, 1]], rtol=0, atol=1e-15)
    assert abs(O.drift(a, b) - (1.0 - 2.0 / 8.0)) <= 1e-15
    assert O.drift(a, b) == O.drift(b, a)


def test_drift_norm_clamped_at_eps():
    # torch.nn.functional.normalize divides by max(|x|, 1e-12): a zero row stays zero
    # (cosine 0) and a row of norm 1e-13 becomes a vector of norm 0.1.
    a = np.zeros((1, 3, 4))
    b = np.zeros((1, 3, 4))
    a[0, 0, 0] = 1e-13
    b[0, 0, 0] = 1.0
    b[0, 1, 2] = 5.0  # a[0, 1] is all zeros
    a[0, 2, 1] = b[0, 2, 1] = 3.0
    cos = O.row_cosine(a, b)[0]
    np.testing.assert_allclose(cos, [0.1, 0.0, 1.0], rtol=1e-12, atol=0)
    ta, tb = torch.from_numpy(a), torch.from_numpy(b)
    tref = (torch.nn.functional.normalize(ta, dim=-1) * torch.nn.functional.normalize(tb, dim=-1)).sum(-1)
    np.testing.assert_allclose(cos, tref.numpy()[0], rtol=1e-14, atol=0)


def test_layer_stable_window_rule():
    assert not O.layer_stable([0.01, 0.01])  # fewer drifts than the window
    assert O.layer_stable([0.9, 0.05, 0.05, 0.05])  # only the newest three count
    assert not O.layer_stable([0.05, 0.05, 0.05, 0.9])
    assert not O.layer_stable([0.25, 0.25, 0.25], threshold=0.25)  # strictly below
    assert O.layer_stable([0.2, 0.3, 0.24], threshold=0.25)  # mean 0.2467
    assert O.layer_stable([0.9, 0.01], window=1)


# --- coverage-driven budgets ---------------------------------------------------------------


def _brute_coverage(svals, tau):
    """Plain-Python restatement: integer masses, a sorted list, a linear scan."""
    L = len(svals)
    S = 55 - max(0, math.ceil(math.log2(L)))
    mass = [math.floor(min(max(float(x), 0.0), 256.0) * 2 ** S) for x in svals]
    M = sum(mass)
    T = M - math.floor(float(M) * tau)
    if T <= 0:
        return 1
    ranked = sorted(range(L), key=lambda i: (-float(svals[i]), i))
    acc = 0
    for k, i in enumerate(ranked, start=1):
        acc += mass[i]
        if acc >= T:
            return k
    raise AssertionError("unreachable: the full set carries the whole mass")


def test_coverage_brute_force_tiny():
    rng = np.random.default_rng(40)
    for trial in range(400):
        L = int(rng.integers(1, 13))
        kind = trial % 4
        if kind == 0:
            s = rng.random(L)
        elif kind == 1:
            s = rng.integers(0, 3, size=L) / 4.0  # ties and zeros
        elif kind == 2:
            s = rng.exponential(size=L) ** 4  # heavy tail
        else:
            s = np.zeros(L)
        s = s.astype(np.float32)
        tau = float(rng.choice([0.0, 0.005, 0.1, 0.25, 0.5, 0.9, 1.0, rng.random()]))
        got = O.coverage_budgets(s.reshape(1, 1, L), tau)[0]
        assert got == _brute_coverage(s, tau), (s, tau)


def test_coverage_closed_forms():
    L = 1000
    # Equal scores: every token has the same mass m, so K = ceil(T / m).
    s = np.full((1, 1, L), 0.25, dtype=np.float32)
    for tau in (0.0, 0.005, 0.3, 0.999):
        m = math.floor(0.25 * 2 ** O.coverage_shift(L))
        M = L * m
        T = M - math.floor(float(M) * tau)
        assert O.coverage_budgets(s, tau)[0] == -(-T // m)
    assert O.coverage_budgets(s, 0.0)[0] == L  # no mass may be dropped
    assert O.coverage_budgets(s, 1.0)[0] == 1  # all of it may
    # One token carries all the mass: K = 1 whatever tau.
    d = np.zeros((1, 1, L), dtype=np.float32)
    d[0, 0, 517] = 3.0
    for tau in (0.0, 0.5, 1.0):
        assert O.coverage_budgets(d, tau)[0] == 1
    # Geometric masses 2^-i at shuffled positions (exact in fixed point):
    # keeping k tokens covers (2 - 2^(1-k)) / (2 - 2^(1-n)) of the mass.
    n = 16
    g = np.zeros((1, 1, n), dtype=np.float32)
    g[0, 0, np.random.default_rng(41).permutation(n)] = 2.0 ** -np.arange(n)
    assert O.coverage_budgets(g, 0.5)[0] == 1
    assert O.coverage_budgets(g, 0.25)[0] == 2
    assert O.coverage_budgets(g, 0.1)[0] == 4
    assert O.coverage_budgets(g, 0.0)[0] == n


def test_coverage_minimality_and_monotonicity():
    rng = np.random.default_rng(42)
    L = 3000
    s = (rng.exponential(size=(2, 3, L)) ** 3).astype(np.float32)
    taus = [0.0, 0.001, 0.005, 0.05, 0.2, 0.6, 1.0]
    ks = np.stack([O.coverage_budgets(s, t) for t in taus])
    assert np.all(np.diff(ks, axis=0) <= 0)  # more coverage slack never keeps more tokens
    for t, k in zip(taus, ks):
        for bg, K in enumerate(k):
            b, g = divmod(bg, 3)
            m = O.token_mass(s[b, g], L)
            M = int(m.sum())
            T = M - math.floor(float(M) * t)
            perm = O.select(s[b:b + 1, g:g + 1], [int(K)])[0, 0]
            top = int(m[perm[:K]].sum())
            assert top >= T  # K tokens reach the target ...
            if K > 1:  # ... and the best K - 1 do not
                best = np.sort(m)[::-1][:K - 1]
                assert int(best.sum()) < T


# --- block-sparse composition --------------------------------------------------------------


def _block_full_mask(perm_bg, K, L, bm):
    """Full-length boolean mask M[p, p'] of block-sparse attention in the compressed
    space, written out in original coordinates from first principles."""
    M = np.zeros((L, L), dtype=bool)
    pos = perm_bg[:K]
    for i in range(K):
        for r in range(i + 1):  # causal on compacted indices
            if bm[i // 128, r // 128]:
                M[pos[i], pos[r]] = True
    return M


def test_block_sparse_matches_sdpa_with_explicit_mask():
    B, Hq, Hkv, L, D = 1, 2, 1, 700, 8
    q = rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    budgets = [600]
    perm = O.select(rng.random((B, Hkv, L)), budgets)
    nb = -(-L // 128)
    bm = rng.random((B, Hkv, nb, nb)) < 0.5
    bm[0, 0, 2, 2] = False  # a diagonal block off: its early rows see only earlier blocks
    bm[0, 0, 0, 0] = False  # block 0 sees nothing at all: its rows are zeros
    out = O.attend_block_sparse(q, k, v, perm, budgets, bm)
    M = _block_full_mask(perm[0, 0], 600, L, bm[0, 0])
    rows = M.any(axis=1)
    ref = _sdpa64(q, k, v, mask=M)
    np.testing.assert_allclose(out[0][:, rows], ref[0][:, rows], rtol=0, atol=1e-12)
    kept = np.zeros(L, bool)
    kept[perm[0, 0, :600]] = True
    assert np.all(out[0][:, ~rows] == 0.0)  # no visible key, or dropped
    assert np.all(out[0][:, perm[0, 0, :128]] == 0.0)  # the rows of block 0


def test_block_sparse_full_mask_is_attend_and_diagonal_mask_is_blockwise():
    B, Hq, Hkv, L, D = 1, 4, 2, 520, 8
    q = rng.standard_normal((B, Hq, L, D))
    k = rng.standard_normal((B, Hkv, L, D))
    v = rng.standard_normal((B, Hkv, L, D))
    budgets = [400, 520]
    perm = O.select(rng.random((B, Hkv, L)), budgets)
    nb = -(-L // 128)
    full = np.ones((B, Hkv, nb, nb), dtype=np.uint8)
    np.testing.assert_array_equal(O.attend_block_sparse(q, k, v, perm, budgets, full),
                                  O.attend(q, k, v, perm, budgets))
    diag = np.broadcast_to(np.eye(nb, dtype=np.uint8), (B, Hkv, nb, nb))
    out = O.attend_block_sparse(q, k, v, perm, budgets, diag)
    for g, K in enumerate(budgets):
        for blk in range(0, K, 128):
            sub = perm[:, g:g + 1, blk:min(K, blk + 128)]  # the block as its own sequence
            n = sub.shape[-1]
            sub_perm = np.broadcast_to(np.arange(n), (1, 1, n))
            hs = slice(2 * g, 2 * g + 2)
            ref = O.attend(q[:, hs][:, :, sub[0, 0]], k[:, g:g + 1][:, :, sub[0, 0]], v[:, g:g + 1][:, :, sub[0, 0]],
                           sub_perm, [n])
            np.testing.assert_allclose(out[0, hs][:, sub[0, 0]], ref[0], rtol=0, atol=1e-12)


# --- fixed-point token masses: hand values and exact integer bounds --------------------------
#
# The coverage reading makes a token's mass the integer floor(clamp(s, 0, 256) * 2^S) with
# S = 55 - ceil(log2 L): the largest shift for which L tokens of the largest score (256) still sum
# to at most 2^63 in a 64-bit integer.  These pins do not call the oracle's formula back: they
# state hand-computed masses and check the bound with exact Python integers, so a shift off by one
# in either direction fails them (see the mutation test below).


def _mass(x, L):
    return int(O.token_mass(np.array([x], dtype=np.float32), L)[0])


def _pin_coverage_masses():
    L = 131072  # 2^17, so the shift is 55 - 17 = 38
    assert _mass(256.0, L) == 2 ** 46  # 2^8 * 2^38
    assert _mass(1.0e6, L) == 2 ** 46  # clamped at 256 first
    assert _mass(1.0, L) == 2 ** 38
    assert _mass(2.0 ** -38, L) == 1  # the smallest score that weighs anything
    assert _mass(2.0 ** -39, L) == 0
    assert _mass(3 * 2.0 ** -38, L) == 3
    assert _mass(1.5 * 2.0 ** -38, L) == 1  # floor, not round
    assert _mass(np.float32(1e-45), L) == 0  # a subnormal weighs nothing
    assert _mass(-3.0, L) == 0 and _mass(np.nan, L) == 0  # negative scores and NaN weigh nothing
    # A float32 value that is not a dyadic fraction of short length: floor of its exact product.
    from fractions import Fraction

    x = np.float32(0.1)
    assert _mass(x, L) == math.floor(Fraction(float(x)) * 2 ** 38)
    # Shifts by hand at small lengths: ceil(log2 L) = 0, 1, 2, 2, 3.
    assert _mass(256.0, 1) == 2 ** 63
    assert _mass(1.0, 2) == 2 ** 54
    assert _mass(1.0, 3) == 2 ** 53
    assert _mass(1.0, 4) == 2 ** 53
    assert _mass(1.0, 5) == 2 ** 52


def _pin_coverage_total_bound():
    lengths = [1, 2, 3, 4, 5, 7, 8, 9, 1000, 8192, 131071, 131072, 131073, 2 ** 30, 2 ** 30 + 1, 2 ** 31 - 1]
    for L in lengths:
        top = _mass(256.0, L)  # the most a single token can weigh at this length
        assert L * top <= 2 ** 63, L  # a head of L such tokens fits the 64-bit total ...
        assert 2 * L * top > 2 ** 63, L  # ... and one more bit of precision would not
    # The largest supported length: an all-256 head stays strictly below 2^63.
    L = 2 ** 31 - 1
    assert L * _mass(256.0, L) == (2 ** 31 - 1) * 2 ** 32 < 2 ** 63


def test_coverage_token_mass_hand_values():
    _pin_coverage_masses()


def test_coverage_head_total_fits_64_bits_and_shift_is_largest():
    _pin_coverage_total_bound()


@pytest.mark.filterwarnings("ignore:invalid value encountered in cast")  # 2^64 overflows the uint64 cast
@pytest.mark.parametrize("delta", [-1, 1])
def test_coverage_mass_pins_catch_a_shift_off_by_one(monkeypatch, delta):
    true_shift = O.coverage_shift
    monkeypatch.setattr(O, "coverage_shift", lambda L: true_shift(L) + delta)
    with pytest.raises(AssertionError):
        _pin_coverage_masses()
    with pytest.raises(AssertionError):
        _pin_coverage_total_bound()


# --- the composed forward against an independent construction -------------------------------


def test_forward_matches_independent_construction():
    # Score by plain loops (Step 1 written out element by element), the kept set by
    # enumerating every K-subset, and the attention by PyTorch SDPA with the mask
    # "kept and causal" written out at full length; dropped rows are zero.
    r = np.random.default_rng(77)
    B, Hq, Hkv, L, D, W = 1, 4, 2, 10, 4, 3
    G = Hq // Hkv
    q = r.standard_normal((B, Hq, L, D))
    k = r.standard_normal((B, Hkv, L, D))
    v = r.standard_normal((B, Hkv, L, D))
    budgets = [4, 6]
    s = 1.0 / math.sqrt(D)
    want_sc = np.zeros((B, Hkv, L))
    for h in range(Hq):
        g = h // G
        for p in range(L - W, L):
            logits = [s * sum(q[0, h, p, d] * k[0, g, j, d] for d in range(D)) for j in range(p + 1)]
            mx = max(logits)
            e = [math.exp(x - mx) for x in logits]
            z = sum(e)
            for j in range(p + 1):
                want_sc[0, g, j] += e[j] / z
    sc, perm, out = O.forward(q, k, v, W, budgets)
    np.testing.assert_allclose(sc, want_sc, rtol=1e-13, atol=1e-15)
    s32 = want_sc.astype(np.float32)
    for g, K in enumerate(budgets):
        kept = _brute_force_topk([float(x) for x in s32[0, g]], K)
        assert perm[0, g, :K].tolist() == kept
        assert perm[0, g, K:].tolist() == sorted(set(range(L)) - set(kept))
        keep = np.zeros(L, bool)
        keep[kept] = True
        mask = keep[None, :] & (np.arange(L)[None, :] <= np.arange(L)[:, None])
        hs = slice(g * G, (g + 1) * G)
        ref = _sdpa64(q[:, hs], k[:, g:g + 1], v[:, g:g + 1], mask=mask)
        np.testing.assert_allclose(out[0, hs][:, keep], ref[0][:, keep], rtol=0, atol=1e-12)
        assert np.all(out[0, hs][:, ~keep] == 0.0)


# --- output projection + residual (skill page Step 3, sciencestack Figure 3) ----------------


def _compress_project_scatter(x, attn_out, w_o, perm, budgets):
    # The page's order written out per head: gather the kept rows (the compressed
    # output), project them with the head's slice of the weight, scatter-add back.
    B, Hq, L, D = attn_out.shape
    Hkv = perm.shape[1]
    G = Hq // Hkv
    y = np.array(x, dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            K = min(budgets[b * Hkv + g], L)
            idx = perm[b, g, :K]
            comp = attn_out[b, h, idx, :]  # [K, D]
            proj = np.zeros((K, w_o.shape[0]))
            for i in range(K):
                for n in range(w_o.shape[0]):
                    proj[i, n] = sum(comp[i, d] * w_o[n, h * D + d] for d in range(D))
            y[b, idx, :] += proj
    return y


def test_out_proj_is_compress_project_scatter_and_torch_linear():
    r = np.random.default_rng(91)
    B, Hq, Hkv, L, D, N = 1, 4, 2, 12, 4, 6
    budgets = [5, 8]
    perm = O.select(r.random((B, Hkv, L)), budgets)
    attn = r.standard_normal((B, Hq, L, D))
    for g in range(Hkv):  # zeros at the rows each group dropped, as attend writes them
        attn[0, g * 2:(g + 1) * 2, perm[0, g, budgets[g]:], :] = 0.0
    x = r.standard_normal((B, L, N))
    w = r.standard_normal((N, Hq * D))
    got = O.out_proj_residual(x, attn, w)
    np.testing.assert_allclose(got, _compress_project_scatter(x, attn, w, perm, budgets)[0], rtol=0, atol=1e-12)
    o = torch.from_numpy(attn[0]).permute(1, 0, 2).reshape(L, Hq * D)
    ref = torch.from_numpy(x[0]) + torch.nn.functional.linear(o, torch.from_numpy(w))
    np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)
    # A row no group keeps is the residual, bit for bit; a row subset equals those rows.
    kept_any = np.zeros(L, bool)
    for g in range(Hkv):
        kept_any[perm[0, g, :budgets[g]]] = True
    np.testing.assert_array_equal(got[~kept_any], x[0][~kept_any])
    rows = np.array([0, 3, 11])
    np.testing.assert_array_equal(O.out_proj_residual(x, attn, w, rows=rows), got[rows])


def test_out_proj_identity_weight_and_zero_attention():
    r = np.random.default_rng(92)
    B, Hq, L, D = 2, 2, 5, 3
    attn = r.standard_normal((B, Hq, L, D))
    x = r.standard_normal((B, L, Hq * D))
    eye = np.eye(Hq * D)
    for b in range(B):
        # Identity weight: the heads' outputs concatenated per position, added to x.
        want = x[b] + np.concatenate([attn[b, h] for h in range(Hq)], axis=1)
        np.testing.assert_array_equal(O.out_proj_residual(x, attn, eye, b=b), want)
        # No attention output: the residual comes back unchanged.
        w = r.standard_normal((Hq * D, Hq * D))
        np.testing.assert_array_equal(O.out_proj_residual(x, np.zeros_like(attn), w, b=b), x[b])
