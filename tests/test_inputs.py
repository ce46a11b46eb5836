"""The seeded input generator: shapes, dtypes, determinism and the planted structure."""

import math

import torch

from long_context_tsa_b200 import inputs as I


def test_workload_table_matches_recipe():
    w = I.WORKLOADS["tiny_fp32_L256"]
    assert (w.B, w.Hq, w.Hkv, w.L, w.D, w.dtype, w.W) == (1, 4, 4, 256, 64, "f32", 16)
    assert w.budgets() == [64] * 4
    assert I.WORKLOADS["gqa_bf16_L8192"].budgets() == [4096] * 8
    assert I.WORKLOADS["gqa_bf16_L32768"].budgets() == [8192] * 8
    assert I.WORKLOADS["gqa_bf16_L131072"].budgets() == [13107] * 8
    rb = I.WORKLOADS["ragged_bf16_L131072"].budgets(seed=0)
    assert len(rb) == 8 and all(6553 <= x <= 65536 for x in rb) and len(set(rb)) > 1
    assert [I.sweep_budget(t, 131072) for t in I.SWEEP_TAUS] == [65536, 32768, 13107, 6553]


def test_make_qkv_is_seeded_and_shaped():
    w = I.custom(Hq=4, Hkv=2, L=64, D=16, dtype="bf16", W=8, sigma=0.5)
    q, k, v = I.make_qkv(w, seed=3)
    assert q.shape == (1, 4, 64, 16) and k.shape == (1, 2, 64, 16) and v.shape == k.shape
    assert q.dtype == torch.bfloat16 and q.is_contiguous()
    q2, k2, v2 = I.make_qkv(w, seed=3)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    q3, _, _ = I.make_qkv(w, seed=4)
    assert not torch.equal(q, q3)


def test_planted_keys_stand_out():
    w = I.custom(Hq=4, Hkv=2, L=512, D=128, dtype="f32", W=16, sigma=0.5, planted=8, sinks=4)
    q, k, _ = I.make_qkv(w, seed=0)
    # Logit of the last window query against each key, per KV group: the planted
    # keys and the sinks carry the shared bias and score ~9 sigma^2 sqrt(d) higher.
    for g in range(2):
        lg = (k[0, g] @ q[0, 2 * g, -1]) / math.sqrt(128)
        top = torch.topk(lg, 12).indices.tolist()
        assert {0, 1, 2, 3} <= set(top)
