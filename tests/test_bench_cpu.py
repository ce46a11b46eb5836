"""Host-side helpers of bench.py: the flop and byte counts behind the reported
rooflines (no GPU needed)."""

import os

import numpy as np

import bench
from long_context_tsa_b200 import inputs as I


def test_block_sparse_flops_reduce_to_the_causal_count():
    w = I.WORKLOADS["gqa_bf16_L8192"]
    budgets = w.budgets()
    nb = -(-w.L // 128)
    ones = np.ones((w.B, w.Hkv, nb, nb), dtype=np.uint8)
    assert bench.block_sparse_flops(w, budgets, ones) == bench.attend_flops(w, budgets)


def test_block_sparse_flops_diagonal_blocks_closed_form():
    w = I.custom(Hq=8, Hkv=2, L=1000, D=128, dtype="bf16", W=16)
    budgets = [300, 1000]
    nb = -(-w.L // 128)
    diag = np.broadcast_to(np.eye(nb, dtype=np.uint8), (1, 2, nb, nb)).copy()
    want = 0.0
    for K in budgets:
        for blk in range(0, K, 128):
            n = min(128, K - blk)
            want += w.G * 4.0 * w.D * n * (n + 1) / 2
    assert bench.block_sparse_flops(w, budgets, diag) == want


def test_block_mask_for_keeps_diagonal_and_sinks():
    w = I.WORKLOADS["gqa_bf16_L8192"]
    bm = bench.block_mask_for(w, 0.3)
    nb = -(-w.L // 128)
    assert bm.shape == (w.B, w.Hkv, nb, nb) and bm.dtype == np.uint8
    assert np.all(bm[:, :, np.arange(nb), np.arange(nb)] == 1)
    assert np.all(bm[:, :, :, 0] == 1)
    frac = bm[:, :, 1:, 1:].mean()
    assert 0.25 < frac < 0.4  # roughly the requested density off the forced blocks


def test_other_rooflines_counts():
    w = I.WORKLOADS["gqa_bf16_L131072"]
    r = bench.other_rooflines(w, 0.19, 0.031, {"hbm_gbs": 6450.3}, "measured")
    score, score_hbm, select = r
    # K read once, the window queries and the scores written
    want = (8 * 131072 * 128 + 32 * 64 * 128) * 2 + 4 * 8 * 131072
    assert abs(score_hbm["achieved"] * 1e9 * 0.19e-3 - want) < 1.0 and score_hbm["bound"] == "hbm"
    # 2 passes x (B x Hkv) groups x (G x W) window rows x L keys exponentials
    assert abs(score["achieved"] * 1e12 * 0.19e-3 - 2 * 8 * 4 * 64 * 131072) < 1e3
    assert score["bound"] == "alu" and 0 < score["frac"] < 1
    # Only the exponentials the MUFU executes: the share matches the kernel's split
    # (in both passes, pair e2 of each 16-pair chunk goes to the FMA pipe when e2 % 3 == 2).
    src = open(os.path.join(os.path.dirname(bench.__file__), "long_context_tsa_b200", "csrc", "score_tc.cu")).read()
    assert src.count("if (e2 % 3 == 2) {") == 2
    assert score["mufu_share"] == sum(1 for e2 in range(16) if e2 % 3 != 2) / 16
    assert abs(score["mufu_issued_frac"] - score["frac"] * score["mufu_share"]) < 1e-12
    # scores read once and the permutation written once: 8 bytes per key per group
    assert abs(select["achieved"] * 1e9 * 0.031e-3 - 8 * 8 * 131072) < 1.0
    assert select["bound"] == "hbm" and 0 < select["frac"] < 1


def test_input_checksum_depends_on_every_element():
    import torch

    a = torch.randn(4, 8, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    b = a.clone()
    b[3, 7] = -b[3, 7]
    assert bench.input_checksum(a) == bench.input_checksum(a.clone())
    assert bench.input_checksum(a) != bench.input_checksum(b)
    assert len(bench.input_checksum(a, a.float()).split(":")) == 2
