"""The library on KV-group slices of one layer reproduces the whole-layer call bit
for bit: scores, permutation and output of every group (the path has no
cross-group step, and the score's key splits depend on L only).  This is the
partition a layer takes across GPUs; here every slice runs on one GPU, one
after the other."""

import pytest
import torch

import long_context_tsa_b200 as T
from long_context_tsa_b200 import inputs as I
from long_context_tsa_b200 import shard

from .parity_util import Run

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("name,world", [("gqa_bf16_L8192", 8), ("gqa_bf16_L32768", 2), ("tiny_fp32_L256", 4)])
def test_kv_group_slices_match_the_whole_layer(name, world):
    w = I.WORKLOADS[name]
    q, k, v = I.make_qkv(w, seed=21, device=DEV)
    budgets = w.budgets(seed=1)
    full = Run(w, q, k, v)
    sc, perm, out = (t.clone() for t in full.forward(budgets))
    for rank in range(world):
        g0, g1 = shard.kv_group_range(rank, world, w.Hkv)
        qs, ks, vs = shard.kv_group_slice(q, k, v, g0, g1)
        bs = shard.slice_budgets(budgets, w.B, w.Hkv, g0, g1)
        desc = T.desc_for(qs, ks)
        ws = T.alloc_workspace(desc, w.W, device=DEV)
        s_sc = torch.empty((w.B, g1 - g0, w.L), dtype=torch.float32, device=DEV)
        s_perm = torch.empty((w.B, g1 - g0, w.L), dtype=torch.int32, device=DEV)
        s_out = torch.full_like(qs, float("nan"))
        T.tsa_forward(desc, qs, ks, vs, w.W, bs, s_out, ws, scores=s_sc, perm=s_perm)
        assert T.tsa_check_status(ws) == 0
        assert torch.equal(s_sc.view(torch.int32), sc[:, g0:g1].view(torch.int32)), f"scores, groups {g0}-{g1}"
        assert torch.equal(s_perm, perm[:, g0:g1]), f"perm, groups {g0}-{g1}"
        G = w.G
        ref = out[:, g0 * G:g1 * G]
        bits = torch.int16 if out.dtype == torch.bfloat16 else torch.int32
        assert torch.equal(s_out.view(bits), ref.contiguous().view(bits)), f"output, groups {g0}-{g1}"
