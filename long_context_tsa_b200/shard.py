"""Host-side partition of the path across GPUs (there is no exchange step).

Every step of the path -- score, select, attention on the compressed tensors,
scatter -- works per (batch entry, KV group): query head h reads only KV head
h // G, and the kept subset it attends over is its group's own ("Token Sparse
Attention: Efficient Long-Context Inference with Interleaved Token Selection",
Figure 3: a token subset per head, no cross-head step).  A layer therefore
splits into independent pieces with no collective: by batch entry, or by
contiguous ranges of KV groups, each taken with the G query heads that read
it.  The library's results for a KV group do not depend on the other groups
in the same call (the score's key splits depend on L only), so a layer split
this way reproduces the single-call result bit for bit.
"""

from __future__ import annotations


def kv_group_range(rank: int, world: int, Hkv: int) -> tuple[int, int]:
    """Contiguous, balanced range [g0, g1) of KV groups owned by `rank` of `world`."""
    if not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    return rank * Hkv // world, (rank + 1) * Hkv // world


def kv_group_slice(q, k, v, g0: int, g1: int):
    """The head-major sub-tensors of KV groups [g0, g1): q [B, (g1-g0)*G, L, D],
    k and v [B, g1-g0, L, D], contiguous (plain views when B == 1)."""
    G = q.shape[1] // k.shape[1]
    return (q[:, g0 * G:g1 * G].contiguous(), k[:, g0:g1].contiguous(), v[:, g0:g1].contiguous())


def slice_budgets(budgets, B: int, Hkv: int, g0: int, g1: int) -> list[int]:
    """The per-(batch, KV group) budgets of groups [g0, g1), in the sliced call's order."""
    return [int(budgets[b * Hkv + g]) for b in range(B) for g in range(g0, g1)]
