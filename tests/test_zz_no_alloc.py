"""tsa_score_noalloc: scoring for callers that cannot allocate device memory.

Such callers (an engine plugin whose host owns all device memory, a loop that
must not call cudaMalloc) cannot provide tsa_score's workspace; the variant
keeps its scratch in a fixed array inside the library.  These checks call it
through the C ABI and compare it with the oracle and with tsa_score on the
same inputs, twice in a row with different shapes (the shared array keeps the
previous call's contents, which must not leak into the next result); fill the
whole array at its documented limit; read its device status word; and check
that a shape needing more than the fixed scratch is refused before any
pointer is looked at.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from long_context_tsa_b200 import _native as N
from long_context_tsa_b200 import inputs as I
from oracle import tsa_oracle as O

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-4, 1e-35  # the score tolerance of the parity tests


def _noalloc_call(desc, q, k, window, out):
    stream = torch.cuda.current_stream().cuda_stream
    return N.lib().tsa_score_noalloc(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), int(window), out.data_ptr(),
                                     stream)


def _noalloc_status():
    # NULL workspace: the status word of tsa_score_noalloc on the current device.
    return N.lib().tsa_check_status(None, 0, torch.cuda.current_stream().cuda_stream)


def _close(a, b):
    a = np.asarray(a, dtype=np.float64)
    return bool(np.all(np.isfinite(a)) and np.all(np.abs(a - b) <= RTOL * np.abs(b) + ATOL))


def _check(w, seed, with_oracle=True):
    q, k, _ = I.make_qkv(w, seed=seed, device="cuda")
    desc = N.desc_for(q, k)
    got = torch.full((w.B, w.Hkv, w.L), float("nan"), dtype=torch.float32, device="cuda")
    assert _noalloc_call(desc, q, k, w.W, got) == 0
    assert _noalloc_status() == 0
    g = got.cpu().numpy()
    if with_oracle:
        ora = O.score(q.float().cpu().numpy(), k.float().cpu().numpy(), w.W)
        assert _close(g, ora)
    ws = N.alloc_workspace(desc, w.W)
    ref = torch.empty_like(got)
    N.tsa_score(desc, q, k, w.W, ref, ws)
    assert N.tsa_check_status(ws) == 0
    assert _close(g, ref.cpu().numpy().astype(np.float64))


def test_noalloc_score_matches_oracle_and_tsa_score_on_two_calls_in_a_row():
    first = I.custom("noalloc_a", Hq=8, Hkv=2, L=3000, D=128, dtype="bf16", W=64, sigma=0.5, planted=16)
    second = I.custom("noalloc_b", B=2, Hq=4, Hkv=4, L=1111, D=64, dtype="f32", W=16, sigma=1.0)
    _check(first, seed=1)
    _check(second, seed=2)


def test_noalloc_score_fills_the_whole_array_at_its_limit():
    # 32/8 heads, window 64, B = 64 at the shortest length with one key split (L = 128
    # in bf16, L = 64 in f32): the partials take exactly the 1 MiB array
    # (512 KV heads x 1 split x 256 window rows x 8 bytes).
    for dtype, D, L in (("bf16", 128, 128), ("f32", 64, 64)):
        w = I.custom("noalloc_limit", B=64, Hq=32, Hkv=8, L=L, D=D, dtype=dtype, W=64, sigma=0.5)
        _check(w, seed=3, with_oracle=False)


def test_noalloc_score_bench_layer():
    # The 128K bf16 layer (8 KV heads x 18 splits x 256 rows x 8 bytes = 295 KB) fits.
    w = I.WORKLOADS["gqa_bf16_L131072"]
    _check(w, seed=4, with_oracle=False)


def test_noalloc_score_refuses_shapes_beyond_its_fixed_scratch():
    # B = 65 needs more than the 1 MiB array: refused with TSA_ERR_WORKSPACE before
    # the (null) pointers are looked at, so nothing can be launched.
    for dtype, L in ((N.TSA_BF16, 128), (N.TSA_F32, 64)):
        big = N.make_desc(B=65, Hq=32, Hkv=8, L=L, D=128, dtype=dtype)
        assert N.lib().tsa_score_noalloc(ctypes.byref(big), None, None, 64, None, None) == \
            N.STATUS["TSA_ERR_WORKSPACE"]
        fits = N.make_desc(B=64, Hq=32, Hkv=8, L=L, D=128, dtype=dtype)
        assert N.lib().tsa_score_noalloc(ctypes.byref(fits), None, None, 64, None, None) == \
            N.STATUS["TSA_ERR_INVALID_ARG"]
