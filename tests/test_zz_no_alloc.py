"""tsa_score_noalloc: scoring for callers that cannot allocate device memory.

Such callers (an engine plugin whose host owns all device memory, a loop that
must not call cudaMalloc) cannot provide tsa_score's workspace; the variant
keeps its scratch in a fixed array inside the library.  These checks call it
through the C ABI and compare it with tsa_score on the same inputs, twice in a
row with different shapes (the shared array keeps the previous call's
contents, which must not leak into the next result), and check that a shape
needing more than the fixed scratch is refused.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from long_context_tsa_b200 import _native as N
from long_context_tsa_b200 import inputs as I

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-4, 1e-35  # the score tolerance of the parity tests


def _noalloc_call(desc, q, k, window, out):
    stream = torch.cuda.current_stream().cuda_stream
    return N.lib().tsa_score_noalloc(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), int(window), out.data_ptr(),
                                     stream)


def _check_against_workspace_path(w, seed):
    q, k, _ = I.make_qkv(w, seed=seed, device="cuda")
    desc = N.desc_for(q, k)
    ws = N.alloc_workspace(desc, w.W)
    ref = torch.empty((w.B, w.Hkv, w.L), dtype=torch.float32, device="cuda")
    N.tsa_score(desc, q, k, w.W, ref, ws)
    assert N.tsa_check_status(ws) == 0
    got = torch.full_like(ref, float("nan"))
    assert _noalloc_call(desc, q, k, w.W, got) == 0
    torch.cuda.synchronize()
    a, b = got.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(a))
    assert np.all(np.abs(a - b) <= RTOL * np.abs(b) + ATOL)


def test_noalloc_score_matches_tsa_score_on_two_calls_in_a_row():
    first = I.custom("noalloc_a", Hq=8, Hkv=2, L=3000, D=128, dtype="bf16", W=64, sigma=0.5, planted=16)
    second = I.custom("noalloc_b", B=2, Hq=4, Hkv=4, L=1111, D=64, dtype="f32", W=16, sigma=1.0)
    _check_against_workspace_path(first, seed=1)
    _check_against_workspace_path(second, seed=2)


def test_noalloc_score_refuses_shapes_beyond_its_fixed_scratch():
    # Partials take B*Hkv * splits * 256 window rows * 8 bytes; with 32/8 heads and
    # window 64 that is 1 MiB at B=64 (fits) and 2 MiB at B=128 (refused).
    ok = N.make_desc(B=64, Hq=32, Hkv=8, L=8192, D=128, dtype=N.TSA_BF16)
    big = N.make_desc(B=128, Hq=32, Hkv=8, L=8192, D=128, dtype=N.TSA_BF16)
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: the call is refused before any launch
    assert N.lib().tsa_score_noalloc(ctypes.byref(big), fake, fake, 64, fake, None) == N.STATUS["TSA_ERR_WORKSPACE"]
    assert N.lib().tsa_workspace_size(ctypes.byref(ok), 64) > 0
