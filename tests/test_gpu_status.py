"""Failure detection on the device without a GPU fault: a bounded wait that
runs out and an out-of-range index both end in a status code the host reads,
and the context stays usable afterwards."""

import numpy as np
import pytest
import torch

import long_context_tsa_b200 as T
from long_context_tsa_b200 import _native as N
from long_context_tsa_b200 import inputs as I
from oracle import tsa_oracle as O

from .parity_util import Run, compare_attend, host

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    T.tsa_debug_set_wait_limit(1000)
    try:
        T.tsa_debug_wait_never_set(ws)
        assert T.tsa_check_status(ws) == N.STATUS["TSA_ERR_TIMEOUT"]
        assert T.tsa_check_status(ws) == 0  # reading clears it
    finally:
        T.tsa_debug_set_wait_limit(0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_out_of_range_index_is_reported_and_context_survives(dtype):
    w = I.custom(Hq=4, Hkv=2, L=300, D=128, dtype=dtype, W=16, sigma=0.5)
    q, k, v = I.make_qkv(w, seed=9, device="cuda")
    budgets = [100, 150]
    perm = O.select(np.random.default_rng(0).random((1, 2, 300)).astype(np.float32), budgets)
    bad = perm.copy()
    bad[0, 0, 50] = 300 + 7  # a kept index past the end
    bad[0, 1, 200] = -3      # a dropped index below zero
    r = Run(w, q, k, v)
    T.tsa_attend(r.desc, q, k, v, torch.from_numpy(bad.astype(np.int32)).cuda(), budgets, r.out, r.ws)
    assert T.tsa_check_status(r.ws) == N.STATUS["TSA_ERR_DEVICE_BOUNDS"]
    out = r.attend(torch.from_numpy(perm.astype(np.int32)).cuda(), budgets)
    compare_attend(out, host(q), host(k), host(v), perm, budgets, dtype)

