"""Host side of the drift metric: the window stability rule through the C ABI
(pure host code) against the oracle, and argument checks that return before
any device work."""

import ctypes

import numpy as np
import pytest

import long_context_tsa_b200 as T
from long_context_tsa_b200 import _native as N
from oracle import tsa_oracle as O

INVALID = 1
WORKSPACE = 3


def test_layer_stable_matches_oracle_on_random_histories():
    rng = np.random.default_rng(0)
    for _ in range(300):
        n = int(rng.integers(0, 8))
        hist = list(rng.uniform(0.0, 0.2, size=n))
        window = int(rng.integers(1, 5))
        thr = float(rng.choice([0.05, 0.1, 0.15]))
        assert T.tsa_layer_stable(hist, window, thr) == O.layer_stable(hist, window, thr), (hist, window, thr)


def test_layer_stable_edges():
    assert T.tsa_layer_stable([0.25, 0.25, 0.25], 3, 0.25) is False  # strictly below
    assert T.tsa_layer_stable([], 1, 1.0) is False
    out = ctypes.c_int32(7)
    assert N.lib().tsa_layer_stable(None, 0, 3, 0.1, ctypes.byref(out)) == 0 and out.value == 0
    assert N.lib().tsa_layer_stable(None, 2, 3, 0.1, ctypes.byref(out)) == INVALID
    arr = (ctypes.c_double * 1)(0.0)
    assert N.lib().tsa_layer_stable(arr, 1, 0, 0.1, ctypes.byref(out)) == INVALID
    assert N.lib().tsa_layer_stable(arr, -1, 1, 0.1, ctypes.byref(out)) == INVALID
    assert N.lib().tsa_layer_stable(arr, 1, 1, 0.1, None) == INVALID


@pytest.mark.parametrize("rows,hidden,dtype,code", [
    (0, 64, 1, INVALID),       # no rows: the mean is undefined
    (4, 0, 1, INVALID),
    (4, 12, 1, INVALID),       # 24-byte bf16 rows are not a multiple of 16 bytes
    (4, 6, 0, INVALID),        # 24-byte f32 rows
    (4, 64, 2, INVALID),       # unknown dtype
])
def test_drift_rejects_bad_shapes(rows, hidden, dtype, code):
    p = 1 << 20  # aligned, never dereferenced: the checks return first
    assert N.lib().tsa_drift(rows, hidden, dtype, p, p, None, p, p, 1 << 16, None) == code


def test_drift_rejects_bad_pointers_and_workspace():
    p = 1 << 20
    lib = N.lib()
    assert lib.tsa_drift(4, 64, 1, p + 8, p, None, p, p, 1 << 16, None) == INVALID  # misaligned input
    assert lib.tsa_drift(4, 64, 1, p, p, None, None, p, 1 << 16, None) == INVALID  # no drift output
    assert lib.tsa_drift(4, 64, 1, p, p, None, p + 4, p, 1 << 16, None) == INVALID  # drift not 8-byte aligned
    assert lib.tsa_drift(4, 64, 1, p, p, p + 2, p, p, 1 << 16, None) == INVALID  # row_cos not 4-byte aligned
    ws_need = T.tsa_drift_workspace_size()
    assert ws_need >= 256
    assert lib.tsa_drift(4, 64, 1, p, p, None, p, p, ws_need - 1, None) == WORKSPACE
