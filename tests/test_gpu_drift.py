"""Drift kernel vs the fp64 oracle through the C ABI.

Tolerance, derived from the arithmetic: each lane sums about hidden/32
products serially in fp32 and the warp adds 32 partials in a 5-level tree, so
|a|^2, |b|^2 and <a,b> (the last relative to sum |a_i b_i| <= |a| |b|) carry a
relative error of at most about (hidden/32 + 5) * 2^-24; the cosine inherits
twice that plus a few roundings of the square roots and the division.  The
test allows 4 * (ceil(hidden/32) + 8) * 2^-24 per row and for the mean.
"""

import math

import numpy as np
import pytest
import torch

import long_context_tsa_b200 as T
from long_context_tsa_b200 import inputs as I
from oracle import tsa_oracle as O

from .parity_util import host

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _tol(hidden):
    return 4 * (math.ceil(hidden / 32) + 8) * 2.0 ** -24


def _run(a, b, with_rows=True):
    rows = a.numel() // a.shape[-1]
    ws = T.alloc_drift_workspace(DEV)
    d = torch.full((1,), float("nan"), dtype=torch.float64, device=DEV)
    rc = torch.full((rows,), float("nan"), dtype=torch.float32, device=DEV) if with_rows else None
    T.tsa_drift(a, b, d, ws, row_cos=rc)
    torch.cuda.synchronize()
    return float(d.item()), (host(rc) if with_rows else None)


@pytest.mark.parametrize("B,L,hidden,dtype", [
    (1, 1, 8, "bf16"),         # one row of one 16-byte vector
    (1, 333, 4096, "bf16"),    # unrolled loop only
    (2, 517, 4104, "bf16"),    # unrolled loop plus a ragged tail of vectors
    (3, 100, 100, "f32"),      # 25 vectors a row: tail loop only
    (1, 2049, 1028, "f32"),
    (1, 5000, 64, "bf16"),     # 8 vectors a row: most lanes idle
])
def test_drift_matches_oracle(B, L, hidden, dtype):
    a, b = I.make_hidden(B, L, hidden, dtype, delta=0.4, seed=L, device=DEV)
    drift, rc = _run(a, b)
    an, bn = host(a), host(b)
    ora_rows = O.row_cosine(an, bn).reshape(-1)
    tol = _tol(hidden)
    assert np.all(np.isfinite(rc))
    assert np.abs(rc - ora_rows).max() <= tol
    assert abs(drift - O.drift(an, bn)) <= tol
    d2, _ = _run(a, b, with_rows=False)  # the drift does not depend on asking for the rows
    assert d2 == drift


def test_drift_special_rows():
    # Identical, negated, orthogonal, zero and below-eps rows (normalize's clamp).
    hidden = 256
    a = torch.zeros((1, 6, hidden), dtype=torch.float32)
    b = torch.zeros_like(a)
    x = torch.randn(hidden, generator=torch.Generator().manual_seed(1))
    a[0, 0] = x; b[0, 0] = x             # cosine 1
    a[0, 1] = x; b[0, 1] = -2 * x        # cosine -1
    a[0, 2, 0] = 1.0; b[0, 2, 1] = 3.0   # orthogonal: 0
    b[0, 3] = x                          # a row of zeros: 0
    a[0, 4, 5] = 1e-13; b[0, 4, 5] = 7.0  # norm below eps: 0.1
    a[0, 5] = x; b[0, 5] = 1e6 * x       # scale invariance: 1
    drift, rc = _run(a.to(DEV), b.to(DEV))
    ora = O.row_cosine(a.numpy(), b.numpy()).reshape(-1)
    # 1e-13 is stored as the nearest float32, so the 0.1 holds to float32 precision.
    np.testing.assert_allclose(ora, [1, -1, 0, 0, 0.1, 1], rtol=1e-7, atol=1e-15)
    np.testing.assert_allclose(rc, ora, rtol=0, atol=_tol(hidden))
    assert abs(drift - O.drift(a.numpy(), b.numpy())) <= _tol(hidden)


def test_drift_full_size_workload():
    # The benchmarked workload: 131072 rows of 4096 bf16 (2 GiB read); the oracle
    # runs over row chunks (its per-row arithmetic does not depend on the chunking).
    w = I.DRIFT_WORKLOAD
    a, b = I.make_hidden(w["B"], w["L"], w["hidden"], w["dtype"], w["delta"], seed=0, device=DEV)
    drift, rc = _run(a, b)
    rows = w["B"] * w["L"]
    ora = np.empty(rows)
    step = 8192
    for r0 in range(0, rows, step):
        ora[r0:r0 + step] = O.row_cosine(host(a.view(rows, -1)[r0:r0 + step]), host(b.view(rows, -1)[r0:r0 + step]))
    tol = _tol(w["hidden"])
    assert np.abs(rc - ora).max() <= tol
    assert abs(drift - (1.0 - ora.mean())) <= tol
    assert 0.0 < drift < 0.1
