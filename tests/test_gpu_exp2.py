"""The FMA-pipe exponential the scoring kernel uses for one pair in three of its
column-sum terms, against the mathematics: relative error within the bound of
its polynomial (3.0e-6 in float32), exact powers of two at integers, and the
documented floor of 2^-126 below the clamp."""

import numpy as np
import pytest
import torch

import long_context_tsa_b200 as T

pytestmark = pytest.mark.gpu


def test_fma_pipe_exp2_within_its_error_bound():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        np.linspace(-126.0, 100.0, 200001),
        rng.uniform(-40.0, 0.0, 200000),
        -np.arange(0, 127, dtype=np.float64),  # integers: exact powers of two
        np.arange(0, 100, dtype=np.float64),
        [-126.5, -200.0, -1e30],                # below the clamp
    ]).astype(np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(0.0))
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    T.tsa_debug_exp2(xd, yd)
    torch.cuda.synchronize()
    y = yd.cpu().numpy().astype(np.float64)
    xs = x.astype(np.float64)
    ok = xs >= -126.0
    ref = np.exp2(xs[ok])
    rel = np.abs(y[ok] - ref) / ref
    assert rel.max() <= 3.1e-6, rel.max()
    ints = ok & (xs == np.round(xs))
    np.testing.assert_array_equal(y[ints], np.exp2(xs[ints]))
    assert np.all(y[~ok] == np.float64(np.float32(2.0 ** -126)))
