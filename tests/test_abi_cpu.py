"""Host-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments with the documented status codes
before touching the device.  No compute call is made here (no GPU needed)."""

import ctypes
import os
import re

import pytest

from long_context_tsa_b200 import _native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tsa.h")

FAKE = 0x100000  # a 16-byte aligned address that is never dereferenced: every call below fails validation first


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(N.LIB_PATH):
        from long_context_tsa_b200 import build

        build.build()
    return N.lib()


def declared_symbols():
    text = open(HEADER).read()
    return set(re.findall(r"TSA_API\s+[\w\s\*]+?\b(tsa_\w+)\s*\(", text))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert names == set(N.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n


def desc(**kw):
    base = dict(B=1, Hq=32, Hkv=8, L=8192, D=128, dtype=N.TSA_BF16, scale=0.0)
    base.update(kw)
    return N.TsaDesc(*[base[f] for f, _ in N.TsaDesc._fields_])


def test_workspace_size(lib):
    d = desc()
    n = lib.tsa_workspace_size(ctypes.byref(d), 64)
    assert n >= 256 + 2 * 8 * 8192 * 4
    assert lib.tsa_workspace_size(ctypes.byref(desc(D=96)), 64) == 0
    assert lib.tsa_workspace_size(ctypes.byref(d), 0) == 0
    assert lib.tsa_workspace_size(None, 64) == 0


def score(lib, d, window=64, q=FAKE, k=FAKE, scores=FAKE, ws=FAKE, ws_bytes=1 << 40):
    return lib.tsa_score(ctypes.byref(d) if d is not None else None, q, k, window, scores, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), "TSA_ERR_UNSUPPORTED"),
    (dict(Hq=30), "TSA_ERR_INVALID_ARG"),
    (dict(Hq=8 * 32), "TSA_ERR_UNSUPPORTED"),  # G = 32
    (dict(dtype=7), "TSA_ERR_INVALID_ARG"),
    (dict(L=0), "TSA_ERR_INVALID_ARG"),
    (dict(B=200), "TSA_ERR_UNSUPPORTED"),  # B * Hkv > 1024
    (dict(B=1, L=1 << 30), "TSA_ERR_UNSUPPORTED"),  # B * Hq * L >= 2^31
    (dict(scale=float("nan")), "TSA_ERR_INVALID_ARG"),
])
def test_score_rejects_bad_shapes(lib, kw, code):
    assert score(lib, desc(**kw)) == N.STATUS[code]


def test_score_rejects_bad_window_pointers_and_workspace(lib):
    d = desc()
    assert score(lib, None) == N.STATUS["TSA_ERR_INVALID_ARG"]
    assert score(lib, d, window=0) == N.STATUS["TSA_ERR_INVALID_ARG"]
    assert score(lib, d, window=8193) == N.STATUS["TSA_ERR_INVALID_ARG"]
    assert score(lib, d, window=65) == N.STATUS["TSA_ERR_UNSUPPORTED"]  # G * W = 260 > 256
    assert score(lib, d, q=FAKE + 8) == N.STATUS["TSA_ERR_INVALID_ARG"]
    assert score(lib, d, k=None) == N.STATUS["TSA_ERR_INVALID_ARG"]
    need = lib.tsa_workspace_size(ctypes.byref(d), 64)
    assert score(lib, d, ws_bytes=need - 1) == N.STATUS["TSA_ERR_WORKSPACE"]


def test_select_and_attend_reject_bad_budgets(lib):
    d = desc()
    for bad in ([4096] * 7 + [0], [4096] * 7 + [-5]):
        b = N._budgets(bad)
        assert lib.tsa_select(ctypes.byref(d), FAKE, b, FAKE, FAKE, 1 << 20, None) == N.STATUS["TSA_ERR_INVALID_ARG"]
        assert lib.tsa_attend(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, b, FAKE, FAKE, 1 << 20, None) == \
            N.STATUS["TSA_ERR_INVALID_ARG"]
    b = N._budgets([4096] * 8)
    assert lib.tsa_select(ctypes.byref(d), FAKE, None, FAKE, FAKE, 1 << 20, None) == N.STATUS["TSA_ERR_INVALID_ARG"]
    assert lib.tsa_select(ctypes.byref(d), FAKE, b, FAKE, FAKE, 64, None) == N.STATUS["TSA_ERR_WORKSPACE"]
    assert lib.tsa_attend(ctypes.byref(d), FAKE, FAKE, FAKE, None, b, FAKE, FAKE, 1 << 20, None) == \
        N.STATUS["TSA_ERR_INVALID_ARG"]


def test_forward_rejects_before_launch(lib):
    d = desc()
    b = N._budgets([4096] * 8)
    assert lib.tsa_forward(ctypes.byref(d), FAKE, FAKE, FAKE, 64, b, FAKE + 4, None, FAKE, FAKE, 1 << 40, None) == \
        N.STATUS["TSA_ERR_INVALID_ARG"]
    assert lib.tsa_forward(ctypes.byref(d), FAKE, FAKE, FAKE, 64, b, None, None, FAKE, FAKE, 256, None) == \
        N.STATUS["TSA_ERR_WORKSPACE"]
    assert lib.tsa_forward_host(ctypes.byref(d), None, FAKE, FAKE, 64, b, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                1 << 40, None) == N.STATUS["TSA_ERR_INVALID_ARG"]


def test_host_h2d_bytes_counts(lib):
    d = desc()
    b = N._budgets([4096] * 8)
    # Plain (pageable) host memory is not mapped into any device: the full-copy count.
    buf = (ctypes.c_uint8 * 64)()
    a = ctypes.addressof(buf)
    n = lib.tsa_forward_host_h2d_bytes(ctypes.byref(d), 64, b, a, a)
    assert n == (d.B * d.Hq + 2 * d.B * d.Hkv) * d.L * d.D * 2
    assert lib.tsa_forward_host_h2d_bytes(ctypes.byref(desc(D=96)), 64, b, a, a) == 0
    assert lib.tsa_forward_host_h2d_bytes(ctypes.byref(d), 0, b, a, a) == 0
    assert lib.tsa_forward_host_h2d_bytes(ctypes.byref(d), 64, N._budgets([0] * 8), a, a) == 0


def test_status_strings(lib):
    for code in range(7):
        assert N.tsa_status_string(code)
    assert N.tsa_status_string(99) == "unknown status"


def test_next_row_calls_reject_before_launch(lib):
    d = desc()
    b = N._budgets([4096] * 8)
    bad_b = N._budgets([4096] * 7 + [0])
    inv, wsz = N.STATUS["TSA_ERR_INVALID_ARG"], N.STATUS["TSA_ERR_WORKSPACE"]
    # Scatter-add attention: same rules as tsa_attend.
    assert lib.tsa_attend_accumulate(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, bad_b, FAKE, FAKE, 1 << 20, None) == inv
    assert lib.tsa_attend_accumulate(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, b, FAKE + 2, FAKE, 1 << 20, None) == inv
    assert lib.tsa_attend_accumulate(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, b, FAKE, FAKE, 16, None) == wsz
    # Block-sparse attention: a mask is required.
    assert lib.tsa_attend_block_sparse(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, b, None, FAKE, FAKE, 1 << 20,
                                       None) == inv
    assert lib.tsa_attend_block_sparse(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, bad_b, FAKE, FAKE, FAKE, 1 << 20,
                                       None) == inv
    # Coverage selection: tau in [0, 1], a budget output, the usual pointer rules.
    for tau in (-0.5, 1.01, float("nan"), float("inf")):
        assert lib.tsa_select_coverage(ctypes.byref(d), FAKE, tau, FAKE, FAKE, FAKE, 1 << 20, None) == inv
    assert lib.tsa_select_coverage(ctypes.byref(d), FAKE, 0.1, FAKE, None, FAKE, 1 << 20, None) == inv
    assert lib.tsa_select_coverage(ctypes.byref(d), FAKE, 0.1, FAKE, FAKE + 2, FAKE, 1 << 20, None) == inv
    assert lib.tsa_select_coverage(ctypes.byref(d), FAKE, 0.1, FAKE, FAKE, FAKE, 16, None) == wsz
    out = (ctypes.c_int32 * 8)()
    assert lib.tsa_forward_coverage(ctypes.byref(d), FAKE, FAKE, FAKE, 64, 2.0, out, None, None, FAKE, FAKE,
                                    1 << 40, None) == inv
    assert lib.tsa_forward_coverage(ctypes.byref(d), FAKE, FAKE, FAKE, 64, 0.1, None, None, None, FAKE, FAKE,
                                    1 << 40, None) == inv
    assert lib.tsa_forward_coverage(ctypes.byref(d), FAKE, FAKE, FAKE, 64, 0.1, out, None, None, FAKE, FAKE,
                                    256, None) == wsz


def test_zero_dropped_and_noalloc_reject_before_launch(lib):
    d = desc()
    b = N._budgets([4096] * 8)
    bad_b = N._budgets([4096] * 7 + [-1])
    inv, wsz = N.STATUS["TSA_ERR_INVALID_ARG"], N.STATUS["TSA_ERR_WORKSPACE"]
    assert lib.tsa_zero_dropped(ctypes.byref(d), FAKE, bad_b, FAKE, FAKE, 1 << 20, None) == inv
    assert lib.tsa_zero_dropped(ctypes.byref(d), FAKE + 4, b, FAKE, FAKE, 1 << 20, None) == inv
    assert lib.tsa_zero_dropped(ctypes.byref(d), FAKE, b, FAKE, FAKE, 16, None) == wsz
    assert lib.tsa_zero_dropped(ctypes.byref(desc(D=96)), FAKE, b, FAKE, FAKE, 1 << 20, None) == \
        N.STATUS["TSA_ERR_UNSUPPORTED"]
    # The no-allocation scorer checks the shape, then its fixed scratch, then the pointers:
    # B = 65 with 32/8 heads and window 64 needs more than its 1 MiB, whatever the pointers.
    # At the shortest lengths (one split: L <= 128 in bf16, L <= 64 in f32) B = 64 fills it exactly.
    for dt, L_fit in ((N.TSA_BF16, 128), (N.TSA_F32, 64)):
        big = N.make_desc(B=65, Hq=32, Hkv=8, L=L_fit, D=128, dtype=dt)
        assert lib.tsa_score_noalloc(ctypes.byref(big), None, None, 64, None, None) == wsz
        fits = N.make_desc(B=64, Hq=32, Hkv=8, L=L_fit, D=128, dtype=dt)
        assert lib.tsa_score_noalloc(ctypes.byref(fits), None, None, 64, None, None) == inv
        two_splits = N.make_desc(B=64, Hq=32, Hkv=8, L=2 * L_fit, D=128, dtype=dt)
        assert lib.tsa_score_noalloc(ctypes.byref(two_splits), None, None, 64, None, None) == wsz
    # The bf16 128K layer (8 KV heads x 18 splits x 256 rows x 8 bytes = 295 KB) fits.
    layer = N.make_desc(B=1, Hq=32, Hkv=8, L=131072, D=128, dtype=N.TSA_BF16)
    assert lib.tsa_score_noalloc(ctypes.byref(layer), None, None, 64, None, None) == inv
    assert lib.tsa_score_noalloc(ctypes.byref(desc(D=96)), None, None, 64, None, None) == \
        N.STATUS["TSA_ERR_UNSUPPORTED"]
    assert lib.tsa_score_noalloc(ctypes.byref(desc()), None, None, 65, None, None) == \
        N.STATUS["TSA_ERR_UNSUPPORTED"]  # G * W = 260 > 256, the same code tsa_score returns


def test_binding_checks_block_mask_shape():
    import torch

    import long_context_tsa_b200 as T

    d = desc(L=1000)
    wrong = torch.zeros((1, 8, 7, 7), dtype=torch.uint8)  # nb = 8 for L = 1000
    with pytest.raises(ValueError):
        T.tsa_attend_block_sparse(d, None, None, None, None, [1] * 8, wrong, None, torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(ValueError):
        T.tsa_attend_block_sparse(d, None, None, None, None, [1] * 8, torch.zeros((1, 8, 8, 8)), None,
                                  torch.zeros(16, dtype=torch.uint8))
