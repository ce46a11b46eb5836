"""ctypes binding of libtsa.so: the C entry points under the same names.

Argument marshalling only -- every step runs in the CUDA kernels of the
library.  Tensors are PyTorch tensors (device memory for the compute calls,
host memory for ``tsa_forward_host``); budgets are Python sequences of ints.
There is no fallback: a missing library raises ``RuntimeError``.
"""

from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtsa.so")

TSA_F32, TSA_BF16 = 0, 1
STATUS_NAMES = {0: "TSA_OK", 1: "TSA_ERR_INVALID_ARG", 2: "TSA_ERR_UNSUPPORTED", 3: "TSA_ERR_WORKSPACE",
                4: "TSA_ERR_CUDA", 5: "TSA_ERR_TIMEOUT", 6: "TSA_ERR_DEVICE_BOUNDS"}
STATUS = {v: k for k, v in STATUS_NAMES.items()}

EXPORTED = ("tsa_workspace_size", "tsa_workspace_init", "tsa_score", "tsa_select", "tsa_attend", "tsa_forward",
            "tsa_forward_host", "tsa_check_status", "tsa_status_string", "tsa_debug_set_wait_limit",
            "tsa_debug_wait_never_set", "tsa_debug_launch_count", "tsa_debug_cta_pair_launch_count", "tsa_score_noalloc",
            "tsa_attend_accumulate", "tsa_drift_workspace_size", "tsa_drift", "tsa_layer_stable",
            "tsa_select_coverage", "tsa_forward_coverage", "tsa_attend_block_sparse", "tsa_debug_exp2", "tsa_zero_dropped",
            "tsa_out_proj_workspace_size", "tsa_out_proj", "tsa_forward_host_h2d_bytes")


class TsaDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("L", ctypes.c_int32),
                ("D", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float)]


class TsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")


_lib = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_SZ = ctypes.c_size_t
_SIGS = {
    "tsa_workspace_size": (_SZ, [ctypes.POINTER(TsaDesc), _I32]),
    "tsa_workspace_init": (ctypes.c_int, [_P, _SZ, _P]),
    "tsa_score": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _I32, _P, _P, _SZ, _P]),
    "tsa_select": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _P, _P, _SZ, _P]),
    "tsa_attend": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "tsa_forward": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _P, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "tsa_forward_host": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _P, _I32, _P, _P, _P, _P, _P, _P, _P,
                                        _SZ, _P]),
    "tsa_forward_host_h2d_bytes": (_SZ, [ctypes.POINTER(TsaDesc), _I32, _P, _P, _P]),
    "tsa_check_status": (ctypes.c_int, [_P, _SZ, _P]),
    "tsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "tsa_debug_set_wait_limit": (None, [ctypes.c_uint64]),
    "tsa_debug_wait_never_set": (ctypes.c_int, [_P, _SZ, _P]),
    "tsa_debug_launch_count": (ctypes.c_uint64, []),
    "tsa_debug_cta_pair_launch_count": (ctypes.c_uint64, []),
    "tsa_score_noalloc": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _I32, _P, _P]),
    "tsa_attend_accumulate": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "tsa_drift_workspace_size": (_SZ, []),
    "tsa_out_proj_workspace_size": (_SZ, [ctypes.POINTER(TsaDesc)]),
    "tsa_out_proj": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _P, _P, _I32, _P, _P, _SZ, _P]),
    "tsa_zero_dropped": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _P, _P, _SZ, _P]),
    "tsa_debug_exp2": (ctypes.c_int, [_P, _P, _I32, _P]),
    "tsa_attend_block_sparse": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "tsa_select_coverage": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, ctypes.c_double, _P, _P, _P, _SZ, _P]),
    "tsa_forward_coverage": (ctypes.c_int, [ctypes.POINTER(TsaDesc), _P, _P, _P, _I32, ctypes.c_double, _P, _P, _P,
                                            _P, _P, _SZ, _P]),
    "tsa_drift": (ctypes.c_int, [ctypes.c_int64, _I32, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "tsa_layer_stable": (ctypes.c_int, [ctypes.POINTER(ctypes.c_double), _I32, _I32, ctypes.c_double,
                                        ctypes.POINTER(ctypes.c_int32)]),
}


def lib() -> ctypes.CDLL:
    """Load libtsa.so (built in-tree by ``long_context_tsa_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA extension missing: {LIB_PATH} (run python -m long_context_tsa_b200.build)")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return getattr(stream, "cuda_stream", stream)


def _budgets(b):
    arr = (ctypes.c_int32 * len(b))(*[int(x) for x in b])
    return arr


def _check(code: int, where: str):
    if code != 0:
        raise TsaError(code, where)


def make_desc(B: int, Hq: int, Hkv: int, L: int, D: int, dtype, scale: float = 0.0) -> TsaDesc:
    if isinstance(dtype, torch.dtype):
        dtype = TSA_F32 if dtype == torch.float32 else TSA_BF16 if dtype == torch.bfloat16 else -1
    return TsaDesc(B, Hq, Hkv, L, D, int(dtype), float(scale))


def desc_for(q: torch.Tensor, k: torch.Tensor, scale: float = 0.0) -> TsaDesc:
    B, Hq, L, D = q.shape
    return make_desc(B, Hq, k.shape[1], L, D, q.dtype, scale)


def tsa_workspace_size(desc: TsaDesc, window: int) -> int:
    return int(lib().tsa_workspace_size(ctypes.byref(desc), int(window)))


def tsa_workspace_init(ws: torch.Tensor, stream=None):
    _check(lib().tsa_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "tsa_workspace_init")


def alloc_workspace(desc: TsaDesc, window: int, device="cuda") -> torch.Tensor:
    """Caller-side workspace allocation (PyTorch owns the memory), zero-filled."""
    n = tsa_workspace_size(desc, window)
    if n == 0:
        raise TsaError(STATUS["TSA_ERR_INVALID_ARG"], "tsa_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def tsa_score(desc, q, k, window, scores, ws, stream=None):
    _check(lib().tsa_score(ctypes.byref(desc), _ptr(q), _ptr(k), int(window), _ptr(scores), _ptr(ws),
                           ws.numel(), _stream(stream)), "tsa_score")


def tsa_select(desc, scores, budgets, perm, ws, stream=None):
    _check(lib().tsa_select(ctypes.byref(desc), _ptr(scores), _budgets(budgets), _ptr(perm), _ptr(ws), ws.numel(),
                            _stream(stream)), "tsa_select")


def tsa_attend(desc, q, k, v, perm, budgets, out, ws, stream=None):
    _check(lib().tsa_attend(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(perm), _budgets(budgets),
                            _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "tsa_attend")


def tsa_out_proj_workspace_size(desc) -> int:
    return int(lib().tsa_out_proj_workspace_size(ctypes.byref(desc)))


def alloc_out_proj_workspace(desc, device="cuda") -> torch.Tensor:
    n = tsa_out_proj_workspace_size(desc)
    if n == 0:
        raise TsaError(STATUS["TSA_ERR_UNSUPPORTED"], "tsa_out_proj_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def tsa_out_proj(desc, attn_out, perm, budgets, w_o, x, ws, stream=None):
    """x[b, p, :] += the projection (w_o, [hidden, Hq*D]) of the heads' attention rows kept at p."""
    hidden = int(w_o.shape[0])
    if x.shape[-1] != hidden or w_o.shape[1] != desc.Hq * desc.D:
        raise ValueError("x must be [B, L, hidden] and w_o [hidden, Hq*D]")
    _check(lib().tsa_out_proj(ctypes.byref(desc), _ptr(attn_out), _ptr(perm), _budgets(budgets), _ptr(w_o), hidden,
                              _ptr(x), _ptr(ws), ws.numel(), _stream(stream)), "tsa_out_proj")


def tsa_zero_dropped(desc, perm, budgets, out, ws, stream=None):
    """+0 at every dropped row of every query head; kept rows untouched."""
    _check(lib().tsa_zero_dropped(ctypes.byref(desc), _ptr(perm), _budgets(budgets), _ptr(out), _ptr(ws), ws.numel(),
                                  _stream(stream)), "tsa_zero_dropped")


def tsa_attend_accumulate(desc, q, k, v, perm, budgets, out, ws, stream=None):
    """out[kept rows] += attention (scatter-add); dropped rows are left as they are."""
    _check(lib().tsa_attend_accumulate(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(perm), _budgets(budgets),
                                       _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "tsa_attend_accumulate")


def tsa_forward(desc, q, k, v, window, budgets, out, ws, scores=None, perm=None, stream=None):
    _check(lib().tsa_forward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), int(window), _budgets(budgets),
                             _ptr(scores), _ptr(perm), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "tsa_forward")


def tsa_forward_host(desc, q_host, k_host, v_host, window, budgets, out_host, q_dev, k_dev, v_dev, out_dev, ws,
                     stream=None):
    _check(lib().tsa_forward_host(ctypes.byref(desc), _ptr(q_host), _ptr(k_host), _ptr(v_host), int(window),
                                  _budgets(budgets), _ptr(out_host), _ptr(q_dev), _ptr(k_dev), _ptr(v_dev),
                                  _ptr(out_dev), _ptr(ws), ws.numel(), _stream(stream)), "tsa_forward_host")


def tsa_forward_host_h2d_bytes(desc, window, budgets, q_host, v_host) -> int:
    """Host-to-device bytes ``tsa_forward_host`` moves for these host inputs (0 for invalid arguments)."""
    return int(lib().tsa_forward_host_h2d_bytes(ctypes.byref(desc), int(window), _budgets(budgets), _ptr(q_host),
                                                _ptr(v_host)))


def tsa_check_status(ws, stream=None) -> int:
    """Synchronise, return the device status code recorded in ``ws`` (0 = ok) and clear it.

    ``ws=None`` reads the status word of ``tsa_score_noalloc`` on the current device."""
    return int(lib().tsa_check_status(_ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def tsa_score_noalloc(desc, q, k, window, scores, stream=None):
    """tsa_score with the library's fixed scratch instead of a caller workspace."""
    _check(lib().tsa_score_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k), int(window), _ptr(scores),
                                   _stream(stream)), "tsa_score_noalloc")


def tsa_status_string(code: int) -> str:
    return lib().tsa_status_string(int(code)).decode()


def tsa_debug_set_wait_limit(polls: int):
    lib().tsa_debug_set_wait_limit(int(polls))


def tsa_debug_wait_never_set(ws, stream=None):
    _check(lib().tsa_debug_wait_never_set(_ptr(ws), ws.numel(), _stream(stream)), "tsa_debug_wait_never_set")


def tsa_debug_launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(lib().tsa_debug_launch_count())


def tsa_debug_cta_pair_launch_count() -> int:
    """Launches of the two-SM attention kernel (opt-in: TSA_ATTEND_CTA_PAIRS=1) so far in this process."""
    return int(lib().tsa_debug_cta_pair_launch_count())


def tsa_score_noalloc(desc, q, k, window, scores, stream=None):
    """tsa_score for callers that cannot allocate: no workspace argument; the
    library's fixed device scratch is used (see include/tsa.h)."""
    _check(lib().tsa_score_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k), int(window), _ptr(scores),
                                   _stream(stream)), "tsa_score_noalloc")


def tsa_drift_workspace_size() -> int:
    return int(lib().tsa_drift_workspace_size())


def alloc_drift_workspace(device="cuda") -> torch.Tensor:
    return torch.empty(tsa_drift_workspace_size(), dtype=torch.uint8, device=device)


def tsa_drift(h_before, h_after, drift, ws, row_cos=None, stream=None):
    """drift[0] = 1 - mean row cosine of two [..., hidden] tensors (f32 or bf16, contiguous);
    row_cos (float32, one per row) receives the cosines when given."""
    if h_before.shape != h_after.shape or h_before.dtype != h_after.dtype:
        raise ValueError("h_before and h_after must have the same shape and dtype")
    if not (h_before.is_contiguous() and h_after.is_contiguous()):
        raise ValueError("hidden states must be contiguous")
    hidden = int(h_before.shape[-1])
    rows = h_before.numel() // max(hidden, 1)
    dtype = TSA_BF16 if h_before.dtype == torch.bfloat16 else TSA_F32 if h_before.dtype == torch.float32 else -1
    _check(lib().tsa_drift(rows, hidden, dtype, _ptr(h_before), _ptr(h_after), _ptr(row_cos), _ptr(drift),
                           _ptr(ws), ws.numel(), _stream(stream)), "tsa_drift")


def tsa_layer_stable(history, window: int = 3, threshold: float = 0.1) -> bool:
    """Window stability rule on host drifts (newest last)."""
    n = len(history)
    arr = (ctypes.c_double * max(n, 1))(*[float(x) for x in history])
    out = ctypes.c_int32(0)
    _check(lib().tsa_layer_stable(arr, n, int(window), float(threshold), ctypes.byref(out)), "tsa_layer_stable")
    return bool(out.value)


def tsa_select_coverage(desc, scores, tau, perm, budgets_out, ws, stream=None):
    """Top-K per KV head with K chosen from the coverage tau; budgets_out (int32 device) receives K."""
    _check(lib().tsa_select_coverage(ctypes.byref(desc), _ptr(scores), float(tau), _ptr(perm), _ptr(budgets_out),
                                     _ptr(ws), ws.numel(), _stream(stream)), "tsa_select_coverage")


def tsa_forward_coverage(desc, q, k, v, window, tau, out, ws, scores=None, perm=None, stream=None):
    """Score, coverage selection and attention; returns the chosen budgets (list of int)."""
    n = desc.B * desc.Hkv
    arr = (ctypes.c_int32 * n)()
    _check(lib().tsa_forward_coverage(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), int(window), float(tau), arr,
                                      _ptr(scores), _ptr(perm), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "tsa_forward_coverage")
    return list(arr)


def tsa_attend_block_sparse(desc, q, k, v, perm, budgets, block_mask, out, ws, stream=None):
    """tsa_attend restricted by a uint8 [B, Hkv, nb, nb] mask over 128 x 128 blocks of compacted (query, key)."""
    nb = (desc.L + 127) // 128
    if block_mask.dtype != torch.uint8 or block_mask.numel() != desc.B * desc.Hkv * nb * nb:
        raise ValueError("block_mask must be uint8 [B, Hkv, ceil(L/128), ceil(L/128)]")
    if not block_mask.is_contiguous():
        raise ValueError("block_mask must be contiguous")
    _check(lib().tsa_attend_block_sparse(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(perm), _budgets(budgets),
                                         _ptr(block_mask), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "tsa_attend_block_sparse")


def tsa_debug_exp2(x, y, stream=None):
    """y = 2^x through the library's FMA-pipe exponential (testing hook)."""
    _check(lib().tsa_debug_exp2(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "tsa_debug_exp2")
