"""Thin Python binding of libpi_ffn.so (include/pi_ffn.h).

Argument marshalling only: every function here has the name of the C entry
point it calls, turns torch tensors into device/host pointers, and raises
``PiError`` on a non-OK status.  Every step of the sparse FFN runs in the
library's CUDA kernels; nothing here computes.  Loading fails loudly when the
library has not been built.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpi_ffn.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "pi_ffn.h")

PI_OK, PI_ERR_INVALID_ARG, PI_ERR_UNSUPPORTED, PI_ERR_OOM = 0, 1, 2, 3
PI_ERR_CUDA, PI_ERR_TIMEOUT, PI_ERR_DEVICE_CHECK, PI_ERR_NOT_LOADED = 4, 5, 6, 7
STATUS = {0: "PI_OK", 1: "PI_ERR_INVALID_ARG", 2: "PI_ERR_UNSUPPORTED", 3: "PI_ERR_OOM",
          4: "PI_ERR_CUDA", 5: "PI_ERR_TIMEOUT", 6: "PI_ERR_DEVICE_CHECK", 7: "PI_ERR_NOT_LOADED"}
ACT = {"relu": 0, "reglu": 1, "drelu": 2}
DTYPE = {"f32": 0, "f16": 1, "bf16": 2, "int4g32": 3, "i8row": 4}
PI_DEBUG_STALL_BARRIER = 1
PI_DEBUG_STALL_PREFILL = 2
PI_DEBUG_STALL_T_POLL = 8


class PiError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")
        self.status = status


class pi_ffn_desc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("d_model", ctypes.c_int), ("d_ff", ctypes.c_int),
                ("rank", ctypes.c_int), ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
                ("act", ctypes.c_int), ("w_dtype", ctypes.c_int), ("pred_dtype", ctypes.c_int),
                ("n_strips", ctypes.c_int), ("threshold", ctypes.c_float), ("eps", ctypes.c_float),
                ("device", ctypes.c_int)]


class pi_expert_weights(ctypes.Structure):
    _fields_ = [("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("s_gate", ctypes.c_void_p), ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("U", ctypes.c_void_p), ("V", ctypes.c_void_p),
                ("s_U", ctypes.c_void_p), ("s_V", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it was never built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m activation_sparse_decode_threshold_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, ip = ctypes.c_void_p, ctypes.c_int
        sigs = {
            "pi_ffn_create": [ctypes.POINTER(pi_ffn_desc), ctypes.POINTER(vp)],
            "pi_ffn_load_layer": [vp, ip, ctypes.POINTER(pi_expert_weights), vp, vp, vp],
            "pi_neuron_table": [vp, ip, ip, vp],
            "pi_strip_offsets": [vp, vp, ctypes.POINTER(ip)],
            "pi_predict": [vp, ip, ip, vp, vp, vp, vp, vp],
            "pi_sparse_ffn_decode": [vp, ip, ip, vp, vp, vp, vp, vp],
            "pi_sparse_ffn_decode_host": [vp, ip, ip, vp, vp, vp],
            "pi_sparse_ffn_decode_batch": [vp, ip, ip, ip, vp, vp, vp, vp, vp],
            "pi_sparse_ffn_decode_partial": [vp, ip, vp, vp, vp, vp, vp],
            "pi_residual_add": [vp, vp, vp, vp],
            "pi_ffn_set_hot_neurons": [vp, ip],
            "pi_dense_ffn_prefill": [vp, ip, ip, ip, vp, vp],
            "pi_sync": [vp, vp],
            "pi_debug_set": [vp, ip, ctypes.c_double],
            "pi_debug_phase_times": [vp, vp],
            "pi_predict_noalloc": [ip, ip, ip, ip, ctypes.c_float, vp, vp, vp, vp, vp, vp, vp, vp],
        }
        for name, args in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.pi_last_error.argtypes = []
        L.pi_last_error.restype = ctypes.c_char_p
        L.pi_ffn_destroy.argtypes = [vp]
        L.pi_ffn_destroy.restype = None
        _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Entry points declared in include/pi_ffn.h."""
    with open(HEADER) as f:
        return re.findall(r"^PI_API\s+[^(]*?\b(pi_\w+)\s*\(", f.read(), flags=re.M)


def _check(st: int, where: str):
    if st != PI_OK:
        raise PiError(st, where, lib().pi_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def pi_last_error() -> str:
    return lib().pi_last_error().decode()


def pi_ffn_create(n_layers, d_model, d_ff, rank, act="reglu", w_dtype="f16", pred_dtype="f16",
                  n_experts=1, top_k=1, n_strips=0, threshold=0.0, eps=1e-6, device=0) -> int:
    desc = pi_ffn_desc(n_layers, d_model, d_ff, rank, n_experts, top_k, ACT[act], DTYPE[w_dtype],
                       DTYPE[pred_dtype], n_strips, threshold, eps, device)
    h = ctypes.c_void_p()
    _check(lib().pi_ffn_create(ctypes.byref(desc), ctypes.byref(h)), "pi_ffn_create")
    return h.value


def pi_ffn_destroy(h: int):
    if h:
        lib().pi_ffn_destroy(h)


def pi_ffn_load_layer(h, layer, experts, router=None, freq=None, stream=None):
    """`experts`: list of objects with attributes w_gate, w_up, w_down, s_gate,
    s_up, s_down, c (bias), U, V, sU, sV (device tensors, None where absent).
    `freq`: host float32 array (n_experts x F) or None."""
    import numpy as np
    arr = (pi_expert_weights * len(experts))()
    for i, e in enumerate(experts):
        arr[i] = pi_expert_weights(_ptr(e.w_gate), _ptr(e.w_up), _ptr(e.w_down),
                                   _ptr(getattr(e, "s_gate", None)), _ptr(getattr(e, "s_up", None)),
                                   _ptr(getattr(e, "s_down", None)), _ptr(e.c), _ptr(e.U), _ptr(e.V),
                                   _ptr(getattr(e, "sU", None)), _ptr(getattr(e, "sV", None)))
    fq = None
    if freq is not None:
        fq = np.ascontiguousarray(np.asarray(freq, np.float32))
    _check(lib().pi_ffn_load_layer(h, layer, arr, _ptr(router),
                                   None if fq is None else fq.ctypes.data, _stream(stream)),
           "pi_ffn_load_layer")


def pi_ffn_set_hot_neurons(h, hot_per_strip: int):
    _check(lib().pi_ffn_set_hot_neurons(h, hot_per_strip), "pi_ffn_set_hot_neurons")


def pi_neuron_table(h, layer, expert, F):
    import numpy as np
    perm = np.empty(F, np.int32)
    _check(lib().pi_neuron_table(h, layer, expert, perm.ctypes.data), "pi_neuron_table")
    return perm


def pi_strip_offsets(h):
    import numpy as np
    n = ctypes.c_int()
    _check(lib().pi_strip_offsets(h, None, ctypes.byref(n)), "pi_strip_offsets")
    off = np.empty(n.value + 1, np.int32)
    _check(lib().pi_strip_offsets(h, off.ctypes.data, None), "pi_strip_offsets")
    return off


def pi_predict(h, layer, expert, x, idx, count, z=None, stream=None):
    _check(lib().pi_predict(h, layer, expert, _ptr(x), _ptr(idx), _ptr(count), _ptr(z),
                            _stream(stream)), "pi_predict")


def pi_sparse_ffn_decode(h, layer_begin, layer_end, resid, trace=None, stats=None, masks=None,
                         stream=None):
    _check(lib().pi_sparse_ffn_decode(h, layer_begin, layer_end, _ptr(resid), _ptr(trace),
                                      _ptr(stats), _ptr(masks), _stream(stream)),
           "pi_sparse_ffn_decode")


def pi_sparse_ffn_decode_batch(h, layer_begin, layer_end, resid, trace=None, stats=None, masks=None,
                               stream=None):
    """`resid`: device float32 tensor [n_tokens x d] (n_tokens = resid.shape[0])."""
    _check(lib().pi_sparse_ffn_decode_batch(h, layer_begin, layer_end, int(resid.shape[0]), _ptr(resid),
                                            _ptr(trace), _ptr(stats), _ptr(masks), _stream(stream)),
           "pi_sparse_ffn_decode_batch")


def pi_sparse_ffn_decode_partial(h, layer, resid, y, stats=None, masks=None, stream=None):
    _check(lib().pi_sparse_ffn_decode_partial(h, layer, _ptr(resid), _ptr(y), _ptr(stats), _ptr(masks),
                                              _stream(stream)), "pi_sparse_ffn_decode_partial")


def pi_residual_add(h, resid, y, stream=None):
    _check(lib().pi_residual_add(h, _ptr(resid), _ptr(y), _stream(stream)), "pi_residual_add")


def pi_sparse_ffn_decode_host(h, layer_begin, layer_end, resid_in, resid_out, stream=None):
    """resid_in / resid_out: host (ideally pinned) float32 tensors of d entries."""
    _check(lib().pi_sparse_ffn_decode_host(h, layer_begin, layer_end, _ptr(resid_in),
                                           _ptr(resid_out), _stream(stream)),
           "pi_sparse_ffn_decode_host")


def pi_dense_ffn_prefill(h, layer_begin, layer_end, n_tokens, resid, stream=None):
    _check(lib().pi_dense_ffn_prefill(h, layer_begin, layer_end, n_tokens, _ptr(resid),
                                      _stream(stream)), "pi_dense_ffn_prefill")


def pi_sync(h, stream=None) -> int:
    """Returns the status (does not raise), so callers can test for timeouts."""
    return lib().pi_sync(h, _stream(stream))


def pi_debug_set(h, flags: int, wait_limit_s: float):
    _check(lib().pi_debug_set(h, flags, wait_limit_s), "pi_debug_set")


def pi_debug_phase_times(h, times=None):
    _check(lib().pi_debug_phase_times(h, _ptr(times)), "pi_debug_phase_times")


def pi_predict_noalloc(d_model, d_ff, rank, pred_dtype, threshold, V, U, bias, x, idx, count, z=None,
                       stream=None):
    """Predictor on caller-owned weights (original order) with no device allocation."""
    _check(lib().pi_predict_noalloc(d_model, d_ff, rank, DTYPE[pred_dtype], threshold, _ptr(V), _ptr(U),
                                    _ptr(bias), _ptr(x), _ptr(idx), _ptr(count), _ptr(z), _stream(stream)),
           "pi_predict_noalloc")
