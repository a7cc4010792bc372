"""C-ABI library: loads, exports every entry point declared in include/pi_ffn.h,
and rejects bad arguments on the host before touching a device (CPU only)."""
import ctypes

import pytest

from activation_sparse_decode_threshold_b200 import binding as B


def test_library_exports_every_declared_symbol():
    L = B.lib()
    names = B.header_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    for n in ("pi_ffn_create", "pi_ffn_load_layer", "pi_neuron_table", "pi_predict",
              "pi_sparse_ffn_decode", "pi_sparse_ffn_decode_host", "pi_dense_ffn_prefill",
              "pi_sync", "pi_last_error", "pi_ffn_destroy"):
        assert n in names


def _desc(**kw):
    base = dict(n_layers=2, d_model=4096, d_ff=11008, rank=1024, n_experts=1, top_k=1,
                act=1, w_dtype=1, pred_dtype=1, n_strips=0, threshold=0.0, eps=1e-6, device=0)
    base.update(kw)
    return B.pi_ffn_desc(**base)


@pytest.mark.parametrize("bad, status", [
    (dict(n_layers=0), B.PI_ERR_INVALID_ARG),
    (dict(d_model=300), B.PI_ERR_INVALID_ARG),
    (dict(d_model=16384), B.PI_ERR_INVALID_ARG),
    (dict(d_model=8192, w_dtype=0, pred_dtype=0), B.PI_ERR_UNSUPPORTED),
    (dict(d_ff=0), B.PI_ERR_INVALID_ARG),
    (dict(rank=1001), B.PI_ERR_INVALID_ARG),
    (dict(rank=2048), B.PI_ERR_INVALID_ARG),
    (dict(act=7), B.PI_ERR_INVALID_ARG),
    (dict(w_dtype=9), B.PI_ERR_INVALID_ARG),
    (dict(pred_dtype=3), B.PI_ERR_INVALID_ARG),
    (dict(w_dtype=1, pred_dtype=2), B.PI_ERR_UNSUPPORTED),
    (dict(n_experts=1, top_k=2), B.PI_ERR_INVALID_ARG),
    (dict(n_experts=8, top_k=1), B.PI_ERR_UNSUPPORTED),
    (dict(n_experts=40, top_k=2), B.PI_ERR_INVALID_ARG),
    (dict(eps=0.0), B.PI_ERR_INVALID_ARG),
    (dict(threshold=float("inf")), B.PI_ERR_INVALID_ARG),
    (dict(d_model=128), B.PI_ERR_INVALID_ARG),
    (dict(rank=0), B.PI_ERR_INVALID_ARG),
    (dict(w_dtype=0, pred_dtype=0, rank=1024), B.PI_ERR_INVALID_ARG),   # fp32 rows hold <= 512
    (dict(w_dtype=3, pred_dtype=0), B.PI_ERR_UNSUPPORTED),              # INT4 with an fp32 predictor
    (dict(n_experts=8, top_k=2, w_dtype=0, pred_dtype=0, rank=256), B.PI_ERR_UNSUPPORTED),
    (dict(pred_dtype=4, rank=1008), B.PI_ERR_INVALID_ARG),   # the 8-bit predictor takes 32 columns per step
])
def test_create_rejects_bad_descriptors_on_host(bad, status):
    h = ctypes.c_void_p()
    st = B.lib().pi_ffn_create(ctypes.byref(_desc(**bad)), ctypes.byref(h))
    assert st == status, B.pi_last_error()
    assert h.value is None
    assert B.pi_last_error()


def test_null_arguments_rejected():
    L = B.lib()
    assert L.pi_ffn_create(None, None) == B.PI_ERR_INVALID_ARG
    assert L.pi_sparse_ffn_decode(None, 0, 1, None, None, None, None, None) == B.PI_ERR_INVALID_ARG
    assert L.pi_predict(None, 0, 0, None, None, None, None, None) == B.PI_ERR_INVALID_ARG
    assert L.pi_ffn_load_layer(None, 0, None, None, None, None) == B.PI_ERR_INVALID_ARG
    assert L.pi_neuron_table(None, 0, 0, None) == B.PI_ERR_INVALID_ARG
    assert L.pi_dense_ffn_prefill(None, 0, 1, 4, None, None) == B.PI_ERR_INVALID_ARG
    assert L.pi_sync(None, None) == B.PI_ERR_INVALID_ARG
    assert L.pi_debug_set(None, 0, 1.0) == B.PI_ERR_INVALID_ARG
    L.pi_ffn_destroy(None)


def test_binding_raises_with_message():
    with pytest.raises(B.PiError) as ei:
        B.pi_ffn_create(0, 4096, 11008, 1024)
    assert ei.value.status == B.PI_ERR_INVALID_ARG
    assert "n_layers" in str(ei.value)
