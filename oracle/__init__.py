"""fp64 CPU oracle for the predictor-guided sparse FFN (test infrastructure).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; the library never imports it and it
imports nothing from the library.  The arithmetic lives in ``oracle.c`` (plain
ascending double-precision loops); this module only marshals numpy arrays and
chains the per-layer steps in the order the pages give them:

  layer input  x = RMSNorm(r)                       (reading: parameterless, eps 1e-6)
  [MoE] route  two experts, softmax weights          (TurboSparse-Mixtral-shaped layer)
  predict      t = V x, z = U t - c, active = z > 0  (PowerInfer (unite.ai), "Adaptive sparse predictor")
  compute      active rows of W_gate/W_up, columns of W_down only
                                                     (PowerInfer (unite.ai), "Neuron-aware operators")
  merge        y summed over neurons in original order (nearauto, "PowerInfer architecture", Fig. 8)
  residual     r <- r + y

Weights are numpy arrays in their stored format: float32, float16, bfloat16
as uint16 bit patterns, or INT4 group-32 as uint8 nibbles plus float16
scales.  W_down is d x F for float formats and neuron-major F x d for INT4.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPES = {"f32": 0, "f16": 1, "bf16": 2, "int4g32": 3, "i8row": 4}
ACTS = {"relu": 0, "reglu": 1, "drelu": 2}
EPS = 1e-6


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB + ".tmp", _SRC, "-lm"]
        )
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        vp, ip, dp = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.or_half_to_double.restype = dp
        L.or_half_to_double.argtypes = [ctypes.c_uint16]
        L.or_bf16_to_double.restype = dp
        L.or_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.or_dequant_int4_g32.argtypes = [vp, vp, ip, vp]
        L.or_load_row.argtypes = [ip, vp, vp, ctypes.c_long, ip, vp]
        L.or_rmsnorm.argtypes = [vp, ip, dp, vp]
        L.or_predict.argtypes = [ip, ip, ip, ip, vp, vp, vp, dp, vp, vp, vp, vp]
        L.or_predict_q.argtypes = [ip, ip, ip, ip, vp, vp, vp, vp, vp, dp, vp, vp, vp, vp]
        L.or_ffn_masked.argtypes = [ip, ip, ip, ip, vp, vp, vp, vp, vp, vp, ip, vp, vp, vp, vp, vp]
        L.or_route_top2.argtypes = [ip, ip, ip, vp, vp, vp, vp, vp]
        L.or_strip_offsets.argtypes = [ip, ip, vp]
        L.or_neuron_table.argtypes = [ip, ip, vp, vp]
        for f in ("or_dequant_int4_g32", "or_load_row", "or_rmsnorm", "or_predict", "or_predict_q",
                  "or_ffn_masked", "or_route_top2", "or_strip_offsets", "or_neuron_table"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype=None):
    if a is None:
        return None
    a = np.asarray(a)
    if dtype is not None:
        a = a.astype(dtype, copy=False)
    return np.ascontiguousarray(a)


# --------------------------------------------------------------------------
# Single steps
# --------------------------------------------------------------------------
def half_to_double(bits: int) -> float:
    return lib().or_half_to_double(int(bits) & 0xFFFF)


def bf16_to_double(bits: int) -> float:
    return lib().or_bf16_to_double(int(bits) & 0xFFFF)


def dequant_int4_g32(q: np.ndarray, scales: np.ndarray, n: int) -> np.ndarray:
    """One neuron vector of n elements from n/2 nibble bytes and n/32 fp16 scales."""
    q = _c(q, np.uint8)
    s = _c(scales, np.float16)
    out = np.empty(n, np.float64)
    lib().or_dequant_int4_g32(_p(q), _p(s), n, _p(out))
    return out


def load_matrix(dtype: str, w: np.ndarray, scales: np.ndarray | None, rows: int, n: int) -> np.ndarray:
    """A stored matrix (rows x n) as float64, row by row through the oracle's decoder."""
    w = _c(w)
    s = _c(scales)
    out = np.empty((rows, n), np.float64)
    L = lib()
    for i in range(rows):
        L.or_load_row(DTYPES[dtype], _p(w), _p(s), i, n, out[i].ctypes.data_as(ctypes.c_void_p))
    return out


def rmsnorm(r: np.ndarray, eps: float = EPS) -> np.ndarray:
    r = _c(r, np.float64)
    x = np.empty_like(r)
    lib().or_rmsnorm(_p(r), r.shape[0], eps, _p(x))
    return x


def predict(x, V, U, c, pdtype: str, threshold: float = 0.0, sV=None, sU=None):
    """t = V x, z = U t - c, mask = z > threshold.  Returns (t, z, mask).
    For the "i8row" format V and U are signed bytes and sV, sU their per-row
    fp32 scales."""
    x = _c(x, np.float64)
    c = _c(c, np.float64)
    V = _c(V)
    U = _c(U)
    rank, d = V.shape
    F = U.shape[0]
    if pdtype == "i8row":
        assert sV is not None and sU is not None, "the i8row predictor needs row scales"
        sV, sU = _c(sV, np.float32), _c(sU, np.float32)
        assert sV.shape == (rank,) and sU.shape == (F,)
    t = np.empty(rank, np.float64)
    z = np.empty(F, np.float64)
    mask = np.empty(F, np.uint8)
    lib().or_predict_q(d, F, rank, DTYPES[pdtype], _p(V), _p(sV), _p(U), _p(sU), _p(c),
                       float(threshold), _p(x), _p(t), _p(z), _p(mask))
    return t, z, mask


@dataclass
class Expert:
    """One FFN (or one MoE expert) in stored format, original neuron order."""
    act: str                 # "relu" (non-gated), "reglu", "drelu"
    wdtype: str              # "f32" | "f16" | "bf16" | "int4g32"
    pdtype: str              # predictor format
    w_gate: np.ndarray       # F x d (W_1 when non-gated)
    w_up: np.ndarray | None  # F x d, None when non-gated
    w_down: np.ndarray       # d x F (float formats) or F x d neuron-major (INT4)
    c: np.ndarray            # F, float32 bias (enters as -c on the gate)
    U: np.ndarray            # F x rank
    V: np.ndarray            # rank x d
    s_gate: np.ndarray | None = None   # INT4 scales, F x d/32 fp16
    s_up: np.ndarray | None = None
    s_down: np.ndarray | None = None   # F x d/32 (per neuron column)
    sU: np.ndarray | None = None       # i8row predictor: fp32 scale per row of U (F)
    sV: np.ndarray | None = None       # and of V (rank)

    @property
    def d(self) -> int:
        return self.V.shape[1]

    @property
    def F(self) -> int:
        return self.U.shape[0]


def ffn_masked(e: Expert, x, mask=None):
    """h and y for the neurons in `mask` (None = all).  Returns (h, y)."""
    x = _c(x, np.float64)
    d, F = e.d, e.F
    h = np.empty(F, np.float64)
    y = np.empty(d, np.float64)
    m = None if mask is None else _c(mask, np.uint8)
    wg, wu, wd = _c(e.w_gate), _c(e.w_up), _c(e.w_down)
    sg, su, sd = _c(e.s_gate), _c(e.s_up), _c(e.s_down)
    c = _c(e.c, np.float64)
    lib().or_ffn_masked(d, F, ACTS[e.act], DTYPES[e.wdtype], _p(wg), _p(sg), _p(wu), _p(su),
                        _p(wd), _p(sd), 1 if e.wdtype == "int4g32" else 0,
                        _p(c), _p(x), _p(m), _p(h), _p(y))
    return h, y


def route_top2(x, Wr, rdtype: str = "f16"):
    """(logits, [e_lo, e_hi], [w_lo, w_hi])."""
    x = _c(x, np.float64)
    Wr = _c(Wr)
    E, d = Wr.shape
    logits = np.empty(E, np.float64)
    ex = np.empty(2, np.int32)
    w = np.empty(2, np.float64)
    lib().or_route_top2(d, E, DTYPES[rdtype], _p(Wr), _p(x), _p(logits), _p(ex), _p(w))
    return logits, ex, w


def strip_offsets(F: int, S: int) -> np.ndarray:
    off = np.empty(S + 1, np.int32)
    lib().or_strip_offsets(F, S, _p(off))
    return off


def neuron_table(F: int, S: int, freq=None) -> np.ndarray:
    perm = np.empty(F, np.int32)
    f = None if freq is None else _c(freq, np.float64)
    lib().or_neuron_table(F, S, _p(f), _p(perm))
    return perm


# --------------------------------------------------------------------------
# One decode layer and the stack
# --------------------------------------------------------------------------
@dataclass
class LayerResult:
    x: np.ndarray            # layer input after RMSNorm
    y: np.ndarray            # FFN output (sum over the two experts for MoE)
    r_out: np.ndarray        # r + y
    z: list                  # per expert used: predictor logits (original order)
    mask: list               # per expert used: predicted-active mask
    h: list                  # per expert used: activations (0 outside the mask)
    experts: list            # expert ids used (ascending)
    weights: list            # their combine weights (1.0 for a dense FFN)
    logits: np.ndarray | None = None   # router logits (MoE)


def decode_layer(r, experts: list, router=None, threshold: float = 0.0, eps: float = EPS) -> LayerResult:
    """One layer of batch-1 decode: RMSNorm -> [route] -> predict -> masked FFN -> residual."""
    r = _c(r, np.float64)
    x = rmsnorm(r, eps)
    logits = None
    if router is None:
        use, wts = [0], [1.0]
    else:
        logits, ex, w = route_top2(x, router)
        use, wts = [int(ex[0]), int(ex[1])], [float(w[0]), float(w[1])]
    y = np.zeros_like(r)
    zs, masks, hs = [], [], []
    for e_id, w_e in zip(use, wts):
        e = experts[e_id]
        _, z, mask = predict(x, e.V, e.U, e.c, e.pdtype, threshold, e.sV, e.sU)
        h, y_e = ffn_masked(e, x, mask)
        if router is None:
            y = y_e
        else:
            y = y + w_e * y_e          # combined in ascending expert index
        zs.append(z)
        masks.append(mask)
        hs.append(h)
    return LayerResult(x=x, y=y, r_out=r + y, z=zs, mask=masks, h=hs, experts=use,
                       weights=wts, logits=logits)


def decode_layer_batch(R, experts: list, router=None, threshold: float = 0.0,
                       eps: float = EPS):
    """One layer of small-batch decode (B independent tokens, rows of R).

    Each token is normalised, routed and predicted on its own.  The rows that
    are read are those of the union of the tokens' predicted sets (per expert),
    each read once for the whole batch; token b keeps its own set: its h is
    computed over the union and set to exactly 0 outside its own predicted set,
    so its output is its batch-1 output (nearauto.com PowerInfer article,
    "Experiments", Fig. 14: the sparse path keeps its gains at small batch
    sizes).  Returns (per-token LayerResults, per-expert union masks)."""
    R = np.atleast_2d(_c(R, np.float64))
    Bn = R.shape[0]
    X = [rmsnorm(R[b], eps) for b in range(Bn)]
    plans = []
    for b in range(Bn):
        if router is None:
            plans.append(([0], [1.0], None))
        else:
            lg, ex, w = route_top2(X[b], router)
            plans.append(([int(ex[0]), int(ex[1])], [float(w[0]), float(w[1])], lg))
    preds = {}
    union = {}
    for b, (use, _, _) in enumerate(plans):
        for e_id in use:
            e = experts[e_id]
            _, z, m = predict(X[b], e.V, e.U, e.c, e.pdtype, threshold, e.sV, e.sU)
            preds[(b, e_id)] = (z, m)
            union[e_id] = m.copy() if e_id not in union else (union[e_id] | m)
    out = []
    for b, (use, wts, lg) in enumerate(plans):
        y = np.zeros_like(R[b])
        zs, masks, hs = [], [], []
        for e_id, w_e in zip(use, wts):
            e = experts[e_id]
            z, m = preds[(b, e_id)]
            h_u, _ = ffn_masked(e, X[b], union[e_id])     # h over the rows read for the batch
            h = np.where(m.astype(bool), h_u, 0.0)          # the token's own set
            _, y_e = ffn_masked(e, X[b], (h != 0).astype(np.uint8))
            y = y_e if router is None else y + w_e * y_e
            zs.append(z)
            masks.append(m)
            hs.append(h)
        out.append(LayerResult(x=X[b], y=y, r_out=R[b] + y, z=zs, mask=masks, h=hs,
                               experts=use, weights=wts, logits=lg))
    return out, union


def decode_stack(r, layers: list, routers=None, threshold: float = 0.0):
    """Free-running stack: r_{l+1} = r_l + FFN_l(RMSNorm(r_l)).  `layers[l]` is a
    list of experts (one for a dense FFN).  Returns (r_final, [LayerResult])."""
    r = _c(r, np.float64)
    out = []
    for l, experts in enumerate(layers):
        res = decode_layer(r, experts, None if routers is None else routers[l], threshold)
        out.append(res)
        r = res.r_out
    return r, out


@dataclass
class PrefillResult:
    x: np.ndarray            # T x d normalised inputs
    y: np.ndarray            # T x d FFN outputs
    r_out: np.ndarray        # T x d residual after the layer
    experts: np.ndarray      # T x 2 experts used (-1 unused), ascending
    weights: np.ndarray      # T x 2 their combine weights
    logits: np.ndarray | None


def prefill_layer(R, experts: list, router=None, eps: float = EPS) -> PrefillResult:
    """One layer of dense multi-token prefill: every token row of R is
    normalised, routed (MoE) and passed through the full FFN of its expert(s)
    with no predictor (PowerInfer-2, "Neuron-cluster heterogeneous computing":
    prefill activates almost every neuron and runs dense).  Rows are
    independent; each is the decode layer with every neuron active."""
    R = np.atleast_2d(_c(R, np.float64))
    T, d = R.shape
    X = np.empty_like(R)
    Y = np.zeros_like(R)
    used = np.full((T, 2), -1, np.int32)
    wts = np.zeros((T, 2), np.float64)
    L = None if router is None else np.empty((T, router.shape[0]), np.float64)
    for t in range(T):
        x = rmsnorm(R[t], eps)
        X[t] = x
        if router is None:
            use, w = [0], [1.0]
        else:
            lg, ex, w2 = route_top2(x, router)
            L[t] = lg
            use, w = [int(ex[0]), int(ex[1])], [float(w2[0]), float(w2[1])]
        for k, (e_id, w_e) in enumerate(zip(use, w)):
            _, y_e = ffn_masked(experts[e_id], x, None)
            Y[t] = y_e if router is None else Y[t] + w_e * y_e
            used[t, k] = e_id
            wts[t, k] = w_e
    return PrefillResult(x=X, y=Y, r_out=R + Y, experts=used, weights=wts, logits=L)
