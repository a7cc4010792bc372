"""Helpers of the GPU parity tests: build a library handle from synthetic
weights, convert the same weights for the oracle, and compare results."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
from activation_sparse_decode_threshold_b200 import binding as B
from activation_sparse_decode_threshold_b200 import synth

# Parity bar (per layer, teacher-forced): predicted-active sets identical in
# original numbering except neurons with |z_oracle| < Z_BAND; layer outputs
# within rel-L2 5e-3 and max-abs 2e-2 of the fp64 oracle.
Z_BAND = 1e-3
REL_L2 = 5e-3
MAX_ABS = 2e-2


# Achieved errors of each parity check, by case name; written as JSON to the
# file named by PI_PARITY_LOG (if set) when the test session ends, so the
# headroom against the bar is on record per workload.
ERRORS: dict = {}


def record_error(case: str, **vals):
    row = ERRORS.setdefault(case, {})
    for k, v in vals.items():
        if isinstance(v, (int, np.integer)):
            row[k] = max(int(v), int(row.get(k, v)))
        else:
            row[k] = max(float(v), float(row.get(k, v)))


def write_errors():
    path = os.environ.get("PI_PARITY_LOG")
    if path and ERRORS:
        with open(path, "w") as f:
            json.dump(ERRORS, f, indent=1, sort_keys=True)


def oracle_expert(cfg: synth.FFNConfig, e: synth.ExpertWeights) -> oracle.Expert:
    n = synth.to_numpy
    return oracle.Expert(act=cfg.act, wdtype=cfg.wdtype, pdtype=cfg.pdtype, w_gate=n(e.w_gate),
                         w_up=n(e.w_up), w_down=n(e.w_down), c=n(e.c), U=n(e.U), V=n(e.V),
                         s_gate=n(e.s_gate), s_up=n(e.s_up), s_down=n(e.s_down),
                         sU=n(e.sU), sV=n(e.sV))


def oracle_layer(cfg, lw: synth.LayerWeights):
    experts = [oracle_expert(cfg, e) for e in lw.experts]
    router = None if lw.router is None else synth.to_numpy(lw.router)
    return experts, router


def create(cfg: synth.FFNConfig, n_layers: int | None = None, n_strips: int = 0,
           threshold: float = 0.0) -> int:
    return B.pi_ffn_create(n_layers or cfg.n_layers, cfg.d, cfg.F, cfg.rank, act=cfg.act,
                           w_dtype=cfg.wdtype, pred_dtype=cfg.pdtype, n_experts=cfg.n_experts,
                           top_k=cfg.top_k, n_strips=n_strips, threshold=threshold)


def freq_of(lw: synth.LayerWeights) -> np.ndarray:
    return np.stack([e.freq for e in lw.experts]).astype(np.float32)


def load(h: int, layer: int, lw: synth.LayerWeights, use_freq: bool = True):
    B.pi_ffn_load_layer(h, layer, lw.experts, lw.router, freq_of(lw) if use_freq else None)


def tables(h: int, lw: synth.LayerWeights, layer: int, F: int):
    return [B.pi_neuron_table(h, layer, e, F) for e in range(len(lw.experts))]


def masks_to_original(words: np.ndarray, perm: np.ndarray, F: int) -> np.ndarray:
    """Bit mask in table order (uint32 words) -> boolean mask in original order."""
    bits = np.unpackbits(words.view(np.uint8), bitorder="little")[:F].astype(bool)
    out = np.zeros(F, bool)
    out[perm[bits.nonzero()[0]]] = True
    return out


def check_active_set(gpu_mask: np.ndarray, z_oracle: np.ndarray, band: float = Z_BAND) -> int:
    """Sets must agree except where |z_oracle| < band; returns how many band
    neurons differ."""
    ref = z_oracle > 0
    diff = np.nonzero(gpu_mask != ref)[0]
    bad = diff[np.abs(z_oracle[diff]) >= band]
    assert bad.size == 0, (f"{bad.size} neurons outside the |z| < {band} band differ, e.g. "
                           f"{bad[:5].tolist()} with z = {z_oracle[bad[:5]].tolist()}")
    return int(diff.size)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def check_output(y_gpu: np.ndarray, y_ref: np.ndarray):
    rl = rel_l2(y_gpu, y_ref)
    ma = float(np.max(np.abs(y_gpu - y_ref)))
    assert rl <= REL_L2 and ma <= MAX_ABS, f"rel-L2 {rl:.3e}, max-abs {ma:.3e}"
    return rl, ma


def decode_traced(h: int, cfg, l0: int, l1: int, r0: torch.Tensor):
    """One token through layers [l0, l1) with trace, stats and masks."""
    nl = l1 - l0
    resid = r0.clone().cuda()
    trace = torch.empty((nl, cfg.d), device="cuda", dtype=torch.float32)
    stats = torch.empty((nl, 4), device="cuda", dtype=torch.int32)
    words = (cfg.F + 31) // 32
    masks = torch.empty((nl, cfg.top_k, words), device="cuda", dtype=torch.int32)
    B.pi_sparse_ffn_decode(h, l0, l1, resid, trace, stats, masks)
    assert B.pi_sync(h) == B.PI_OK, B.pi_last_error()
    return (resid.cpu().double().numpy(), trace.cpu().double().numpy(),
            stats.cpu().numpy(), masks.cpu().numpy().view(np.uint32))


def check_layer(cfg, experts, router, perms, r_in: np.ndarray, r_out: np.ndarray,
                stats_row: np.ndarray, mask_rows: np.ndarray, case: str | None = None):
    """Teacher-forced parity of one layer: routing, predicted sets, output."""
    x = oracle.rmsnorm(r_in)
    if router is None:
        use, wts = [0], [1.0]
    else:
        logits, ex, w = oracle.route_top2(x, router)
        use, wts = [int(ex[0]), int(ex[1])], [float(w[0]), float(w[1])]
        gpu_use = [int(stats_row[2]), int(stats_row[3])]
        if gpu_use != use:
            srt = np.sort(logits)[::-1]
            assert srt[1] - srt[2] < Z_BAND, f"experts {gpu_use} vs oracle {use}"
            use = gpu_use
            p = np.exp(logits - logits.max())
            p = p / p.sum()
            wts = [p[use[0]] / (p[use[0]] + p[use[1]]), p[use[1]] / (p[use[0]] + p[use[1]])]
    y = np.zeros_like(r_in)
    n_pred = n_nz = band = 0
    for slot, (e_id, w_e) in enumerate(zip(use, wts)):
        e = experts[e_id]
        _, z, _ = oracle.predict(x, e.V, e.U, e.c, e.pdtype, 0.0, e.sV, e.sU)
        gm = masks_to_original(mask_rows[slot], perms[e_id], cfg.F)
        band += check_active_set(gm, z)
        h, y_e = oracle.ffn_masked(e, x, gm.astype(np.uint8))   # the GPU's (valid) selection
        y = y_e if router is None else y + w_e * y_e
        n_pred += int(gm.sum())
        n_nz += int(np.count_nonzero(h))
    assert int(stats_row[0]) == n_pred
    assert abs(int(stats_row[1]) - n_nz) <= max(2, n_pred // 500)
    rl, ma = check_output(r_out - r_in, y)
    if case:
        record_error(case, rel_l2=rl, max_abs=ma, band=band)
    return dict(rel_l2=rl, max_abs=ma, band=band, active=n_pred, nonzero=n_nz)
