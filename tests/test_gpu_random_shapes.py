"""GPU parity over a seeded sweep of small random shapes, formats, activations,
strip counts and sparsities (decode, teacher-forced per layer against the fp64
oracle), plus the dense prefill on the same layers.  The shapes exercise
ragged strips, strips longer than one staging round, column slices of several
widths and both d_model classes of the kernels."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_decode_threshold_b200 import binding as B
from activation_sparse_decode_threshold_b200 import synth
import gpu_util as G

pytestmark = pytest.mark.gpu

_BASE = {"reglu": "llama7b", "drelu": "mistral7b", "relu": "falcon40b"}
_FMT = [("f16", "f16"), ("bf16", "bf16"), ("int4g32", "f16"), ("int4g32", "bf16"), ("f32", "f32")]


def _cases(n=10, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        act = ["reglu", "drelu", "relu"][i % 3]
        wd, pd = _FMT[rng.integers(len(_FMT))]
        d = int(rng.choice([256, 512, 768, 1024] if wd != "f32" else [256, 512]))
        F = int(rng.integers(60, 3000)) if i % 2 else 128 * int(rng.integers(1, 24))
        rank = int(rng.choice([16, 32, 48, 64, 128]))
        strips = int(rng.choice([0, 7, 33, 148]))
        active = float(rng.choice([0.05, 0.1, 0.3]))
        out.append(pytest.param(act, wd, pd, d, F, rank, strips, active, 1,
                                id=f"{act}-{wd}-{pd}-d{d}-F{F}-r{rank}-S{strips}-a{active}"))
    # MoE layers (top-2 over 4 or 6 experts, 16-bit predictors)
    for i in range(3):
        wd, pd = [("int4g32", "f16"), ("f16", "f16"), ("bf16", "bf16")][i]
        d = int(rng.choice([256, 512]))
        F = 128 * int(rng.integers(2, 12))
        E = int(rng.choice([4, 6]))
        out.append(pytest.param("drelu" if i != 1 else "reglu", wd, pd, d, F, 32, 0, 0.1, E,
                                id=f"moe{E}-{wd}-{pd}-d{d}-F{F}"))
    return out


@pytest.fixture
def handles():
    hs = []
    yield hs
    torch.cuda.synchronize()
    for h in hs:
        B.pi_ffn_destroy(h)


@pytest.mark.parametrize("act,wd,pd,d,F,rank,strips,active,E", _cases())
def test_random_shape_decode(handles, act, wd, pd, d, F, rank, strips, active, E):
    base = "mixtral47b" if E > 1 else _BASE[act]
    cfg = synth.small(synth.CONFIGS[base], n_layers=2, d=d, F=F, rank=rank, wdtype=wd, pdtype=pd,
                      mean_active=active, act=act, n_experts=E, top_k=2 if E > 1 else 1)
    h = G.create(cfg, cfg.n_layers, n_strips=strips)
    handles.append(h)
    lws = [synth.make_layer(cfg, l, "cuda") for l in range(cfg.n_layers)]
    for l, lw in enumerate(lws):
        G.load(h, l, lw)
    olayers = [G.oracle_layer(cfg, lw) for lw in lws]
    perms = [G.tables(h, lw, l, cfg.F) for l, lw in enumerate(lws)]
    for t in range(2):
        rL, trace, stats, masks = G.decode_traced(h, cfg, 0, cfg.n_layers, synth.token_input(cfg, t))
        outs = list(trace[1:]) + [rL]
        for l in range(cfg.n_layers):
            ex, router = olayers[l]
            G.check_layer(cfg, ex, router, perms[l], trace[l], outs[l], stats[l], masks[l],
                          case="decode/random-shapes")
    # the dense prefill of the same layer where its shape allows it
    if wd != "f32" and d % 256 == 0 and F % 128 == 0:
        R = synth.prefill_input(cfg, 96, "cuda")
        out = R.clone()
        B.pi_dense_ffn_prefill(h, 0, 1, 96, out)
        assert B.pi_sync(h) == B.PI_OK
        ex, router = olayers[0]
        Rn = R.double().cpu().numpy()
        res = oracle.prefill_layer(Rn, ex, router)
        ok = np.ones(Rn.shape[0], bool)
        if res.logits is not None:   # tokens whose top-2 choice is within rounding are left out
            srt = np.sort(res.logits, axis=1)[:, ::-1]
            ok = (srt[:, 1] - srt[:, 2]) > 1e-4
        y_gpu = out.double().cpu().numpy() - Rn
        G.check_output(y_gpu[ok].ravel(), res.y[ok].ravel())
