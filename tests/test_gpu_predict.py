"""GPU parity of pi_predict (the predictor alone) against the fp64 oracle, for
every predictor format and both d_model classes of the kernel, through the C
ABI.

pi_predict runs its own instantiations of the decode kernel (predictor-only
kinds, a dense one and a MoE one, both with the rows of t split over the
CTAs), so each is checked here on its own: the active set must equal
the oracle's outside the |z| < 1e-3 band and the logits must agree element by
element.  Full-size cases use the workloads' real layer shapes in the launch
configuration of the benchmark (one CTA per SM)."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_decode_threshold_b200 import binding as B
from activation_sparse_decode_threshold_b200 import synth
import gpu_util as G

pytestmark = pytest.mark.gpu

CASES = {
    # name: (config, expert index to predict)
    "small-f16-d4096-class": (synth.small(synth.CONFIGS["llama7b"], n_layers=1, d=768, F=2000, rank=128), 0),
    "small-f16-d8192-class": (synth.small(synth.CONFIGS["falcon40b"], n_layers=1, d=5120, F=1500, rank=64), 0),
    "small-bf16-d4096-class": (synth.small(synth.CONFIGS["mistral7b"], n_layers=1, d=1024, F=3000, rank=96), 0),
    "small-bf16-d8192-class": (synth.small(synth.CONFIGS["mistral7b"], n_layers=1, d=8192, F=700, rank=32), 0),
    "small-moe-f16": (synth.small(synth.CONFIGS["mixtral47b"], n_layers=1, d=512, F=1024, rank=64,
                                  n_experts=4), 3),
    "small-moe-bf16": (synth.small(synth.CONFIGS["mixtral47b"], n_layers=1, d=512, F=1100, rank=48,
                                   n_experts=3, pdtype="bf16", wdtype="int4g32"), 1),
    "small-i8-d4096-class": (synth.small(synth.CONFIGS["llama7b-i8pred"], n_layers=1, d=1024, F=2500, rank=256), 0),
    "small-i8-d8192-class": (synth.small(synth.CONFIGS["llama7b-i8pred"], n_layers=1, d=6144, F=900, rank=96), 0),
    "small-moe-i8": (synth.small(synth.CONFIGS["mixtral47b-i8pred"], n_layers=1, d=512, F=1000, rank=64,
                                 n_experts=3), 2),
    "full-llama7b-i8pred": (synth.small(synth.CONFIGS["llama7b-i8pred"], n_layers=1), 0),
    "full-mixtral47b-i8pred": (synth.small(synth.CONFIGS["mixtral47b-i8pred"], n_layers=1), 6),
    "full-llama7b": (synth.small(synth.CONFIGS["llama7b"], n_layers=1), 0),
    "full-falcon40b": (synth.small(synth.CONFIGS["falcon40b"], n_layers=1), 0),
    "full-mistral7b": (synth.small(synth.CONFIGS["mistral7b"], n_layers=1), 0),
    "full-mixtral47b": (synth.small(synth.CONFIGS["mixtral47b"], n_layers=1), 5),
}


def _z_tol(z_ref: np.ndarray) -> float:
    # fp32 dot products over r terms (t carried as 16-bit parts, exact products)
    return 1e-4 + 2e-5 * float(np.max(np.abs(z_ref)))


@pytest.mark.parametrize("name", sorted(CASES))
def test_predict_matches_oracle(name):
    cfg, expert = CASES[name]
    lw = synth.make_layer(cfg, 0, "cuda")
    h = G.create(cfg, 1)
    try:
        G.load(h, 0, lw)
        ex, _ = G.oracle_layer(cfg, lw)
        e = ex[expert]
        del lw
        torch.cuda.empty_cache()
        perm = B.pi_neuron_table(h, 0, expert, cfg.F)
        F = cfg.F
        idx = torch.empty(F, dtype=torch.int32, device="cuda")
        cnt = torch.empty(1, dtype=torch.int32, device="cuda")
        z = torch.empty(F, dtype=torch.float32, device="cuda")
        band = 0
        for t in (0, 1, 2):
            x32 = oracle.rmsnorm(synth.token_input(cfg, t).double().numpy()).astype(np.float32)
            B.pi_predict(h, 0, expert, torch.from_numpy(x32).cuda(), idx, cnt, z)
            assert B.pi_sync(h) == B.PI_OK, B.pi_last_error()
            n = int(cnt.item())
            got = idx[:n].cpu().numpy()
            assert np.all(np.diff(got) > 0), "table positions must be ascending"
            assert n == 0 or (got[0] >= 0 and got[-1] < F)
            gm = np.zeros(F, bool)
            gm[perm[got]] = True
            _, z_or, _ = oracle.predict(x32.astype(np.float64), e.V, e.U, e.c, e.pdtype, 0.0, e.sV, e.sU)
            band += G.check_active_set(gm, z_or)
            z_gpu = np.empty(F)
            z_gpu[perm] = z.cpu().double().numpy()
            err = float(np.max(np.abs(z_gpu - z_or)))
            assert err <= _z_tol(z_or), f"max |z_gpu - z_oracle| = {err:.3e}"
            # the count and the mask agree with the logits the kernel returned
            assert n == int(np.count_nonzero(z.cpu().numpy() > 0.0))
            G.record_error(f"predict/{name}", max_abs_z=err, band=int(band), active=n)
        assert band <= 3 * max(2, F // 2000)
    finally:
        torch.cuda.synchronize()
        B.pi_ffn_destroy(h)
