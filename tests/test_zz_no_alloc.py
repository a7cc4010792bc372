"""pi_predict_noalloc: the predictor for callers that cannot allocate device
memory where they predict (no handle, scratch in a static device array).

Its outputs must match pi_predict's on the same layer -- a handle loaded with
the identity neuron table, so table positions are original indices -- within
the tolerances of the other predictor tests, on two calls in a row (the second
call runs on the scratch the first one left behind)."""
import numpy as np
import pytest
import torch

from activation_sparse_decode_threshold_b200 import binding as B
from activation_sparse_decode_threshold_b200 import synth

pytestmark = pytest.mark.gpu

Z_BAND = 1e-3


def test_predict_noalloc_matches_pi_predict_on_two_calls():
    cfg = synth.small(synth.CONFIGS["llama7b"], n_layers=1)
    lw = synth.make_layer(cfg, 0, "cuda")
    e = lw.experts[0]
    h = B.pi_ffn_create(1, cfg.d, cfg.F, cfg.rank, act=cfg.act, w_dtype=cfg.wdtype, pred_dtype=cfg.pdtype)
    try:
        B.pi_ffn_load_layer(h, 0, lw.experts, None, None)          # identity table
        F = cfg.F
        for t in (3, 4):                                            # two calls in a row
            r = synth.token_input(cfg, t).cuda()
            x = (r * torch.rsqrt(torch.mean(r * r) + 1e-6)).contiguous()
            idx, cnt, z = (torch.empty(F, dtype=torch.int32, device="cuda"),
                           torch.empty(1, dtype=torch.int32, device="cuda"),
                           torch.empty(F, dtype=torch.float32, device="cuda"))
            B.pi_predict(h, 0, 0, x, idx, cnt, z)
            idx2, cnt2, z2 = (torch.full((F,), -7, dtype=torch.int32, device="cuda"),
                              torch.empty(1, dtype=torch.int32, device="cuda"),
                              torch.empty(F, dtype=torch.float32, device="cuda"))
            B.pi_predict_noalloc(cfg.d, F, cfg.rank, cfg.pdtype, 0.0, e.V, e.U, e.c, x, idx2, cnt2, z2)
            torch.cuda.synchronize()
            assert B.pi_sync(h) == B.PI_OK
            zr, zn = z.cpu().double().numpy(), z2.cpu().double().numpy()
            assert np.max(np.abs(zn - zr)) <= 1e-4 + 1e-5 * np.max(np.abs(zr))
            n_ref, n_new = int(cnt.item()), int(cnt2.item())
            assert n_new >= 0, "the no-allocation predictor gave up on a bounded wait"
            a = set(idx[:n_ref].cpu().numpy().tolist())
            b = set(idx2[:n_new].cpu().numpy().tolist())
            got = idx2[:n_new].cpu().numpy()
            assert np.all(np.diff(got) > 0)
            diff = np.array(sorted(a ^ b), dtype=np.int64)
            assert diff.size == 0 or np.all(np.abs(zr[diff]) < Z_BAND), diff[:8]
            assert abs(n_ref - n_new) <= diff.size
    finally:
        torch.cuda.synchronize()
        B.pi_ffn_destroy(h)


def test_predict_noalloc_rejects_sizes_beyond_its_limits():
    z = torch.empty(8, dtype=torch.float32, device="cuda")
    i = torch.empty(8, dtype=torch.int32, device="cuda")
    with pytest.raises(B.PiError) as ei:
        B.pi_predict_noalloc(16384, 8, 64, "f16", 0.0, z, z, z, z, i, i)
    assert ei.value.status == B.PI_ERR_INVALID_ARG
    with pytest.raises(B.PiError):
        B.pi_predict_noalloc(4096, 10**7, 64, "f16", 0.0, z, z, z, z, i, i)
