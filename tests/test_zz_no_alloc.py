"""pi_predict_noalloc: the predictor for callers that cannot allocate device
memory where they predict (a serving loop whose device memory is committed at
start-up, a runtime that owns the allocator, code without a handle).  Its
scratch is one static device array shared by every call.

Each case runs two calls in a row (the second runs on the scratch the first
left behind) and checks them against the fp64 oracle's predictor on the same
stored weights: logits element by element, and the active set exactly except
neurons whose oracle logit lies within 1e-3 of the threshold.  The cases cover
every predictor format, both d_model classes of the kernel, the rank limits
(512 for F32, 1024 for 16-bit), fewer neurons than SMs (strips left empty) and
non-zero thresholds.  This file is collected last, so a failure here comes
after every other test has run."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_decode_threshold_b200 import binding as B
from activation_sparse_decode_threshold_b200 import synth

pytestmark = pytest.mark.gpu

Z_BAND = 1e-3

CASES = [
    # (predictor format, d_model, d_ff, rank, threshold)
    ("f32", 256, 1000, 32, 0.0),
    ("f32", 4096, 700, 512, 0.03),
    ("f16", 4096, 11008, 1024, 0.0),     # the Llama-2-7B layer shape
    ("f16", 8192, 100, 64, 0.05),        # fewer neurons than SMs
    ("bf16", 256, 3000, 1024, 0.0),
    ("bf16", 8192, 2000, 64, -0.02),
]


def _weights(pdtype: str, d: int, F: int, r: int):
    cfg = synth.small(synth.CONFIGS["llama7b"], n_layers=1, d=d, F=F, rank=r, pdtype=pdtype,
                      wdtype=pdtype)
    e = synth.make_expert(cfg, 0, 0, "cuda")
    return e.V.contiguous(), e.U.contiguous(), e.c.contiguous()


def _z_tol(z_ref: np.ndarray) -> float:
    return 1e-4 + 2e-5 * float(np.max(np.abs(z_ref)))


@pytest.mark.parametrize("pdtype,d,F,r,thr", CASES, ids=[f"{c[0]}-d{c[1]}-F{c[2]}-r{c[3]}-thr{c[4]}"
                                                          for c in CASES])
def test_predict_noalloc_matches_oracle_on_two_calls(pdtype, d, F, r, thr):
    V, U, c = _weights(pdtype, d, F, r)
    Vn, Un, cn = synth.to_numpy(V), synth.to_numpy(U), synth.to_numpy(c)
    for t in (3, 4):                                                # two calls in a row
        rr = synth.token_input(synth.small(synth.CONFIGS["llama7b"], d=d), t).double().numpy()
        x32 = oracle.rmsnorm(rr).astype(np.float32)
        x = torch.from_numpy(x32).cuda()
        idx = torch.full((F,), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((1,), -9, dtype=torch.int32, device="cuda")
        z = torch.empty(F, dtype=torch.float32, device="cuda")
        B.pi_predict_noalloc(d, F, r, pdtype, thr, V, U, c, x, idx, cnt, z)
        torch.cuda.synchronize()
        n = int(cnt.item())
        assert n >= 0, "the no-allocation predictor gave up on a bounded wait"
        _, z_or, m_or = oracle.predict(x32.astype(np.float64), Vn, Un, cn, pdtype, thr)
        zg = z.cpu().double().numpy()
        err = float(np.max(np.abs(zg - z_or)))
        assert err <= _z_tol(z_or), f"max |z - z_oracle| = {err:.3e}"
        got = idx[:n].cpu().numpy()
        assert np.all(np.diff(got) > 0) and (n == 0 or (got[0] >= 0 and got[-1] < F))
        gm = np.zeros(F, bool)
        gm[got] = True
        diff = np.nonzero(gm != m_or.astype(bool))[0]
        assert np.all(np.abs(z_or[diff] - thr) < Z_BAND), diff[:8]
        # the list is exactly the set of the returned logits above the threshold
        assert np.array_equal(np.nonzero(z.cpu().numpy() > np.float32(thr))[0], got)


def test_predict_noalloc_rejects_sizes_beyond_its_limits():
    z = torch.empty(8, dtype=torch.float32, device="cuda")
    i = torch.empty(8, dtype=torch.int32, device="cuda")
    with pytest.raises(B.PiError) as ei:
        B.pi_predict_noalloc(16384, 8, 64, "f16", 0.0, z, z, z, z, i, i)
    assert ei.value.status == B.PI_ERR_INVALID_ARG
    with pytest.raises(B.PiError):
        B.pi_predict_noalloc(4096, 10**7, 64, "f16", 0.0, z, z, z, z, i, i)
    with pytest.raises(B.PiError):
        B.pi_predict_noalloc(4096, 1000, 2048, "f16", 0.0, z, z, z, z, i, i)
