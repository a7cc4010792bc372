"""GPU parity of the small-batch decode (pi_sparse_ffn_decode_batch) against the
fp64 oracle, through the C ABI.

Each token of a batch is checked on its own, teacher-forced on the GPU's own
layer input from the trace: its predicted set (the token's mask bits) must
equal the oracle's outside the |z| < 1e-3 band, and its layer output must be
the oracle's masked FFN of that set within the parity bar.  The per-layer
union statistics must agree with the token masks.  Small cases span several
strips, ragged strip tails, batches of 1, 3, 8 and 11 tokens (one to three
launches: 8 tokens per launch with F16 weights, 4 with BF16);
full-size cases run the Llama-2-7B and TurboSparse-Mistral-7B shapes."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_decode_threshold_b200 import binding as B
from activation_sparse_decode_threshold_b200 import synth
import gpu_util as G

pytestmark = pytest.mark.gpu

SMALL = {
    "reglu-f16": synth.small(synth.CONFIGS["llama7b"], n_layers=3, d=512, F=1000, rank=64),
    "drelu-bf16": synth.small(synth.CONFIGS["mistral7b"], n_layers=2, d=768, F=2100, rank=128),
    "relu-f16-nongated": synth.small(synth.CONFIGS["falcon40b"], n_layers=2, d=1024, F=4100, rank=256),
    "fewer-neurons-than-strips": synth.small(synth.CONFIGS["llama7b"], n_layers=2, d=256, F=100, rank=32),
}


@pytest.fixture
def handles():
    hs = []
    yield hs
    torch.cuda.synchronize()
    for h in hs:
        B.pi_ffn_destroy(h)


def batch_traced(h, cfg, l0, l1, R0: torch.Tensor):
    nb, nl = R0.shape[0], l1 - l0
    resid = R0.clone().cuda().contiguous()
    trace = torch.empty((nl, nb, cfg.d), device="cuda", dtype=torch.float32)
    stats = torch.empty((nl, 4), device="cuda", dtype=torch.int32)
    words = (cfg.F + 31) // 32
    masks = torch.empty((nl, nb, words), device="cuda", dtype=torch.int32)
    B.pi_sparse_ffn_decode_batch(h, l0, l1, resid, trace, stats, masks)
    assert B.pi_sync(h) == B.PI_OK, B.pi_last_error()
    return (resid.cpu().double().numpy(), trace.cpu().double().numpy(), stats.cpu().numpy(),
            masks.cpu().numpy().view(np.uint32))


def check_batch_layer(cfg, experts, perm, r_in, r_out, stats_row, mask_rows, case, groups=1):
    """Every token of one layer (teacher-forced): its set and its output."""
    nb = r_in.shape[0]
    union_bits = np.zeros(cfg.F, bool)
    tot = 0
    for b in range(nb):
        x = oracle.rmsnorm(r_in[b])
        e = experts[0]
        _, z, _ = oracle.predict(x, e.V, e.U, e.c, e.pdtype)
        gm = G.masks_to_original(mask_rows[b], perm, cfg.F)
        band = G.check_active_set(gm, z)
        _, y = oracle.ffn_masked(e, x, gm.astype(np.uint8))
        rl, ma = G.check_output(r_out[b] - r_in[b], y)
        G.record_error(case, rel_l2=rl, max_abs=ma, band=band)
        union_bits |= gm
        tot += int(gm.sum())
    assert int(stats_row[1]) == tot
    if groups == 1:
        assert int(stats_row[0]) == int(union_bits.sum())
    assert int(stats_row[0]) <= tot and int(stats_row[2]) <= int(stats_row[0])


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("nb", [1, 3, 8, 11])
def test_batch_decode_small(handles, name, nb):
    cfg = SMALL[name]
    h = G.create(cfg)
    handles.append(h)
    lws = [synth.make_layer(cfg, l, "cuda") for l in range(cfg.n_layers)]
    for l, lw in enumerate(lws):
        G.load(h, l, lw)
    olayers = [G.oracle_layer(cfg, lw) for lw in lws]
    perms = [B.pi_neuron_table(h, l, 0, cfg.F) for l in range(cfg.n_layers)]
    R0 = synth.token_inputs(cfg, nb, "cpu", 7)
    rL, trace, stats, masks = batch_traced(h, cfg, 0, cfg.n_layers, R0)
    assert np.array_equal(trace[0], R0.double().numpy())
    outs = list(trace[1:]) + [rL]
    for l in range(cfg.n_layers):
        ex, _ = olayers[l]
        tpl = 4 if cfg.wdtype == "bf16" else 8     # tokens per launch
        check_batch_layer(cfg, ex, perms[l], trace[l], outs[l], stats[l], masks[l],
                          f"batch/small/{name}", groups=(nb + tpl - 1) // tpl)


def test_batch_decode_is_deterministic_and_rows_independent(handles):
    """Same inputs give the same bits; a token's result does not depend on
    which other tokens share its batch beyond rounding of the union (its own
    set and output are checked against the oracle either way)."""
    cfg = SMALL["reglu-f16"]
    h = G.create(cfg)
    handles.append(h)
    for l in range(cfg.n_layers):
        G.load(h, l, synth.make_layer(cfg, l, "cuda"))
    R0 = synth.token_inputs(cfg, 6, "cuda", 40)
    a = R0.clone()
    b = R0.clone()
    B.pi_sparse_ffn_decode_batch(h, 0, cfg.n_layers, a)
    B.pi_sparse_ffn_decode_batch(h, 0, cfg.n_layers, b)
    assert B.pi_sync(h) == B.PI_OK
    assert torch.equal(a, b)
    # layer by layer equals the stack
    c = R0.clone()
    for l in range(cfg.n_layers):
        B.pi_sparse_ffn_decode_batch(h, l, l + 1, c)
    assert B.pi_sync(h) == B.PI_OK
    assert torch.equal(a, c)


def test_batch_decode_rejects_unsupported(handles):
    cfg = synth.small(synth.CONFIGS["mixtral47b"], n_layers=1, d=512, F=1024, rank=64, n_experts=4)
    h = G.create(cfg, 1)
    handles.append(h)
    G.load(h, 0, synth.make_layer(cfg, 0, "cuda"))
    r = torch.zeros((2, cfg.d), device="cuda")
    with pytest.raises(B.PiError) as ei:
        B.pi_sparse_ffn_decode_batch(h, 0, 1, r)
    assert ei.value.status == B.PI_ERR_UNSUPPORTED
    cfg2 = SMALL["reglu-f16"]
    h2 = G.create(cfg2, 1)
    handles.append(h2)
    G.load(h2, 0, synth.make_layer(cfg2, 0, "cuda"))
    with pytest.raises(B.PiError) as ei:
        B.pi_sparse_ffn_decode_batch(h2, 0, 1, torch.zeros((33, cfg2.d), device="cuda"))
    assert ei.value.status == B.PI_ERR_INVALID_ARG


FULL = [("llama7b", 4), ("llama7b", 16), ("mistral7b", 8)]


@pytest.mark.parametrize("name,nb", FULL, ids=[f"{n}-batch{b}" for n, b in FULL])
def test_batch_decode_full_size_sampled_layers(handles, name, nb):
    cfg = synth.CONFIGS[name]
    h = G.create(cfg)
    handles.append(h)
    for l in range(cfg.n_layers):
        G.load(h, l, synth.make_layer(cfg, l, "cuda"))
    torch.cuda.empty_cache()
    R0 = synth.token_inputs(cfg, nb, "cpu", 100)
    rL, trace, stats, masks = batch_traced(h, cfg, 0, cfg.n_layers, R0)
    assert np.all(np.isfinite(rL))
    outs = list(trace[1:]) + [rL]
    for l in sorted({0, cfg.n_layers // 2, cfg.n_layers - 1}):
        lw = synth.make_layer(cfg, l, "cuda")
        ex, _ = G.oracle_layer(cfg, lw)
        del lw
        perm = B.pi_neuron_table(h, l, 0, cfg.F)
        sel = list(range(nb)) if nb <= 8 else [0, 7, 8, nb - 1]
        sub_stats = stats[l].copy()
        if len(sel) < nb:
            # only a sample of the tokens is checked: the union figures of the
            # full batch are checked for consistency alone
            sub_stats[1] = sum(int(G.masks_to_original(masks[l][b], perm, cfg.F).sum()) for b in sel)
            sub_stats[0] = 0
            sub_stats[2] = 0
        check_batch_layer(cfg, ex, perm, trace[l][sel], outs[l][sel], sub_stats, masks[l][sel],
                          f"batch/full/{name}-batch{nb}", groups=2)
