"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

Small cases (the oracle finishes in seconds) span several strips and ragged
strip tails; full-size cases run the workloads at their real shapes in the
launch configuration the benchmark uses (one CTA per SM) and check sampled
layers teacher-forced on the GPU's own trace."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_decode_threshold_b200 import binding as B
from activation_sparse_decode_threshold_b200 import synth
import gpu_util as G

pytestmark = pytest.mark.gpu

SMALL = {
    # name: (config, strips)
    "reglu-f16": synth.small(synth.CONFIGS["llama7b"], n_layers=3, d=512, F=1000, rank=64),
    "drelu-bf16": synth.small(synth.CONFIGS["mistral7b"], n_layers=3, d=768, F=2100, rank=128),
    "relu-f16-nongated": synth.small(synth.CONFIGS["falcon40b"], n_layers=2, d=1024, F=4100, rank=256),
    "reglu-f32": synth.small(synth.CONFIGS["relu1"], n_layers=2, d=256, F=333, rank=32),
    "moe-int4-drelu": synth.small(synth.CONFIGS["mixtral47b"], n_layers=2, d=512, F=1024, rank=64,
                                  n_experts=4),
    "fewer-neurons-than-strips": synth.small(synth.CONFIGS["llama7b"], n_layers=2, d=256, F=100,
                                             rank=32),
    # INT4 experts with the speculative kinds (gate|up|down records)
    "reglu-int4": synth.small(synth.CONFIGS["llama7b"], n_layers=2, d=512, F=1200, rank=64,
                              wdtype="int4g32"),
    "relu-int4-nongated": synth.small(synth.CONFIGS["falcon40b"], n_layers=2, d=512, F=1500, rank=64,
                                      wdtype="int4g32"),
    # INT4 at d_model 8192: two x vectors per thread, so every warp's tensor-core
    # gather dots take k-groups from both of its vector ranges
    "relu-int4-d8192": synth.small(synth.CONFIGS["falcon40b"], n_layers=2, d=8192, F=1500, rank=64,
                                   wdtype="int4g32"),
    "moe-int4-drelu-d8192": synth.small(synth.CONFIGS["mixtral47b"], n_layers=2, d=8192, F=1024, rank=64,
                                        n_experts=4),
    # the 8-bit per-row predictor with 16-bit and INT4 weights, dense and MoE
    "reglu-f16-i8pred": synth.small(synth.CONFIGS["llama7b-i8pred"], n_layers=3, d=512, F=1000, rank=128),
    "drelu-bf16-i8pred": synth.small(synth.CONFIGS["mistral7b"], n_layers=2, d=768, F=2100, rank=64,
                                     pdtype="i8row"),
    "moe-int4-i8pred": synth.small(synth.CONFIGS["mixtral47b-i8pred"], n_layers=2, d=512, F=1024, rank=128,
                                   n_experts=4),
}


@pytest.fixture
def handles():
    hs = []
    yield hs
    torch.cuda.synchronize()
    for h in hs:
        B.pi_ffn_destroy(h)


def _build(cfg, handles, n_strips=0, threshold=0.0, use_freq=True, n_layers=None):
    L = n_layers or cfg.n_layers
    h = G.create(cfg, L, n_strips, threshold)
    handles.append(h)
    lws = [synth.make_layer(cfg, l, "cuda") for l in range(L)]
    for l, lw in enumerate(lws):
        G.load(h, l, lw, use_freq)
    return h, lws


# ---------------------------------------------------------------------------
def test_neuron_table_and_strips_match_oracle(handles):
    cfg = SMALL["reglu-f16"]
    h, lws = _build(cfg, handles, n_layers=1)
    off = B.pi_strip_offsets(h)
    S = len(off) - 1
    assert np.array_equal(off, oracle.strip_offsets(cfg.F, S))
    freq32 = G.freq_of(lws[0])[0]
    perm = B.pi_neuron_table(h, 0, 0, cfg.F)
    assert np.array_equal(perm, oracle.neuron_table(cfg.F, S, freq32.astype(np.float64)))


def test_predict_parity_single_layer_fp32(handles):
    """64 tokens of the single-layer fp32 workload: predicted sets and logits."""
    cfg = synth.CONFIGS["relu1"]
    h, lws = _build(cfg, handles)
    ex, _ = G.oracle_layer(cfg, lws[0])
    perm = B.pi_neuron_table(h, 0, 0, cfg.F)
    idx = torch.empty(cfg.F, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, dtype=torch.int32, device="cuda")
    z = torch.empty(cfg.F, dtype=torch.float32, device="cuda")
    band = 0
    for t in range(cfg.n_tokens):
        x32 = oracle.rmsnorm(synth.token_input(cfg, t).double().numpy()).astype(np.float32)
        B.pi_predict(h, 0, 0, torch.from_numpy(x32).cuda(), idx, cnt, z)
        assert B.pi_sync(h) == B.PI_OK
        n = int(cnt.item())
        got = idx[:n].cpu().numpy()
        assert np.all(np.diff(got) > 0), "table positions must be ascending"
        gm = np.zeros(cfg.F, bool)
        gm[perm[got]] = True
        _, z_or, _ = oracle.predict(x32.astype(np.float64), ex[0].V, ex[0].U, ex[0].c, "f32")
        band += G.check_active_set(gm, z_or)
        z_gpu = np.empty(cfg.F)
        z_gpu[perm] = z.cpu().double().numpy()
        assert np.max(np.abs(z_gpu - z_or)) <= 1e-4 + 1e-5 * np.max(np.abs(z_or))
    assert band <= 2


def test_decode_single_layer_fp32_all_tokens(handles):
    cfg = synth.CONFIGS["relu1"]
    h, lws = _build(cfg, handles)
    ex, router = G.oracle_layer(cfg, lws[0])
    perms = G.tables(h, lws[0], 0, cfg.F)
    for t in range(cfg.n_tokens):
        r0 = synth.token_input(cfg, t)
        r1, trace, stats, masks = G.decode_traced(h, cfg, 0, 1, r0)
        assert np.array_equal(trace[0], r0.double().numpy())
        G.check_layer(cfg, ex, router, perms, trace[0], r1, stats[0], masks[0], case="decode/relu1")


@pytest.mark.parametrize("name", sorted(SMALL))
def test_decode_stack_small(handles, name):
    cfg = SMALL[name]
    h, lws = _build(cfg, handles)
    olayers = [G.oracle_layer(cfg, lw) for lw in lws]
    perms = [G.tables(h, lw, l, cfg.F) for l, lw in enumerate(lws)]
    for t in range(4):
        r0 = synth.token_input(cfg, t)
        rL, trace, stats, masks = G.decode_traced(h, cfg, 0, cfg.n_layers, r0)
        outs = list(trace[1:]) + [rL]
        for l in range(cfg.n_layers):
            ex, router = olayers[l]
            G.check_layer(cfg, ex, router, perms[l], trace[l], outs[l], stats[l], masks[l],
                          case=f"decode/small/{name}")


@pytest.mark.parametrize("name", ["drelu-bf16", "moe-int4-drelu"])
def test_decode_is_deterministic_and_splits_agree(handles, name):
    """The same input gives the same bits on every call, whatever ran before
    on the handle (the fixed-point totals and input buffers are reset by the
    kernel itself), and splitting the layer range into one call per layer
    gives the same bits as one call."""
    cfg = SMALL[name]
    h, _ = _build(cfg, handles)
    r0 = synth.token_input(cfg, 5).cuda()
    other = synth.token_input(cfg, 6).cuda() * 3.0
    outs = []
    for _ in range(2):
        r = r0.clone()
        B.pi_sparse_ffn_decode(h, 0, cfg.n_layers, r)
        outs.append(r.clone())
        # another token through part of the stack between the two calls
        o = other.clone()
        B.pi_sparse_ffn_decode(h, 1, cfg.n_layers, o)
    r = r0.clone()
    for l in range(cfg.n_layers):
        B.pi_sparse_ffn_decode(h, l, l + 1, r)
    outs.append(r)
    assert B.pi_sync(h) == B.PI_OK
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(outs[0], outs[2])


def test_host_buffer_entry_point_matches_device_call(handles):
    cfg = SMALL["reglu-f16"]
    h, _ = _build(cfg, handles)
    r0 = synth.token_input(cfg, 1)
    rin = r0.clone().pin_memory()
    rout = torch.empty_like(rin).pin_memory()
    B.pi_sparse_ffn_decode_host(h, 0, cfg.n_layers, rin, rout)
    rd = r0.clone().cuda()
    B.pi_sparse_ffn_decode(h, 0, cfg.n_layers, rd)
    assert B.pi_sync(h) == B.PI_OK
    assert torch.equal(rout, rd.cpu())


def test_threshold_extremes_empty_and_dense(handles):
    cfg = SMALL["reglu-f16"]
    lw = synth.make_layer(cfg, 0, "cuda")
    ex, _ = G.oracle_layer(cfg, lw)
    r0 = synth.token_input(cfg, 2)
    # nothing predicted active: the layer adds exactly zero
    h = G.create(cfg, 1, threshold=1e30)
    handles.append(h)
    G.load(h, 0, lw)
    r1, _, stats, _ = G.decode_traced(h, cfg, 0, 1, r0)
    assert stats[0][0] == 0 and np.array_equal(r1, r0.double().numpy())
    # everything active: the dense FFN
    h2 = G.create(cfg, 1, threshold=-1e30)
    handles.append(h2)
    G.load(h2, 0, lw)
    r1, _, stats, _ = G.decode_traced(h2, cfg, 0, 1, r0)
    assert stats[0][0] == cfg.F
    x = oracle.rmsnorm(r0.double().numpy())
    _, y = oracle.ffn_masked(ex[0], x)
    G.check_output(r1 - r0.double().numpy(), y)


def test_identity_table_gives_same_result_within_rounding(handles):
    cfg = SMALL["reglu-f16"]
    h1, _ = _build(cfg, handles, use_freq=True, n_layers=1)
    h2, _ = _build(cfg, handles, use_freq=False, n_layers=1)
    assert np.array_equal(B.pi_neuron_table(h2, 0, 0, cfg.F), np.arange(cfg.F))
    r0 = synth.token_input(cfg, 3)
    a, _, sa, _ = G.decode_traced(h1, cfg, 0, 1, r0)
    b, _, sb, _ = G.decode_traced(h2, cfg, 0, 1, r0)
    assert abs(int(sa[0][0]) - int(sb[0][0])) <= 1
    G.check_output(a - r0.double().numpy(), b - r0.double().numpy())


@pytest.mark.parametrize("flag", ["PI_DEBUG_STALL_BARRIER", "PI_DEBUG_STALL_T_POLL"])
def test_bounded_wait_reports_timeout_and_context_survives(handles, flag):
    # a grid barrier that misses one arrival, or a poll of the rows of t for a
    # tag that no CTA writes: the bounded wait runs out, the kernel returns
    cfg = SMALL["reglu-f16"]
    h, _ = _build(cfg, handles, n_layers=1)
    r = synth.token_input(cfg, 0).cuda()
    B.pi_debug_set(h, getattr(B, flag), 0.05)
    B.pi_sparse_ffn_decode(h, 0, 1, r.clone())
    assert B.pi_sync(h) == B.PI_ERR_TIMEOUT
    B.pi_debug_set(h, 0, 2.0)
    r2 = r.clone()
    B.pi_sparse_ffn_decode(h, 0, 1, r2)
    assert B.pi_sync(h) == B.PI_OK
    assert torch.isfinite(r2).all() and not torch.equal(r2, r)


# ---------------------------------------------------------------------------
# Full-size workloads (launch configuration of the benchmark: one CTA per SM)
# ---------------------------------------------------------------------------
# (workload, target active fraction: None = the workload's own; the mistral7b
# sweep points are the ones the benchmark reports)
FULL = [("llama7b", None), ("mistral7b", None), ("falcon40b", None), ("mixtral47b", None),
        ("mistral7b", 0.5), ("mistral7b", 0.2), ("mistral7b", 0.05),
        ("llama7b-i8pred", None), ("mixtral47b-i8pred", None)]


@pytest.mark.parametrize("name,active", FULL, ids=[f"{n}@{a}" if a else n for n, a in FULL])
def test_full_size_sampled_layers(handles, name, active):
    cfg = synth.CONFIGS[name]
    h = G.create(cfg)
    handles.append(h)
    for l in range(cfg.n_layers):
        G.load(h, l, synth.make_layer(cfg, l, "cuda", active))
    torch.cuda.empty_cache()
    target = cfg.mean_active if active is None else active
    sample = sorted({0, cfg.n_layers // 2, cfg.n_layers - 1})
    for t in (0, 1):
        r0 = synth.token_input(cfg, t)
        rL, trace, stats, masks = G.decode_traced(h, cfg, 0, cfg.n_layers, r0)
        assert np.all(np.isfinite(rL))
        outs = list(trace[1:]) + [rL]
        for l in sample:
            lw = synth.make_layer(cfg, l, "cuda", active)
            ex, router = G.oracle_layer(cfg, lw)
            perms = G.tables(h, lw, l, cfg.F)
            del lw
            G.check_layer(cfg, ex, router, perms, trace[l], outs[l], stats[l], masks[l],
                          case=f"decode/full/{name}@{target}")
        frac = stats[:, 0].mean() / (cfg.F * cfg.top_k)
        assert abs(frac - target) < 0.05, f"predicted active fraction {frac:.3f}"


@pytest.mark.parametrize("scale", [1e-3, 1e3])
def test_residual_scale_matches_oracle(handles, scale):
    """RMSNorm makes each layer's input scale-free: residuals scaled by 1e-3
    or 1e3 still match the oracle layer by layer (every CTA forms the sum of
    squares of the whole input in fp32, t comes from x, and y's fixed-point
    total depends on x alone).  Far larger residuals keep the right layer
    inputs too, but the fp32 residual's own rounding then swamps a layer's
    increment y."""
    cfg = SMALL["reglu-f16"]
    h, lws = _build(cfg, handles)
    olayers = [G.oracle_layer(cfg, lw) for lw in lws]
    perms = [G.tables(h, lw, l, cfg.F) for l, lw in enumerate(lws)]
    r0 = synth.token_input(cfg, 9) * scale
    rL, trace, stats, masks = G.decode_traced(h, cfg, 0, cfg.n_layers, r0)
    outs = list(trace[1:]) + [rL]
    for l in range(cfg.n_layers):
        ex, router = olayers[l]
        x = oracle.rmsnorm(trace[l])
        _, z, _ = oracle.predict(x, ex[0].V, ex[0].U, ex[0].c, ex[0].pdtype)
        gm = G.masks_to_original(masks[l][0], perms[l][0], cfg.F)
        band = G.check_active_set(gm, z)
        _, y = oracle.ffn_masked(ex[0], x, gm.astype(np.uint8))
        rl, ma = G.check_output(outs[l] - trace[l], y)
        G.record_error(f"decode/scale{scale:g}", rel_l2=rl, max_abs=ma, band=band)


def test_residual_out_of_range_reports_device_check(handles):
    """A residual so large (|r| ~ 1e20) that its sum of squares leaves the
    fp32 range is reported as a failed device check, not returned as a
    silently wrong answer; the handle stays usable."""
    cfg = SMALL["reglu-f16"]
    h, _ = _build(cfg, handles, n_layers=1)
    r0 = (synth.token_input(cfg, 9) * 1e20).cuda()
    r = r0.clone()
    B.pi_sparse_ffn_decode(h, 0, 1, r)
    assert B.pi_sync(h) == B.PI_ERR_DEVICE_CHECK
    r2 = synth.token_input(cfg, 9).cuda()
    B.pi_sparse_ffn_decode(h, 0, 1, r2)
    assert B.pi_sync(h) == B.PI_OK
    assert torch.isfinite(r2).all()


# ---------------------------------------------------------------------------
# VRAM budget: cold records in pinned host memory
# ---------------------------------------------------------------------------
BUDGET = {
    "reglu-f16": (SMALL["reglu-f16"], 2),
    "drelu-bf16": (SMALL["drelu-bf16"], 3),
    "moe-int4-drelu": (SMALL["moe-int4-drelu"], 1),
    "relu-f16-nongated": (SMALL["relu-f16-nongated"], 5),
}


@pytest.mark.parametrize("name", sorted(BUDGET))
def test_vram_budget_gives_the_same_bits_and_matches_oracle(handles, name):
    """Most records live in pinned host memory (only the hottest few of each
    strip stay in HBM); decode gives the same bits as the all-HBM handle and
    matches the oracle layer by layer."""
    cfg, hot = BUDGET[name]
    h0, lws = _build(cfg, handles)
    h1 = G.create(cfg)
    handles.append(h1)
    B.pi_ffn_set_hot_neurons(h1, hot)
    for l, lw in enumerate(lws):
        G.load(h1, l, lw)
    olayers = [G.oracle_layer(cfg, lw) for lw in lws]
    perms = [G.tables(h1, lw, l, cfg.F) for l, lw in enumerate(lws)]
    for t in range(3):
        r0 = synth.token_input(cfg, t)
        a, trace, stats, masks = G.decode_traced(h1, cfg, 0, cfg.n_layers, r0)
        b, _, _, _ = G.decode_traced(h0, cfg, 0, cfg.n_layers, r0)
        assert np.array_equal(a, b)
        outs = list(trace[1:]) + [a]
        for l in range(cfg.n_layers):
            ex, router = olayers[l]
            G.check_layer(cfg, ex, router, perms[l], trace[l], outs[l], stats[l], masks[l],
                          case=f"decode/vram-budget/{name}")


def test_vram_budget_rejections(handles):
    cfg = SMALL["reglu-f16"]
    h, _ = _build(cfg, handles, n_layers=1)
    with pytest.raises(B.PiError):             # after a layer is loaded
        B.pi_ffn_set_hot_neurons(h, 1)
    h2 = G.create(cfg, 1)
    handles.append(h2)
    with pytest.raises(B.PiError):             # more than the smallest strip
        B.pi_ffn_set_hot_neurons(h2, cfg.F)
    B.pi_ffn_set_hot_neurons(h2, 1)
    G.load(h2, 0, synth.make_layer(cfg, 0, "cuda"))
    R = synth.prefill_input(cfg, 4, "cuda")
    with pytest.raises(B.PiError) as ei:
        B.pi_dense_ffn_prefill(h2, 0, 1, 4, R)
    assert ei.value.status == B.PI_ERR_UNSUPPORTED


def test_i8_predictor_rank_must_be_a_multiple_of_32():
    # the 8-bit predictor's integer logits take 32 columns of U per step
    with pytest.raises(B.PiError) as ei:
        B.pi_ffn_create(1, 512, 1000, 48, act="reglu", w_dtype="f16", pred_dtype="i8row")
    assert ei.value.status == B.PI_ERR_INVALID_ARG
    h = B.pi_ffn_create(1, 512, 1000, 64, act="reglu", w_dtype="f16", pred_dtype="i8row")
    B.pi_ffn_destroy(h)
