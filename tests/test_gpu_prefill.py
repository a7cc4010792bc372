"""GPU parity of the dense tensor-core prefill (pi_dense_ffn_prefill) against
the fp64 oracle's dense prefill layer, through the C ABI.

Small cases cover every activation, the three weight formats the prefill
takes, token counts that leave a ragged last tile (1, 200, 300 tokens), MoE
experts with uneven token counts, and a two-layer stack.  The full-size case
is the 512-token prompt of the 47B MoE shape, checked on sampled tokens."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_decode_threshold_b200 import binding as B
from activation_sparse_decode_threshold_b200 import synth
import gpu_util as G

pytestmark = pytest.mark.gpu

SMALL = {
    "reglu-f16": synth.small(synth.CONFIGS["llama7b"], n_layers=2, d=512, F=1024, rank=64),
    "drelu-bf16": synth.small(synth.CONFIGS["mistral7b"], n_layers=2, d=768, F=1536, rank=64),
    "relu-f16-nongated": synth.small(synth.CONFIGS["falcon40b"], n_layers=2, d=512, F=2048, rank=64),
    "moe-int4-drelu": synth.small(synth.CONFIGS["mixtral47b"], n_layers=2, d=512, F=1024, rank=64,
                                  n_experts=4),
    "reglu-int4": synth.small(synth.CONFIGS["llama7b"], n_layers=2, d=512, F=1024, rank=64,
                              wdtype="int4g32"),
}

# logits closer than this between the 2nd and 3rd expert make the choice of
# expert depend on rounding; such tokens are left out of the element check
ROUTE_MARGIN = 1e-4


@pytest.fixture
def handles():
    hs = []
    yield hs
    torch.cuda.synchronize()
    for h in hs:
        B.pi_ffn_destroy(h)


def _build(cfg, handles, n_layers=None):
    L = n_layers or cfg.n_layers
    h = G.create(cfg, L)
    handles.append(h)
    lws = [synth.make_layer(cfg, l, "cuda") for l in range(L)]
    for l, lw in enumerate(lws):
        G.load(h, l, lw)
    return h, lws


def _prefill(h, R, l0, l1):
    r = R.clone().contiguous()
    B.pi_dense_ffn_prefill(h, l0, l1, r.shape[0], r)
    assert B.pi_sync(h) == B.PI_OK, B.pi_last_error()
    return r


def _routable(res) -> np.ndarray:
    """Tokens whose top-2 choice is clear of rounding."""
    if res.logits is None:
        return np.ones(res.y.shape[0], bool)
    s = np.sort(res.logits, axis=1)[:, ::-1]
    return (s[:, 1] - s[:, 2]) > ROUTE_MARGIN


def _check(y_gpu, res, case=None):
    ok = _routable(res)
    assert ok.mean() > 0.9
    rl, ma = G.check_output(y_gpu[ok].ravel(), res.y[ok].ravel())
    if case:
        G.record_error(case, rel_l2=rl, max_abs=ma)
    return rl, ma


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("T", [1, 200, 300])
def test_prefill_single_layer(handles, name, T):
    cfg = SMALL[name]
    h, lws = _build(cfg, handles, n_layers=1)
    R = synth.prefill_input(cfg, T, "cuda")
    out = _prefill(h, R, 0, 1)
    ex, router = G.oracle_layer(cfg, lws[0])
    Rn = R.double().cpu().numpy()
    res = oracle.prefill_layer(Rn, ex, router)
    y_gpu = out.double().cpu().numpy() - Rn
    assert np.all(np.isfinite(y_gpu))
    _check(y_gpu, res, f"prefill/small/{name}")


def test_prefill_two_layer_stack(handles):
    cfg = SMALL["moe-int4-drelu"]
    h, lws = _build(cfg, handles)
    T = 160
    R = synth.prefill_input(cfg, T, "cuda")
    out = _prefill(h, R, 0, 2)
    mid = _prefill(h, R, 0, 1)
    # layer by layer equals the stack (same kernels, same order: bit-exact)
    assert torch.equal(_prefill(h, mid, 1, 2), out)
    # teacher-forced: each layer against the oracle on the GPU's own input
    R0 = R.double().cpu().numpy()
    R1 = mid.double().cpu().numpy()
    for l, (rin, rout) in enumerate([(R0, R1), (R1, out.double().cpu().numpy())]):
        ex, router = G.oracle_layer(cfg, lws[l])
        res = oracle.prefill_layer(rin, ex, router)
        _check(rout - rin, res)


def test_prefill_is_deterministic(handles):
    cfg = SMALL["moe-int4-drelu"]
    h, _ = _build(cfg, handles, n_layers=1)
    R = synth.prefill_input(cfg, 300, "cuda")
    a = _prefill(h, R, 0, 1)
    b = _prefill(h, R, 0, 1)
    assert torch.equal(a, b)


def test_prefill_token_order_permutes_rows(handles):
    """Rows are independent: permuting the prompt permutes the outputs."""
    cfg = SMALL["reglu-f16"]
    h, _ = _build(cfg, handles, n_layers=1)
    R = synth.prefill_input(cfg, 257, "cuda")
    p = torch.randperm(257, generator=torch.Generator().manual_seed(5)).cuda()
    a = _prefill(h, R, 0, 1)
    b = _prefill(h, R[p], 0, 1)
    assert torch.equal(a[p], b)


def test_prefill_rejects_unsupported_shapes(handles):
    cfg = synth.small(synth.CONFIGS["llama7b"], n_layers=1, d=512, F=1000, rank=64)
    h, _ = _build(cfg, handles)
    R = synth.prefill_input(cfg, 4, "cuda")
    with pytest.raises(B.PiError) as ei:
        B.pi_dense_ffn_prefill(h, 0, 1, 4, R)
    assert ei.value.status == B.PI_ERR_UNSUPPORTED


def _tile_rows(Rn: np.ndarray, router: np.ndarray) -> np.ndarray:
    """Tokens that cover every 128-row tile half of every expert's GEMM rows:
    the first, middle and last list position of each half, the list of an
    expert being its tokens in ascending order (the kernel's sort order)."""
    ex = np.array([oracle.route_top2(oracle.rmsnorm(row), router)[1] for row in Rn])
    rows = set()
    for e in range(router.shape[0]):
        toks = np.nonzero((ex == e).any(axis=1))[0]
        for h0 in range(0, toks.size, 128):
            half = toks[h0:h0 + 128]
            rows.update(int(half[i]) for i in (0, half.size // 2, half.size - 1))
    return np.array(sorted(rows))


def test_prefill_full_size_moe_512_tokens(handles):
    """The 47B MoE shape, INT4 experts, one 512-token prompt through layer 0
    and the last layer; teacher-forced on the GPU's own layer input, each
    layer checked against the oracle on tokens that cover every 128-row tile
    half of every expert (first, middle and last list position of each half,
    so each expert's ragged last tile is covered too)."""
    cfg = synth.CONFIGS["mixtral47b"]
    T = cfg.prefill_tokens
    h = G.create(cfg, 2)
    handles.append(h)
    layers = [0, cfg.n_layers - 1]
    for slot, l in enumerate(layers):
        G.load(h, slot, synth.make_layer(cfg, l, "cuda"))
    R = synth.prefill_input(cfg, T, "cuda")
    mid = _prefill(h, R, 0, 1)
    out = _prefill(h, mid, 1, 2)
    assert torch.isfinite(out).all()
    assert torch.equal(_prefill(h, R, 0, 2), out)      # the stack call is the same arithmetic
    for slot, (rin, rout) in enumerate([(R, mid), (mid, out)]):
        lw = synth.make_layer(cfg, layers[slot], "cuda")
        ex, router = G.oracle_layer(cfg, lw)
        del lw
        Rall = rin.double().cpu().numpy()
        rows = _tile_rows(Rall, router)
        assert rows.size >= 2 * cfg.n_experts
        Rn = Rall[rows]
        res = oracle.prefill_layer(Rn, ex, router)
        y_gpu = rout.double().cpu().numpy()[rows] - Rn
        ok = _routable(res)
        rl, ma = G.check_output(y_gpu[ok].ravel(), res.y[ok].ravel())
        G.record_error("prefill/full/mixtral47b-512tok", rel_l2=rl, max_abs=ma, rows=int(ok.sum()))


def test_prefill_bounded_wait_reports_timeout_and_handle_survives(handles):
    """A prefill whose tensor-core issuer never sees its first stage published
    (PI_DEBUG_STALL_PREFILL) gives up after the handle's wait limit, releases
    its tensor memory and reports PI_ERR_TIMEOUT; the next prefill on the same
    handle is correct."""
    cfg = SMALL["moe-int4-drelu"]
    h, lws = _build(cfg, handles, n_layers=1)
    R = synth.prefill_input(cfg, 200, "cuda")
    B.pi_debug_set(h, B.PI_DEBUG_STALL_PREFILL, 0.05)
    r = R.clone()
    B.pi_dense_ffn_prefill(h, 0, 1, 200, r)
    assert B.pi_sync(h) == B.PI_ERR_TIMEOUT
    B.pi_debug_set(h, 0, 2.0)
    out = _prefill(h, R, 0, 1)
    ex, router = G.oracle_layer(cfg, lws[0])
    Rn = R.double().cpu().numpy()
    res = oracle.prefill_layer(Rn, ex, router)
    _check(out.double().cpu().numpy() - Rn, res)
