"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test checks the oracle against what the pages or the mathematics fix:
hand-derived fixtures under tests/golden/ (each cites its page and section),
closed forms, brute force on 8-neuron layers, IEEE bit patterns, and special
cases that reduce to an independent numpy restatement.  A plausible mistake in
the oracle (a dropped bias, a flipped sign, a transposed W_down, a wrong nibble
order, a mis-ranked tie, a wrong activation) fails at least one of them.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def f32(a):
    return np.ascontiguousarray(np.asarray(a, np.float32))


def expert_from(oracle, act, wg, wu, wd_dF, c, U=None, V=None, wdtype="f32", pdtype="f32"):
    """Float-format expert; predictor defaults to the exact one (V = I, U = W_gate)."""
    wg = np.asarray(wg)
    d = wg.shape[1]
    if V is None:
        V = np.eye(d)
        U = wg
    return oracle.Expert(act=act, wdtype=wdtype, pdtype=pdtype, w_gate=f32(wg),
                         w_up=None if wu is None else f32(wu), w_down=f32(wd_dF),
                         c=f32(c), U=f32(U), V=f32(V))


# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------
def test_float_format_bit_patterns(oracle_mod):
    g = gold("float_formats.json")
    for hx, v in g["f16"]:
        got = oracle_mod.half_to_double(int(hx, 16))
        assert got == v and np.signbit(got) == np.signbit(v), hx
    for hx, v in g["bf16"]:
        assert oracle_mod.bf16_to_double(int(hx, 16)) == v, hx


def test_f16_decoder_matches_numpy_on_all_finite_patterns(oracle_mod):
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    vals = bits.astype(np.uint16).view(np.float16).astype(np.float64)
    fin = np.isfinite(vals)
    m = oracle_mod.load_matrix("f16", bits.astype(np.uint16).view(np.float16)[fin][None, :],
                               None, 1, int(fin.sum()))[0]
    assert np.array_equal(m, vals[fin])


def test_bf16_decoder_matches_torch(oracle_mod):
    rng = np.random.default_rng(0)
    x = torch.from_numpy(rng.standard_normal(4096).astype(np.float32) * 10).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    m = oracle_mod.load_matrix("bf16", bits[None, :], None, 1, 4096)[0]
    assert np.array_equal(m, x.double().numpy())


def test_int4_hand_packed_fixture(oracle_mod):
    g = gold("int4_g32.json")
    q = np.frombuffer(bytes.fromhex(g["bytes_hex"]), np.uint8)
    s = np.array([int(h, 16) for h in g["scales_f16_hex"]], np.uint16).view(np.float16)
    out = oracle_mod.dequant_int4_g32(q, s, g["n"])
    assert np.array_equal(out, np.array(g["expected"], np.float64))


def test_int4_on_grid_weights_round_trip_through_writer(oracle_mod):
    """Weights already on the INT4 grid (w = s*q, s an fp16 value, |q| <= 7 with
    a +-7 in every group) survive the model writer and the oracle's reader."""
    from activation_sparse_decode_threshold_b200.synth import quantize_int4_g32
    rng = np.random.default_rng(1)
    rows, n = 6, 128
    s = rng.uniform(0.01, 2.0, (rows, n // 32)).astype(np.float16).astype(np.float64)
    q = rng.integers(-7, 8, (rows, n // 32, 32))
    q[:, :, 5] = 7
    w = (q * s[:, :, None]).reshape(rows, n)
    qb, sb = quantize_int4_g32(torch.from_numpy(w))
    back = oracle_mod.load_matrix("int4g32", qb.numpy(), sb.numpy(), rows, n)
    assert np.array_equal(back, w)


# ---------------------------------------------------------------------------
# RMSNorm closed forms
# ---------------------------------------------------------------------------
def test_rmsnorm_closed_form(oracle_mod):
    x = oracle_mod.rmsnorm(np.array([3.0, 4.0]), 1e-6)
    assert np.allclose(x, np.array([3.0, 4.0]) / np.sqrt(12.5 + 1e-6), rtol=0, atol=1e-15)
    r = np.random.default_rng(2).standard_normal(4096) * 7.0
    x = oracle_mod.rmsnorm(r, 1e-6)
    m = np.mean(r * r)
    assert abs(np.mean(x * x) - m / (m + 1e-6)) < 1e-13
    assert np.all(np.sign(x) == np.sign(r))


# ---------------------------------------------------------------------------
# Activations, bias sign, zero contribution
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("act", ["relu", "reglu", "drelu"])
def test_activation_fixture(oracle_mod, act):
    g = gold("activations.json")
    gv, uv = g["g"], g["u"]
    F = len(gv)
    wg = np.array(gv, np.float64)[:, None]
    wu = None if act == "relu" else np.array(uv, np.float64)[:, None]
    e = expert_from(oracle_mod, act, wg, wu, np.ones((1, F)), np.zeros(F))
    h, y = oracle_mod.ffn_masked(e, np.array([1.0]))
    assert np.array_equal(h, np.array(g["expected_h"][act], np.float64))
    assert y[0] == g["expected_y"][act]


@pytest.mark.parametrize("act", ["relu", "reglu", "drelu"])
def test_inactive_neurons_contribute_exact_zero(oracle_mod, act):
    """PowerInfer-2 (citnews), 'Dynamic neuron cache': neurons that are not
    activated do not affect the output.  h_i is exactly zero (+0, or -0 for
    ReGLU when u_i < 0) whenever g_i <= 0 (or u_i <= 0 under dReLU)."""
    rng = np.random.default_rng(3)
    d, F = 16, 64
    wg, wu = rng.standard_normal((F, d)), rng.standard_normal((F, d))
    c = rng.standard_normal(F)
    x = rng.standard_normal(d)
    e = expert_from(oracle_mod, act, wg, None if act == "relu" else wu, rng.standard_normal((d, F)), c)
    h, _ = oracle_mod.ffn_masked(e, x)
    g = f32(wg).astype(np.float64) @ x - f32(c).astype(np.float64)
    u = f32(wu).astype(np.float64) @ x
    off = g <= 0
    if act == "drelu":
        off |= u <= 0
    assert np.all(h[off] == 0.0)
    assert np.all(h[~off] != 0.0)


def test_bias_enters_with_minus_sign(oracle_mod):
    e = expert_from(oracle_mod, "relu", [[1.0]], None, [[1.0]], [0.25])
    h, y = oracle_mod.ffn_masked(e, np.array([1.0]))
    assert h[0] == 0.75 and y[0] == 0.75


# ---------------------------------------------------------------------------
# Fig. 8 worked example and merge
# ---------------------------------------------------------------------------
def test_fig8_predict_and_merge(oracle_mod):
    g = gold("fig8_merge.json")
    x = np.array(g["x"], np.float64)
    wd = np.array(g["w_down_columns"], np.float64).T        # d x F
    e = expert_from(oracle_mod, "reglu", g["w_gate"], g["w_up"], wd, g["c"])
    _, z, mask = oracle_mod.predict(x, e.V, e.U, e.c, "f32")
    assert sorted(np.nonzero(mask)[0].tolist()) == g["predicted"]
    assert 7 in g["hot"] and not mask[7]                      # hot-labelled, not firing
    h, y = oracle_mod.ffn_masked(e, x, mask)
    assert np.array_equal(h, np.array(g["expected_h"], np.float64))
    assert np.array_equal(y, np.array(g["expected_y"], np.float64))

    def part(ids):
        m = np.zeros(8, np.uint8)
        m[ids] = 1
        return oracle_mod.ffn_masked(e, x, m)[1]
    gpu = part([i for i in g["predicted"] if i in g["hot"]])   # {3, 5}
    cpu = part([i for i in g["predicted"] if i not in g["hot"]])  # {4}
    assert np.array_equal(gpu, np.array(g["expected_gpu_part"], np.float64))
    assert np.array_equal(cpu, np.array(g["expected_cpu_part"], np.float64))
    assert np.array_equal(gpu + cpu, y)


# ---------------------------------------------------------------------------
# Brute force over all 256 masks of 8-neuron layers
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("act", ["relu", "reglu", "drelu"])
def test_brute_force_all_masks(oracle_mod, act):
    rng = np.random.default_rng(5)
    d, F = 4, 8
    wg = rng.integers(-3, 4, (F, d)).astype(np.float64)
    wu = rng.integers(-3, 4, (F, d)).astype(np.float64)
    wd = rng.integers(-3, 4, (d, F)).astype(np.float64)
    c = rng.integers(-2, 3, F).astype(np.float64)
    x = rng.integers(-2, 3, d).astype(np.float64)
    e = expert_from(oracle_mod, act, wg, None if act == "relu" else wu, wd, c)
    h_dense, y_dense = oracle_mod.ffn_masked(e, x)
    truth = set(np.nonzero(h_dense)[0].tolist())
    assert 0 < len(truth) < F
    for bits in itertools.product([0, 1], repeat=F):
        m = np.array(bits, np.uint8)
        h, y = oracle_mod.ffn_masked(e, x, m)
        sel = set(np.nonzero(m)[0].tolist())
        assert np.array_equal(h, np.where(m == 1, h_dense, 0.0))
        if truth <= sel:
            assert np.array_equal(y, y_dense)
        else:
            missing = sorted(truth - sel)
            assert np.array_equal(y_dense - y, sum(h_dense[k] * wd[:, k] for k in missing))


def test_ground_truth_mask_equals_dense_bit_exact(oracle_mod):
    rng = np.random.default_rng(6)
    d, F = 64, 512
    wg, wu, wd = rng.standard_normal((F, d)), rng.standard_normal((F, d)), rng.standard_normal((d, F))
    c = rng.standard_normal(F) + 1.0
    x = rng.standard_normal(d)
    for act in ("relu", "reglu", "drelu"):
        e = expert_from(oracle_mod, act, wg, None if act == "relu" else wu, wd, c)
        h, y = oracle_mod.ffn_masked(e, x)
        h2, y2 = oracle_mod.ffn_masked(e, x, (h != 0).astype(np.uint8))
        assert np.array_equal(y, y2) and np.array_equal(h, h2)


# ---------------------------------------------------------------------------
# Special cases that reduce to an independent dense restatement (numpy)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("wdtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("act", ["relu", "reglu", "drelu"])
def test_dense_ffn_matches_numpy_gemv_chain(oracle_mod, act, wdtype):
    rng = np.random.default_rng(7)
    d, F = 96, 320
    wg = torch.from_numpy(rng.standard_normal((F, d)).astype(np.float32))
    wu = torch.from_numpy(rng.standard_normal((F, d)).astype(np.float32))
    wd = torch.from_numpy(rng.standard_normal((d, F)).astype(np.float32))
    c = rng.standard_normal(F).astype(np.float32)
    x = rng.standard_normal(d)
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[wdtype]
    from activation_sparse_decode_threshold_b200.synth import to_numpy
    W = [w.to(tdt) for w in (wg, wu, wd)]
    e = oracle_mod.Expert(act=act, wdtype=wdtype, pdtype="f32", w_gate=to_numpy(W[0]),
                          w_up=None if act == "relu" else to_numpy(W[1]), w_down=to_numpy(W[2]),
                          c=c, U=np.zeros((F, 1), np.float32), V=np.zeros((1, d), np.float32))
    h, y = oracle_mod.ffn_masked(e, x)
    Wg, Wu, Wd = (w.double().numpy() for w in W)
    g = Wg @ x - c.astype(np.float64)
    u = Wu @ x
    ref_h = {"relu": np.maximum(g, 0), "reglu": np.maximum(g, 0) * u,
             "drelu": np.maximum(g, 0) * np.maximum(u, 0)}[act]
    ref_y = Wd @ ref_h
    assert np.allclose(h, ref_h, rtol=1e-12, atol=1e-12)
    assert np.allclose(y, ref_y, rtol=1e-11, atol=1e-11)


def test_int4_ffn_matches_dequantised_dense(oracle_mod):
    """INT4 layer (W_down neuron-major) equals the float FFN on the dequantised
    weights, which numpy computes from the hand-checked reader."""
    from activation_sparse_decode_threshold_b200.synth import quantize_int4_g32
    rng = np.random.default_rng(8)
    d, F = 64, 96
    wg, wu = rng.standard_normal((F, d)), rng.standard_normal((F, d))
    wdT = rng.standard_normal((F, d))
    qg, sg = quantize_int4_g32(torch.from_numpy(wg))
    qu, su = quantize_int4_g32(torch.from_numpy(wu))
    qd, sd = quantize_int4_g32(torch.from_numpy(wdT))
    c = rng.standard_normal(F).astype(np.float32)
    x = rng.standard_normal(d)
    e = oracle_mod.Expert(act="drelu", wdtype="int4g32", pdtype="f32", w_gate=qg.numpy(),
                          w_up=qu.numpy(), w_down=qd.numpy(), c=c,
                          U=np.zeros((F, 1), np.float32), V=np.zeros((1, d), np.float32),
                          s_gate=sg.numpy(), s_up=su.numpy(), s_down=sd.numpy())
    h, y = oracle_mod.ffn_masked(e, x)
    Dg = oracle_mod.load_matrix("int4g32", qg.numpy(), sg.numpy(), F, d)
    Du = oracle_mod.load_matrix("int4g32", qu.numpy(), su.numpy(), F, d)
    Dd = oracle_mod.load_matrix("int4g32", qd.numpy(), sd.numpy(), F, d)
    ref_h = np.maximum(Dg @ x - c, 0) * np.maximum(Du @ x, 0)
    assert np.allclose(h, ref_h, rtol=1e-12, atol=1e-12)
    assert np.allclose(y, Dd.T @ ref_h, rtol=1e-11, atol=1e-11)
    # dequantised values are close to the originals (the writer is sane)
    assert np.max(np.abs(Dg - wg)) <= np.max(np.abs(wg)) / 7.0


def test_predictor_matches_numpy_low_rank(oracle_mod):
    rng = np.random.default_rng(9)
    d, F, r = 128, 300, 16
    V = rng.standard_normal((r, d)).astype(np.float32)
    U = rng.standard_normal((F, r)).astype(np.float32)
    c = rng.standard_normal(F).astype(np.float32)
    x = rng.standard_normal(d)
    t, z, mask = oracle_mod.predict(x, V, U, c, "f32")
    tr = V.astype(np.float64) @ x
    zr = U.astype(np.float64) @ tr - c
    assert np.allclose(t, tr, rtol=1e-13, atol=1e-13)
    assert np.allclose(z, zr, rtol=1e-12, atol=1e-12)
    assert np.array_equal(mask.astype(bool), z > 0)


def test_exact_predictor_reproduces_truth_set(oracle_mod):
    """r = d, V = I, U = W_gate, no noise: z equals g exactly, so the predicted
    set equals the set of neurons whose gate fires (recall = precision = 1)."""
    rng = np.random.default_rng(10)
    d, F = 32, 200
    wg = rng.standard_normal((F, d)).astype(np.float32)
    wu = rng.standard_normal((F, d)).astype(np.float32)
    c = rng.standard_normal(F).astype(np.float32)
    x = rng.standard_normal(d)
    e = expert_from(oracle_mod, "reglu", wg, wu, rng.standard_normal((d, F)), c)
    _, z, mask = oracle_mod.predict(x, e.V, e.U, e.c, "f32")
    h, _ = oracle_mod.ffn_masked(e, x)
    assert np.array_equal(mask.astype(bool), h != 0)


def test_threshold_minus_infinity_gives_dense(oracle_mod):
    rng = np.random.default_rng(11)
    d, F = 32, 100
    e = expert_from(oracle_mod, "reglu", rng.standard_normal((F, d)), rng.standard_normal((F, d)),
                    rng.standard_normal((d, F)), rng.standard_normal(F),
                    U=rng.standard_normal((F, 4)), V=rng.standard_normal((4, d)))
    x = rng.standard_normal(d)
    _, _, mask = oracle_mod.predict(x, e.V, e.U, e.c, "f32", threshold=-np.inf)
    assert mask.all()
    assert np.array_equal(oracle_mod.ffn_masked(e, x, mask)[1], oracle_mod.ffn_masked(e, x)[1])


def test_int8_row_predictor_fixture(oracle_mod):
    """Hand-derived fixture of the 8-bit per-row predictor format (signed bytes
    in two's complement, -128 and -127 included, one fp32 scale per row)."""
    g = gold("int8_row_predict.json")
    V = np.array(g["V_bytes"], np.uint8).view(np.int8)
    U = np.array(g["U_bytes"], np.uint8).view(np.int8)
    t, z, mask = oracle_mod.predict(np.array(g["x"]), V, U, f32(g["c"]), "i8row", 0.0,
                                    f32(g["V_scales"]), f32(g["U_scales"]))
    assert np.array_equal(t, np.array(g["t"]))
    assert np.array_equal(z, np.array(g["z"]))
    assert np.array_equal(mask, np.array(g["mask"], np.uint8))


def test_int8_row_predictor_equals_float_predictor_on_its_values(oracle_mod):
    """With power-of-two scales every dequantised element s * q is exact in
    fp32, so the 8-bit predictor must give the float predictor's t, z and mask
    on those fp32 values bit for bit (an independent route to the same
    numbers: numpy forms s * q, the float path reads it back)."""
    rng = np.random.default_rng(21)
    d, F, r = 96, 150, 16
    qV = rng.integers(-128, 128, (r, d)).astype(np.int8)
    qU = rng.integers(-128, 128, (F, r)).astype(np.int8)
    sV = (2.0 ** rng.integers(-9, -4, r)).astype(np.float32)
    sU = (2.0 ** rng.integers(-9, -4, F)).astype(np.float32)
    c = rng.standard_normal(F).astype(np.float32) * 0.1
    x = rng.standard_normal(d)
    Vf = f32(sV[:, None] * qV.astype(np.float32))
    Uf = f32(sU[:, None] * qU.astype(np.float32))
    t1, z1, m1 = oracle_mod.predict(x, qV, qU, c, "i8row", 0.0, sV, sU)
    t2, z2, m2 = oracle_mod.predict(x, Vf, Uf, c, "f32", 0.0)
    assert np.array_equal(t1, t2) and np.array_equal(z1, z2) and np.array_equal(m1, m2)
    # and the numbers are the low-rank predictor of the dequantised matrices
    assert np.allclose(z1, Uf.astype(np.float64) @ (Vf.astype(np.float64) @ x) - c, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("moe", [False, True])
def test_batch_decode_is_per_token_decode_over_the_union(oracle_mod, moe):
    """Small-batch decode reads the union of the tokens' predicted rows once,
    but each token keeps its own set, so its output is its batch-1 output bit
    for bit.  The case is built so that the rule matters: some token has a
    neuron in the union, outside its own set, whose gate fires."""
    rng = np.random.default_rng(31)
    d, F, r, Bn = 24, 64, 6, 5
    E = 3 if moe else 1
    experts = []
    for _ in range(E):
        wg = rng.standard_normal((F, d))
        U, V = rng.standard_normal((F, r)), rng.standard_normal((r, d))
        experts.append(expert_from(oracle_mod, "reglu", wg, rng.standard_normal((F, d)),
                                   rng.standard_normal((d, F)), rng.standard_normal(F) * 0.5, U=U, V=V))
    router = rng.standard_normal((E, d)).astype(np.float16) if moe else None
    R = rng.standard_normal((Bn, d))
    res, union = oracle_mod.decode_layer_batch(R, experts, router)
    matters = False
    for b in range(Bn):
        one = oracle_mod.decode_layer(R[b], experts, router)
        assert one.experts == res[b].experts
        assert np.array_equal(one.y, res[b].y)
        for k, e_id in enumerate(one.experts):
            assert np.array_equal(one.mask[k], res[b].mask[k])
            assert np.array_equal(one.h[k], res[b].h[k])
            h_all, _ = oracle_mod.ffn_masked(experts[e_id], one.x)
            extra = union[e_id].astype(bool) & ~one.mask[k].astype(bool)
            matters |= bool(np.any(h_all[extra] != 0))
    for e_id, u in union.items():
        ref = np.zeros(F, bool)
        for b in range(Bn):
            for k, e2 in enumerate(res[b].experts):
                if e2 == e_id:
                    ref |= res[b].mask[k].astype(bool)
        assert np.array_equal(u.astype(bool), ref)
    assert matters


# ---------------------------------------------------------------------------
# Neuron table
# ---------------------------------------------------------------------------
def test_neuron_table_fixture(oracle_mod):
    g = gold("neuron_table.json")
    assert oracle_mod.strip_offsets(g["F"], g["S"]).tolist() == g["offsets"]
    assert oracle_mod.neuron_table(g["F"], g["S"], g["freq"]).tolist() == g["perm"]


def test_neuron_table_properties(oracle_mod):
    rng = np.random.default_rng(12)
    F, S = 11008, 148
    freq = rng.random(F) ** 4
    perm = oracle_mod.neuron_table(F, S, freq)
    assert np.array_equal(np.sort(perm), np.arange(F))          # a permutation
    inv = np.empty(F, np.int64)
    inv[perm] = np.arange(F)
    assert np.array_equal(perm[inv], np.arange(F))              # perm o perm^-1 = id
    off = oracle_mod.strip_offsets(F, S)
    loads = np.array([freq[perm[off[b]:off[b + 1]]].sum() for b in range(S)])
    assert loads.max() - loads.min() <= freq.max() + 1e-12       # snake dealing balances
    for b in range(S):                                          # hottest first in a strip
        f = freq[perm[off[b]:off[b + 1]]]
        assert np.all(np.diff(f) <= 0)
    assert np.array_equal(oracle_mod.neuron_table(F, S, None), np.arange(F))


def test_permuted_layer_equals_identity_layer(oracle_mod):
    """A layer stored in table order, with its results mapped back through the
    table, equals the layer in original order (exact with integer weights)."""
    rng = np.random.default_rng(13)
    d, F, S = 8, 40, 3
    wg = rng.integers(-3, 4, (F, d)).astype(np.float64)
    wu = rng.integers(-3, 4, (F, d)).astype(np.float64)
    wd = rng.integers(-3, 4, (d, F)).astype(np.float64)
    c = rng.integers(-2, 3, F).astype(np.float64)
    U = rng.integers(-2, 3, (F, 4)).astype(np.float64)
    V = rng.integers(-2, 3, (4, d)).astype(np.float64)
    x = rng.integers(-2, 3, d).astype(np.float64)
    perm = oracle_mod.neuron_table(F, S, rng.random(F))
    e0 = expert_from(oracle_mod, "reglu", wg, wu, wd, c, U=U, V=V)
    e1 = expert_from(oracle_mod, "reglu", wg[perm], wu[perm], wd[:, perm], c[perm], U=U[perm], V=V)
    _, z0, m0 = oracle_mod.predict(x, e0.V, e0.U, e0.c, "f32")
    _, z1, m1 = oracle_mod.predict(x, e1.V, e1.U, e1.c, "f32")
    assert np.array_equal(z1, z0[perm]) and np.array_equal(m1, m0[perm])
    h0, y0 = oracle_mod.ffn_masked(e0, x, m0)
    h1, y1 = oracle_mod.ffn_masked(e1, x, m1)
    assert np.array_equal(h1, h0[perm]) and np.array_equal(y1, y0)


# ---------------------------------------------------------------------------
# MoE routing and combine
# ---------------------------------------------------------------------------
def test_route_top2_fixture(oracle_mod):
    for case in gold("route_top2.json")["cases"]:
        Wr = np.array(case["router"], np.float16)
        logits, ex, w = oracle_mod.route_top2(np.array(case["x"], np.float64), Wr)
        assert np.array_equal(logits, np.array(case["logits"], np.float64))
        assert ex.tolist() == case["experts"]
        assert np.allclose(w, case["weights"], rtol=0, atol=1e-15)


def test_moe_with_identical_experts_equals_single_ffn(oracle_mod):
    rng = np.random.default_rng(14)
    d, F, E = 32, 64, 4
    e = expert_from(oracle_mod, "drelu", rng.standard_normal((F, d)), rng.standard_normal((F, d)),
                    rng.standard_normal((d, F)), rng.standard_normal(F) * 0.1,
                    U=rng.standard_normal((F, 8)), V=rng.standard_normal((8, d)))
    router = rng.standard_normal((E, d)).astype(np.float16)
    r = rng.standard_normal(d)
    single = oracle_mod.decode_layer(r, [e])
    moe = oracle_mod.decode_layer(r, [e] * E, router)
    assert len(moe.experts) == 2 and moe.experts[0] < moe.experts[1]
    assert abs(sum(moe.weights) - 1.0) < 1e-15
    assert np.allclose(moe.y, single.y, rtol=1e-14, atol=1e-14)


def test_moe_combine_uses_selected_experts_only(oracle_mod):
    rng = np.random.default_rng(15)
    d, F, E = 16, 32, 4
    experts = [expert_from(oracle_mod, "reglu", rng.standard_normal((F, d)),
                           rng.standard_normal((F, d)), rng.standard_normal((d, F)),
                           rng.standard_normal(F) * 0.1, U=rng.standard_normal((F, 4)),
                           V=rng.standard_normal((4, d))) for _ in range(E)]
    router = rng.standard_normal((E, d)).astype(np.float16)
    r = rng.standard_normal(d)
    res = oracle_mod.decode_layer(r, experts, router)
    x = oracle_mod.rmsnorm(r)
    ys = [oracle_mod.decode_layer(r, [experts[k]]).y for k in res.experts]
    ref = res.weights[0] * ys[0] + res.weights[1] * ys[1]
    assert np.array_equal(res.y, ref)
    lg = router.astype(np.float64) @ x
    top = sorted(np.argsort(-lg, kind="stable")[:2].tolist())
    assert res.experts == top


# ---------------------------------------------------------------------------
# Stack composition
# ---------------------------------------------------------------------------
def test_stack_is_residual_composition(oracle_mod):
    rng = np.random.default_rng(16)
    d, F = 16, 48
    layers = [[expert_from(oracle_mod, "reglu", rng.standard_normal((F, d)),
                           rng.standard_normal((F, d)), rng.standard_normal((d, F)) * 0.1,
                           rng.standard_normal(F), U=rng.standard_normal((F, 4)),
                           V=rng.standard_normal((4, d)))] for _ in range(3)]
    r0 = rng.standard_normal(d)
    r_final, res = oracle_mod.decode_stack(r0, layers)
    r = r0.copy()
    for l in range(3):
        x = r / np.sqrt(np.mean(r * r) + 1e-6)
        assert np.allclose(res[l].x, x, rtol=1e-14, atol=1e-14)
        r = r + res[l].y
    assert np.allclose(r_final, r, rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------------------
# Dense prefill (PowerInfer-2, "Neuron-cluster heterogeneous computing")
# ---------------------------------------------------------------------------
def test_prefill_equals_matrix_form(oracle_mod):
    """T tokens through a dense ReGLU FFN equal the matrix form of the layer,
    Y = (relu(X Wg^T - c) * (X Wu^T)) Wd^T with X the row-wise RMSNorm of R,
    written with numpy matmuls."""
    rng = np.random.default_rng(21)
    T, d, F = 7, 16, 40
    wg, wu = rng.standard_normal((F, d)), rng.standard_normal((F, d))
    wd, c = rng.standard_normal((d, F)), rng.standard_normal(F)
    e = expert_from(oracle_mod, "reglu", wg, wu, wd, c)
    R = rng.standard_normal((T, d))
    res = oracle_mod.prefill_layer(R, [e])
    X = R / np.sqrt((R * R).mean(axis=1, keepdims=True) + 1e-6)
    wg32, wu32, wd32, c32 = (f32(a).astype(np.float64) for a in (wg, wu, wd, c))
    H = np.maximum(X @ wg32.T - c32, 0) * (X @ wu32.T)
    assert np.allclose(res.x, X, rtol=1e-14, atol=1e-14)
    assert np.allclose(res.y, H @ wd32.T, rtol=1e-12, atol=1e-12)
    assert np.array_equal(res.r_out, R + res.y)


def test_prefill_rows_are_decode_with_every_neuron_active(oracle_mod):
    """Each prefill row is the decode layer of that token with threshold -inf
    (every neuron active), for an INT4 dReLU MoE; routing per token."""
    from activation_sparse_decode_threshold_b200.synth import quantize_int4_g32
    rng = np.random.default_rng(22)
    T, d, F, E = 5, 64, 32, 4
    experts = []

    def q4(shape):
        q, s = quantize_int4_g32(torch.from_numpy(rng.standard_normal(shape).astype(np.float32)))
        return q.numpy(), s.numpy()
    for _ in range(E):
        qg, sg = q4((F, d))
        qu, su = q4((F, d))
        qd, sd = q4((F, d))
        experts.append(oracle_mod.Expert(
            act="drelu", wdtype="int4g32", pdtype="f16", w_gate=qg, w_up=qu, w_down=qd,
            c=f32(rng.standard_normal(F) * 0.1), U=rng.standard_normal((F, 8)).astype(np.float16),
            V=rng.standard_normal((8, d)).astype(np.float16), s_gate=sg, s_up=su, s_down=sd))
    router = rng.standard_normal((E, d)).astype(np.float16)
    R = rng.standard_normal((T, d))
    res = oracle_mod.prefill_layer(R, experts, router)
    for t in range(T):
        ref = oracle_mod.decode_layer(R[t], experts, router, threshold=-np.inf)
        assert all(m.all() for m in ref.mask)
        assert res.experts[t].tolist() == ref.experts
        assert np.array_equal(res.y[t], ref.y)
    # token order does not matter: a permutation of the rows permutes the results
    p = rng.permutation(T)
    assert np.array_equal(oracle_mod.prefill_layer(R[p], experts, router).y, res.y[p])
