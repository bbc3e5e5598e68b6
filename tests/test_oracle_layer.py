"""Pins for the oracle's grouped FP8 GEMMs, SwiGLU, requantization and combine (CPU only).

Sources: "metrale_model_layers fp8_grouped_tc_w8a8.rs", run_fp8_grouped_w8a8 (act-quant ->
gate+up with quantized SiLU products -> down; "a row's bits still do not depend on the other
rows"); "MATE Mega MoE", API (activation swiglu) and Current Limits (contiguous bf16 output);
"MindIE-SD Fused MoE", parameter table (w13 [E, hidden, 2*inter], w2 [E, inter, hidden],
w13_bias [E, 2*inter], w2_bias [E, hidden]) and execution flow.

Pins: special cases that reduce to an exact integer matmul (numpy), a dense fp64 torch matmul
on the dequantized operands, closed forms for the bias / SwiGLU path, and invariances
(expert relabeling, token subsets and order, the permuted formulation).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

# E4M3 codes of the small integers -8..8 (exact values; checked against torch below)
INT_CODES = {v: int(torch.tensor([float(v)]).to(torch.float8_e4m3fn).view(torch.uint8)[0])
             for v in range(-8, 9)}


def _int_operands(rng, shape):
    v = rng.integers(-8, 9, shape)
    codes = np.vectorize(INT_CODES.get)(v).astype(np.uint8)
    return v.astype(np.int64), codes


@pytest.mark.parametrize("recipe", [0, 1])
def test_gemv_unit_scales_is_integer_matmul(recipe):
    rng = np.random.default_rng(0)
    K, N = 384, 200                       # K != N catches a transposed operand
    g = 128 if recipe == 0 else 32
    av, aq = _int_operands(rng, K)
    wv, wq = _int_operands(rng, (K, N))
    one = (np.ones, np.float32) if recipe == 0 else (lambda s, dtype: np.full(s, 127, dtype), np.uint8)
    as_ = one[0](K // g, dtype=one[1])
    ws = one[0]((K // g, N), dtype=one[1])
    out = oracle.scaled_gemv(recipe, aq, as_, wq, ws)
    assert np.array_equal(out, (av @ wv).astype(np.float64))


@pytest.mark.parametrize("recipe", [0, 1])
def test_gemv_block_scales_weight_each_group(recipe):
    rng = np.random.default_rng(1)
    K, N = 256, 96
    g = 128 if recipe == 0 else 32
    G = K // g
    av, aq = _int_operands(rng, K)
    wv, wq = _int_operands(rng, (K, N))
    ea = rng.integers(-6, 7, G)
    ew = rng.integers(-6, 7, (G, N))
    if recipe == 0:
        as_ = np.exp2(ea).astype(np.float32) * np.float32(1.5)
        ws = np.exp2(ew).astype(np.float32) * np.float32(1.25)
    else:
        as_ = (ea + 127).astype(np.uint8)
        ws = (ew + 127).astype(np.uint8)
    out = oracle.scaled_gemv(recipe, aq, as_, wq, ws)
    ref = np.zeros(N)
    for gi in range(G):
        part = av[gi * g:(gi + 1) * g] @ wv[gi * g:(gi + 1) * g]
        sa = float(as_[gi]) if recipe == 0 else 2.0 ** ea[gi]
        sw = ws[gi].astype(np.float64) if recipe == 0 else np.exp2(ew[gi].astype(np.float64))
        ref += sa * sw * part
    assert np.array_equal(out, ref)


def _single_expert_problem(H, I, recipe=0, seed=0):
    shp = synth.Shape("one", 3, H, I, 1, 1, renormalize=1, recipe=recipe, seed=seed)
    return shp, synth.make_problem(shp)


def _dequant_rows(codes, scales, recipe):
    """codes [..., K] uint8 + scales [..., K/g] -> fp64 values, via torch's float8 decode."""
    g = 128 if recipe == 0 else 32
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()
    s = scales.astype(np.float64) if recipe == 0 else np.exp2(scales.astype(np.float64) - 127)
    return v * np.repeat(s, g, axis=-1)


def _dequant_weight(codes, scales, recipe):
    """codes [K, N], scales [K/g, N] -> fp64 [K, N]."""
    g = 128 if recipe == 0 else 32
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()
    s = scales.astype(np.float64) if recipe == 0 else np.exp2(scales.astype(np.float64) - 127)
    return v * np.repeat(s, g, axis=0)


@pytest.mark.parametrize("recipe", [0, 1])
def test_dense_case_matches_torch_fp64_swiglu_mlp(recipe):
    """E = k = 1: the layer is a dense SwiGLU MLP on dequantized operands.  Gate+up and the
    SwiGLU product are checked against a torch fp64 matmul (the act codes agree wherever the
    fp64 value is not within 1e-9 of a rounding boundary), and y against torch on the oracle's
    own act codes."""
    H, I = 256, 384
    shp, p = _single_expert_problem(H, I, recipe)
    ni = p.numpy_inputs()
    c = oracle.Config(**shp.cfg())
    y, act_q, act_s = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"],
                                     logits=ni["logits"], want_act=True)
    xq, xs = oracle.quantize_tokens(ni["x"], recipe)
    xd = _dequant_rows(xq, xs, recipe)                                  # [T,H]
    w13 = _dequant_weight(ni["w13"][0], ni["w13s"][0], recipe)          # [H,2I]
    w2 = _dequant_weight(ni["w2"][0], ni["w2s"][0], recipe)             # [I,H]
    h = torch.from_numpy(xd) @ torch.from_numpy(w13)
    a = (torch.nn.functional.silu(h[:, :I]) * h[:, I:]).numpy().astype(np.float32)
    for t in range(shp.num_tokens):
        q_ref, s_ref = oracle.quant_row(a[t], recipe)
        assert np.mean(q_ref == act_q[t, 0]) > 0.995
        assert np.mean(s_ref == act_s[t, 0]) > 0.9
    ad = _dequant_rows(act_q[:, 0], act_s[:, 0], recipe)
    o = (torch.from_numpy(ad) @ torch.from_numpy(w2)).numpy()          # weight is exactly 1
    yref = np.array([[oracle.bf16_from_double(v) for v in row] for row in o], np.uint16)
    assert np.array_equal(y, yref)


def test_bias_and_swiglu_closed_form():
    """W13 = 0, gate bias 1, up bias 2: act = silu(1) * 2 everywhere (gate first, up second);
    one group -> every code is 448 and the scale is amax/448; W2 = identity, b2 = 0.25."""
    H = I = 128
    shp = synth.Shape("cf", 1, H, I, 1, 1, renormalize=1)
    x = np.zeros((1, H), np.uint16)
    logits = np.zeros((1, 1), np.float32)
    w13 = np.zeros((1, H, 2 * I), np.uint8)
    w13s = np.ones((1, 1, 2 * I), np.float32)
    w2 = np.zeros((1, I, H), np.uint8)
    w2[0][np.arange(I), np.arange(H)] = INT_CODES[1]
    w2s = np.ones((1, 1, H), np.float32)
    bf = lambda v: np.array([v], np.float32).view(np.uint32).astype(np.uint64) >> 16
    b13 = np.concatenate([np.full(I, bf(1.0)[0]), np.full(I, bf(2.0)[0])]).astype(np.uint16)[None]
    b2 = np.full((1, H), bf(0.25)[0], np.uint16)
    c = oracle.Config(**shp.cfg())
    y, act_q, act_s = oracle.forward(c, x, w13, w13s, w2, w2s, logits=logits, b13=b13, b2=b2,
                                     want_act=True)
    a = np.float32(1.0 / (1.0 + math.exp(-1.0)) * 2.0)
    s = np.float32(a / np.float32(448.0))
    assert np.all(act_q == 0x7E) and np.all(act_s == s)
    expect = oracle.bf16_from_double(448.0 * float(s) + 0.25)
    assert np.all(y == expect)
    # swapping gate and up would give silu(2) * 1 instead
    assert abs(float(a) - 1.0 / (1.0 + math.exp(-2.0)) * 2.0) > 0.1


def test_zero_weights_leave_weighted_down_bias():
    """W2 = 0: y_t = bf16( sum_j w_j * b2[e_j] ), which pins the combine's weights and order."""
    shp = synth.Shape("zb", 9, 128, 128, 4, 2, renormalize=0, biases=True, seed=3)
    p = synth.make_problem(shp)
    ni = p.numpy_inputs()
    w2 = np.zeros_like(ni["w2"])
    c = oracle.Config(**shp.cfg())
    y = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], w2, ni["w2s"], logits=ni["logits"],
                       b13=ni["b13"], b2=ni["b2"])
    idx, w, _ = oracle.route(c, ni["logits"])
    b2f = oracle.bf16_bits_to_f32(ni["b2"]).astype(np.float64)
    for t in range(shp.num_tokens):
        acc = sum(float(w[t, j]) * b2f[idx[t, j]] for j in range(2))
        assert np.array_equal(y[t], [oracle.bf16_from_double(v) for v in acc])


def test_w2_scale_doubling_doubles_output():
    shp = synth.Shape("lin", 5, 256, 256, 3, 2, renormalize=1, seed=5)
    ni = synth.make_problem(shp).numpy_inputs()
    c = oracle.Config(**shp.cfg())
    y1 = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"], logits=ni["logits"])
    y2 = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"] * 2,
                        logits=ni["logits"])
    assert np.array_equal(oracle.bf16_bits_to_f32(y2), 2 * oracle.bf16_bits_to_f32(y1))


@pytest.mark.parametrize("recipe", [0, 1])
def test_expert_relabeling_invariance(recipe):
    shp = synth.Shape("rel", 11, 256, 128, 6, 3, renormalize=1, recipe=recipe, biases=True,
                      per_expert_scale=True, seed=6)
    ni = synth.make_problem(shp).numpy_inputs()
    c = oracle.Config(**shp.cfg())
    y = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"],
                       logits=ni["logits"], per_expert_scale=ni["per_expert_scale"],
                       b13=ni["b13"], b2=ni["b2"])
    perm = np.random.default_rng(0).permutation(6)
    inv = np.argsort(perm)
    # new expert i is old expert perm[i]; logits columns move with it.  The logits have no ties,
    # so the selection (and its order) is the same set of old experts.
    yp = oracle.forward(c, ni["x"], ni["w13"][perm], ni["w13s"][perm], ni["w2"][perm],
                        ni["w2s"][perm], logits=ni["logits"][:, perm],
                        per_expert_scale=ni["per_expert_scale"][perm],
                        b13=ni["b13"][perm], b2=ni["b2"][perm])
    assert np.array_equal(y, yp)
    assert len(set(inv)) == 6


def test_rows_independent_of_batch_and_order():
    """A row's output bits do not depend on the other rows (metrale module doc)."""
    shp = synth.Shape("bi", 23, 256, 256, 5, 2, renormalize=1, seed=7)
    ni = synth.make_problem(shp).numpy_inputs()
    c = oracle.Config(**shp.cfg())
    args = (ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"])
    y = oracle.forward(c, *args, logits=ni["logits"])
    sel = np.array([22, 0, 7, 7, 3], np.int32)
    ys = oracle.forward(c, *args, logits=ni["logits"], tokens=sel)
    assert np.array_equal(ys, y[sel])
    rev = np.arange(23)[::-1].copy()
    c2 = oracle.Config(**shp.cfg())
    yr = oracle.forward(c2, ni["x"][rev], *args[1:], logits=ni["logits"][rev])
    assert np.array_equal(yr, y[rev])


@pytest.mark.parametrize("name", ["tiny"] + [f"rand{i}" for i in range(6)])
def test_per_token_equals_permuted_formulation(name):
    shp = synth.SHAPES[name] if name in synth.SHAPES else synth.random_shape(int(name[4:]))
    ni = synth.make_problem(shp).numpy_inputs()
    c = oracle.Config(**shp.cfg())
    y = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"],
                       logits=ni["logits"], per_expert_scale=ni["per_expert_scale"],
                       b13=ni["b13"], b2=ni["b2"])
    yp = oracle.forward_permuted(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"],
                                 ni["logits"], ni["per_expert_scale"], ni["b13"], ni["b2"])
    assert np.array_equal(y, yp)


def test_given_routing_path_matches_computed_routing():
    shp = synth.SHAPES["tiny"]
    ni = synth.make_problem(shp).numpy_inputs()
    c = oracle.Config(**shp.cfg())
    idx, w, _ = oracle.route(c, ni["logits"])
    y1 = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"], logits=ni["logits"])
    y2 = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"], topk_idx=idx,
                        topk_weights=w)
    assert np.array_equal(y1, y2)


def test_bf16_rounding_from_double():
    assert oracle.bf16_from_double(1.0) == 0x3F80
    assert oracle.bf16_from_double(1.0 + 2 ** -8) == 0x3F80          # tie -> even
    assert oracle.bf16_from_double(1.0 + 3 * 2 ** -8) == 0x3F82       # tie -> even (up)
    assert oracle.bf16_from_double(1.0 + 2 ** -8 + 2 ** -30) == 0x3F81
    assert oracle.bf16_from_double(-2.5) == 0xC020
    assert oracle.bf16_from_double(0.0) == 0 and oracle.bf16_from_double(-0.0) == 0x8000
    rng = np.random.default_rng(9)
    v = rng.standard_normal(2000) * 10.0 ** rng.uniform(-30, 30, 2000)
    # one rounding from double agrees with torch's fp64 -> bf16 conversion
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_from_double(x) for x in v], np.uint16)
    assert np.array_equal(got, ref)
