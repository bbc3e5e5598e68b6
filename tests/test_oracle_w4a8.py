"""Pins for the oracle's W4A8 recipe (recipe 2): E2M1 (FP4) weights with one UE8M0 power-of-two
scale per 32 K-elements, MXFP8 activations (CPU only).

Sources: "DeepGEMM PR #371: Add W8A8 (FP8xFP8) Mega MoE support", Changes (the W8A8 kernel is
derived from the W4A8 (FP8xFP4) path: e2m1 weights, the same 4-packed UE8M0 scale factors);
"MATE Mega MoE", Use Mega MoE when (the W4A8 mixed-dtype GEMM path).

Pins: the E2M1 value table of the format's definition (tests/golden/e2m1_values.txt) and a
brute-force nearest search for the input rounding; a GEMM with unit scales and the packed
nibble order written out here, compared with an exact integer matmul; per-group scales; a
dense fp64 SwiGLU MLP for one expert; scale linearity.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e2m1_values.txt")


def _golden():
    tab = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        c, v = line.split()
        tab[int(c)] = float(v)
    return tab


def test_e2m1_decode_matches_the_format_table():
    tab = _golden()
    assert sorted(tab) == list(range(16))
    for c, v in tab.items():
        d = oracle.e2m1_decode(c)
        assert d == v and np.signbit(d) == np.signbit(v), (c, d, v)


def test_input_rounding_is_nearest_even_on_the_e2m1_grid():
    """The synthetic weights' FP4 rounding: brute force over the 16 codes, ties to the code
    with an even mantissa bit, saturation at 6."""
    tab = _golden()
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.normal(0, 3, 2000), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, 9.0, -0.0]])
    codes = synth._e2m1_codes(torch.tensor(v, dtype=torch.float32)).numpy()
    for x, c in zip(v.astype(np.float32), codes):
        a = min(abs(float(x)), 6.0)
        best = min(range(8), key=lambda k: (abs(tab[k] - a), k % 2))   # nearest, then even
        want = best | (8 if x < 0 and best else 0)
        assert c == want, (x, c, want)


def _pack(codes):
    """[K, N] codes 0..15 -> [K, N/2] bytes, column 2j in the low nibble, 2j+1 in the high."""
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


E4M3_INT = {v: int(torch.tensor([float(v)]).to(torch.float8_e4m3fn).view(torch.uint8)[0])
            for v in range(-8, 9)}


def _operands(rng, K, N):
    tab = _golden()
    av = rng.integers(-8, 9, K)
    aq = np.vectorize(E4M3_INT.get)(av).astype(np.uint8)
    wc = rng.integers(0, 16, (K, N)).astype(np.uint8)
    wv = np.vectorize(tab.get)(wc)
    return av.astype(np.float64), aq, wc, wv


def test_gemv_unit_scales_is_exact_matmul_with_packed_nibbles():
    rng = np.random.default_rng(1)
    K, N = 192, 160                        # K != N catches a transposed operand
    av, aq, wc, wv = _operands(rng, K, N)
    as_ = np.full(K // 32, 127, np.uint8)
    ws = np.full((K // 32, N), 127, np.uint8)
    out = oracle.scaled_gemv(2, aq, as_, _pack(wc), ws)
    assert np.array_equal(out, av @ wv)
    # the other nibble order gives a different answer (the pin can tell them apart)
    swapped = (wc[:, 1::2] | (wc[:, 0::2] << 4)).astype(np.uint8)
    assert not np.array_equal(oracle.scaled_gemv(2, aq, as_, swapped, ws), av @ wv)


def test_gemv_block_scales_weight_each_32_group():
    rng = np.random.default_rng(2)
    K, N = 128, 64
    av, aq, wc, wv = _operands(rng, K, N)
    ea = rng.integers(-6, 7, K // 32)
    ew = rng.integers(-6, 7, (K // 32, N))
    out = oracle.scaled_gemv(2, aq, (ea + 127).astype(np.uint8), _pack(wc), (ew + 127).astype(np.uint8))
    ref = np.zeros(N)
    for g in range(K // 32):
        ref += 2.0 ** ea[g] * np.exp2(ew[g].astype(np.float64)) * (av[32 * g:32 * g + 32] @ wv[32 * g:32 * g + 32])
    assert np.array_equal(out, ref)


def _dequant_w4(packed, scales):
    """[K, N/2] bytes + UE8M0 [K/32, N] -> fp64 [K, N] via the golden table."""
    tab = np.array([v for _, v in sorted(_golden().items())])
    codes = np.empty((packed.shape[0], packed.shape[1] * 2), np.uint8)
    codes[:, 0::2] = packed & 15
    codes[:, 1::2] = packed >> 4
    return tab[codes] * np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=0)


def test_dense_case_matches_torch_fp64_swiglu_mlp():
    """E = k = 1: the layer is a dense SwiGLU MLP on the dequantized operands."""
    H, I = 256, 384
    shp = synth.Shape("one_w4", 3, H, I, 1, 1, renormalize=1, recipe=2, seed=7)
    p = synth.make_problem(shp)
    ni = p.numpy_inputs()
    assert ni["w13"].shape == (1, H, I) and ni["w2"].shape == (1, I, H // 2)
    c = oracle.Config(**shp.cfg())
    y, act_q, act_s = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"],
                                     logits=ni["logits"], want_act=True)
    xq, xs = oracle.quantize_tokens(ni["x"], 2)
    xd = torch.from_numpy(xq).view(torch.float8_e4m3fn).double().numpy() * \
        np.repeat(np.exp2(xs.astype(np.float64) - 127), 32, axis=-1)
    w13 = _dequant_w4(ni["w13"][0], ni["w13s"][0])
    w2 = _dequant_w4(ni["w2"][0], ni["w2s"][0])
    h = torch.from_numpy(xd) @ torch.from_numpy(w13)
    a = (torch.nn.functional.silu(h[:, :I]) * h[:, I:]).numpy().astype(np.float32)
    for t in range(shp.num_tokens):
        q_ref, s_ref = oracle.quant_row(a[t], 2)
        assert np.mean(q_ref == act_q[t, 0]) > 0.995
        assert np.mean(s_ref == act_s[t, 0]) > 0.9
    ad = torch.from_numpy(act_q[:, 0]).view(torch.float8_e4m3fn).double().numpy() * \
        np.repeat(np.exp2(act_s[:, 0].astype(np.float64) - 127), 32, axis=-1)
    o = (torch.from_numpy(ad) @ torch.from_numpy(w2)).numpy()
    yref = np.array([[oracle.bf16_from_double(v) for v in row] for row in o], np.uint16)
    assert np.array_equal(y, yref)


def test_w2_scale_step_doubles_the_output():
    """Adding one to every W2 UE8M0 byte multiplies the down projection by exactly 2, so y
    doubles exactly (bf16 rounding commutes with a power of two)."""
    shp = synth.Shape("lin_w4", 5, 128, 256, 4, 2, renormalize=1, recipe=2, seed=8)
    p = synth.make_problem(shp)
    ni = p.numpy_inputs()
    c = oracle.Config(**shp.cfg())
    y1 = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"], logits=ni["logits"])
    y2 = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], (ni["w2s"] + 1).astype(np.uint8),
                        logits=ni["logits"])
    f1 = oracle.bf16_bits_to_f32(y1).astype(np.float64)
    f2 = oracle.bf16_bits_to_f32(y2).astype(np.float64)
    assert np.array_equal(2.0 * f1, f2)


@pytest.mark.parametrize("seed", [0, 1])
def test_per_token_equals_permuted_formulation(seed):
    shp = synth.random_shape(seed, recipe=2)
    p = synth.make_problem(shp)
    ni = p.numpy_inputs()
    c = oracle.Config(**shp.cfg())
    y = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"], logits=ni["logits"],
                       per_expert_scale=ni["per_expert_scale"])
    yp = oracle.forward_permuted(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"], ni["logits"],
                                 per_expert_scale=ni["per_expert_scale"])
    assert np.array_equal(y, yp)
