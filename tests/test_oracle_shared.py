"""Pins for the oracle's shared expert (CPU only).

Source: "metrale_model_layers fp8_grouped_tc_w8a8.rs", run_fp8_grouped_w8a8: the shared expert's
gate/up and down projections run in the same grouped steps as the routed experts, on the same
quantized layer input.  Reading: it is one more expert (index num_experts) that every token uses
with weight 1, after the routed slots.

Pins: with every routed down projection zero the layer is the shared expert alone, checked
against a dense torch fp64 SwiGLU MLP; with every down projection zero the output is a closed
form in the down biases (weight 1 on the shared expert's); the permuted formulation agrees bit
for bit; the routed experts' part is unchanged by adding a shared expert.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
import synth
from test_oracle_layer import _dequant_rows, _dequant_weight


def _run(shp, ni, **over):
    c = oracle.Config(**shp.cfg())
    args = dict(logits=ni["logits"], per_expert_scale=ni["per_expert_scale"], b13=ni["b13"], b2=ni["b2"])
    args.update(over)
    return oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"], **args)


@pytest.mark.parametrize("recipe", [0, 1])
def test_shared_expert_alone_matches_dense_torch_mlp(recipe):
    H, I, E = 256, 384, 4
    shp = synth.Shape("sh", 5, H, I, E, 2, renormalize=1, recipe=recipe, seed=21, shared_experts=1)
    ni = synth.make_problem(shp).numpy_inputs()
    w2 = ni["w2"].copy()
    w2[:E] = 0                                         # routed experts contribute nothing
    c = oracle.Config(**shp.cfg())
    y, act_q, act_s = oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], w2, ni["w2s"],
                                     logits=ni["logits"], want_act=True)
    assert act_q.shape[1] == 3                         # two routed slots + the shared one
    xq, xs = oracle.quantize_tokens(ni["x"], recipe)
    xd = _dequant_rows(xq, xs, recipe)
    w13 = _dequant_weight(ni["w13"][E], ni["w13s"][E], recipe)
    w2s = _dequant_weight(ni["w2"][E], ni["w2s"][E], recipe)
    h = torch.from_numpy(xd) @ torch.from_numpy(w13)
    a = (torch.nn.functional.silu(h[:, :I]) * h[:, I:]).numpy().astype(np.float32)
    for t in range(shp.num_tokens):
        q_ref, _ = oracle.quant_row(a[t], recipe)
        assert np.mean(q_ref == act_q[t, 2]) > 0.995
    ad = _dequant_rows(act_q[:, 2], act_s[:, 2], recipe)
    o = (torch.from_numpy(ad) @ torch.from_numpy(w2s)).numpy()
    yref = np.array([[oracle.bf16_from_double(v) for v in row] for row in o], np.uint16)
    assert np.array_equal(y, yref)


def test_zero_down_weights_give_biases_with_unit_shared_weight():
    """W2 = 0 everywhere: y_t = bf16( sum_j w_j * b2[e_j] + 1 * b2[E] )."""
    E = 4
    shp = synth.Shape("shb", 9, 128, 128, E, 2, renormalize=0, biases=True, seed=22, shared_experts=1)
    ni = synth.make_problem(shp).numpy_inputs()
    w2 = np.zeros_like(ni["w2"])
    y = oracle.forward(oracle.Config(**shp.cfg()), ni["x"], ni["w13"], ni["w13s"], w2, ni["w2s"],
                       logits=ni["logits"], b13=ni["b13"], b2=ni["b2"])
    idx, w, _ = oracle.route(oracle.Config(**shp.cfg()), ni["logits"])
    b2f = oracle.bf16_bits_to_f32(ni["b2"]).astype(np.float64)
    assert b2f.shape[0] == E + 1
    for t in range(shp.num_tokens):
        acc = sum(float(w[t, j]) * b2f[idx[t, j]] for j in range(2)) + b2f[E]
        assert np.array_equal(y[t], [oracle.bf16_from_double(v) for v in acc])


@pytest.mark.parametrize("name", ["tiny", "rand1", "rand4"])
def test_shared_per_token_equals_permuted_formulation(name):
    base = synth.SHAPES[name] if name in synth.SHAPES else synth.random_shape(int(name[4:]))
    shp = replace(base, shared_experts=1)
    ni = synth.make_problem(shp).numpy_inputs()
    c = oracle.Config(**shp.cfg())
    y = _run(shp, ni)
    yp = oracle.forward_permuted(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"],
                                 ni["logits"], ni["per_expert_scale"], ni["b13"], ni["b2"])
    assert np.array_equal(y, yp)


def test_adding_a_shared_expert_keeps_the_routed_part():
    """The shared expert's down projection zeroed (and no biases): same bits as no shared expert."""
    base = synth.Shape("sh0", 7, 256, 256, 6, 2, renormalize=1, seed=23)
    shp = replace(base, shared_experts=1)
    ni1 = synth.make_problem(shp).numpy_inputs()
    ni0 = synth.make_problem(base).numpy_inputs()
    w2 = ni1["w2"].copy()
    w2[6] = 0
    c1 = oracle.Config(**shp.cfg())
    y1 = oracle.forward(c1, ni1["x"], ni1["w13"], ni1["w13s"], w2, ni1["w2s"], logits=ni1["logits"])
    y0 = _run(base, ni0)
    assert np.array_equal(y0, y1)


def test_shared_experts_field_is_validated():
    shp = replace(synth.SHAPES["tiny"], shared_experts=2)
    ni = synth.make_problem(replace(shp, shared_experts=0)).numpy_inputs()
    with pytest.raises(ValueError):
        _run(shp, ni)
