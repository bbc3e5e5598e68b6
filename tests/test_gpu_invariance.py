"""GPU properties that hold at any size.

- A row's output bits do not depend on the other rows of the batch ("metrale_model_layers
  fp8_grouped_tc_w8a8.rs", module doc): a subset, a reversed batch and single tokens give the
  same bits as the full batch.
- Runs are deterministic: the same call twice gives the same bits (no atomics in any
  reduction; "DeepGEMM PR #371", Testing: bitwise-identical outputs).
- The given-routing path (custom routing function, "MindIE-SD Fused MoE") equals the computed
  routing when fed the same ids and weights.
"""
import numpy as np
import pytest
import torch

import synth
from _helpers import GpuProblem, bits, lib_cfg

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "decode", "skewed", "prefill", "large"])
def test_batch_invariance(name):
    """Full-size prefill and large run the wide kernels on the full batch and on the half batch,
    the narrow (swap-AB) kernels on the single tokens."""
    prob = synth.make_problem(name, device="cuda" if name in ("prefill", "large") else "cpu")
    gp = GpuProblem(prob)
    y_full = bits(gp.forward())
    T = prob.shape.num_tokens
    rng = np.random.default_rng(3)
    subsets = [np.arange(T)[::-1].copy(), np.sort(rng.choice(T, max(1, T // 2), replace=False)),
               np.array([0]), np.array([T - 1])]
    for sub in subsets:
        sub_t = torch.from_numpy(sub).cuda()
        c = lib_cfg(prob.shape.with_tokens(len(sub)))
        ws = gp.moe.new_workspace(c)
        y = gp.forward(x=gp.d.x[sub_t].contiguous(), logits=gp.d.logits[sub_t].contiguous(), cfg=c, workspace=ws)
        assert np.array_equal(bits(y), y_full[sub]), f"rows changed with batch composition ({len(sub)} rows)"


@pytest.mark.parametrize("name", ["decode", "skewed"])
def test_deterministic(name):
    gp = GpuProblem(synth.make_problem(name))
    a = bits(gp.forward())
    b = bits(gp.forward())
    assert np.array_equal(a, b)


def test_given_routing_matches_computed():
    gp = GpuProblem(synth.make_problem("decode"))
    y1 = bits(gp.forward())
    T, K = gp.shape.num_tokens, gp.shape.top_k
    idx = gp.ws_region("topk_idx", torch.int32, T * K).clone().view(T, K)
    w = gp.ws_region("topk_weights", torch.float32, T * K).clone().view(T, K)
    y2 = bits(gp.forward(topk_idx=idx, topk_weights=w))
    assert np.array_equal(y1, y2)


@pytest.mark.parametrize("recipe", [0, 1, 2])
def test_narrow_and_wide_kernels_agree_bit_for_bit(recipe):
    """A batch with few rows per expert runs the swap-AB (narrow) GEMMs; the same tokens inside a
    large batch run the wide GEMMs.  Both compute each row with the same operations, so the rows
    must agree bit for bit (a row's output does not depend on the other rows)."""
    from dataclasses import replace
    base = replace(synth.SHAPES["decode"], recipe=recipe, biases=True)
    small = synth.make_problem(base)                       # 64 tokens: 512 rows <= 32 * 128 -> narrow
    big_shape = base.with_tokens(4096)                     # 32768 rows -> wide
    x_big, logits_big, _ = synth.make_activations(big_shape)
    assert torch.equal(x_big[:64], small.x) and torch.equal(logits_big[:64], small.logits)
    gp = GpuProblem(small)
    y_small = bits(gp.forward())
    c = lib_cfg(big_shape)
    ws = gp.moe.new_workspace(c)
    y_big = bits(gp.forward(x=x_big.cuda(), logits=logits_big.cuda(), cfg=c, workspace=ws))
    assert np.array_equal(y_small, y_big[:64])
