"""Fused against unfused gate+up, bit for bit ("DeepGEMM PR #371", Testing: the overlapped kernel's
outputs are bitwise identical to the non-overlapped baseline).

moe_forward computes SwiGLU and the requantization inside the gate+up GEMM's epilogue.
moe_debug_unfused_gate_up runs the same build's steps apart: the GEMM stores the fp32 gate/up sums
h, then a separate kernel adds the bias, applies SwiGLU and requantizes.  On the same routing the
act codes and scales in the workspace must be identical.  The problems cover every GEMM kernel the
forward picks: the swap-AB kernels (tiny, decode, W4A8 decode), the CTA-pair kernel (the large
problem cut to 2048 tokens, and a problem with biases), the block-scaled kernels (skewed MXFP8).
As a check on h itself, the fp32 gate/up sums of a few rows are compared with the oracle's
pre-activation values through the act codes' scales: SwiGLU of h reproduces the oracle's act."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import GpuProblem, oracle_cfg

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": synth.SHAPES["tiny"],
    "decode": synth.SHAPES["decode"],
    "decode_w4a8": synth.SHAPES["decode_w4a8"],
    "large_2048": synth.SHAPES["large"].with_tokens(2048),
    "wide_biases": synth.Shape("uf_wide", 600, 512, 384, 4, 2, renormalize=1, seed=71, biases=True),
    "skewed": synth.SHAPES["skewed"],
    "wide_mx_biases": synth.Shape("uf_mx", 600, 512, 384, 4, 2, renormalize=1, recipe=1, seed=72, biases=True),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fused_equals_unfused_bit_for_bit(name):
    shape = CASES[name]
    dev = "cuda" if name == "large_2048" else "cpu"
    prob = synth.make_problem(shape, device=dev)
    gp = GpuProblem(prob)
    ni = prob.numpy_inputs()
    idx, w, _ = oracle.route(oracle_cfg(shape), ni["logits"], ni["per_expert_scale"])
    idx_d, w_d = torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda()
    A = shape.num_tokens * shape.top_k
    I = shape.inter
    nw = (I // 128) * gp.layout["scale_rows"]

    gp.forward(topk_idx=idx_d, topk_weights=w_d)
    assert gp.status() == 0
    q_fused = gp.ws_region("act_q", torch.uint8, A * I).clone()
    s_fused = gp.ws_region("act_s", torch.int32, nw).clone().view(-1, gp.layout["scale_rows"])[:, :A]

    gp.workspace.zero_()
    h = gp.moe.debug_unfused_gate_up(gp.cfg, gp.d.x, idx_d, gp.weights, gp.workspace, w13_bias=gp.d.w13_bias)
    torch.cuda.synchronize()
    assert gp.status() == 0
    q_un = gp.ws_region("act_q", torch.uint8, A * I)
    s_un = gp.ws_region("act_s", torch.int32, nw).view(-1, gp.layout["scale_rows"])[:, :A]
    assert torch.isfinite(h).all()
    assert torch.equal(q_fused, q_un), f"{name}: act codes differ in {(q_fused != q_un).sum().item()} bytes"
    assert torch.equal(s_fused, s_un), f"{name}: act scales differ"


def test_unfused_h_matches_the_oracle_pre_activation():
    """The stored h is the grouped GEMM's promoted gate/up sum: for the routed rows of a few
    tokens, SwiGLU of h (fp64, host) lies within one E4M3 code step of the oracle's requantized
    act (its codes times its scales)."""
    shape = synth.Shape("uf_h", 64, 256, 256, 4, 2, renormalize=1, seed=73)
    prob = synth.make_problem(shape)
    gp = GpuProblem(prob)
    ni = prob.numpy_inputs()
    idx, w, _ = oracle.route(oracle_cfg(shape), ni["logits"], None)
    h = gp.moe.debug_unfused_gate_up(gp.cfg, gp.d.x, torch.from_numpy(idx).cuda(), gp.weights,
                                     gp.workspace).double().cpu().numpy()
    _, _, _, row_of = oracle.permute(idx, shape.num_experts)
    I = shape.inter
    # transformed column r holds original column (I if up else 0) + 128 j + i, r = 256 j + 128 up + i
    r = np.arange(2 * I)
    orig = np.where((r // 128) & 1, I, 0) + 128 * (r // 256) + r % 128
    hh = np.empty_like(h)
    hh[:, orig] = h
    tok = np.arange(8)
    _, rq, rs = oracle.forward(oracle_cfg(shape), ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"],
                               topk_idx=idx, topk_weights=w, tokens=tok, want_act=True)
    for t in tok:
        for j in range(shape.top_k):
            g, u = hh[row_of[t, j], :I], hh[row_of[t, j], I:]
            act = g / (1.0 + np.exp(-g)) * u
            sc = np.repeat(rs[t, j].astype(np.float64), 128)
            deq = torch.from_numpy(np.ascontiguousarray(rq[t, j])).view(torch.float8_e4m3fn).double().numpy() * sc
            tol = 2.0 ** -3 * np.abs(deq) + 2.0 ** -9 * sc + 1e-6
            assert np.all(np.abs(act - deq) <= tol), (t, j, float(np.max(np.abs(act - deq) - tol)))
