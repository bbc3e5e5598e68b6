"""Pins for the oracle's gate in front of the router (CPU only).

Source: "mlx_native ops/moe_gate.rs": one pass per token does RMS-Norm of the bf16 hidden state
(learned fp32 norm weight, eps), the router matmul against fp32 router weights [E, hidden], then
top-K, softmax and per-expert scale.  The oracle computes the norm and the matmul in fp64 and
rounds the logits once to fp32; the routing is the router's own (pinned in test_oracle_route).

Pins: a torch fp64 RMSNorm + matmul, a closed form with one-hot router rows, scale invariance of
RMSNorm, and the eps term.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def _bf16(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_gate_matches_torch_fp64_rmsnorm_matmul():
    s = synth.Shape("g", 7, 384, 128, 24, 4, seed=40)
    p = synth.make_problem(s)
    nw, rw, eps = synth.make_gate(s)
    x = p.numpy_inputs()["x"]
    got = oracle.gate_logits(x, nw.numpy(), rw.numpy(), eps)
    xf = torch.from_numpy(oracle.bf16_bits_to_f32(x)).double()
    xn = xf * torch.rsqrt((xf * xf).mean(dim=1, keepdim=True) + eps) * nw.double()
    ref = (xn @ rw.double().T).float().numpy()
    assert got.shape == (7, 24)
    assert np.max(np.abs(got - ref)) <= 1e-6 * np.max(np.abs(ref))
    assert np.mean(got == ref) > 0.95          # same fp64 value rounded once to fp32


def test_one_hot_router_rows_give_normalized_inputs():
    """router_w[e] = one-hot at h = e: logits[t, e] = x[t, e] * w[e] / rms(x[t])."""
    H, E = 256, 16
    rng = np.random.default_rng(3)
    xv = rng.standard_normal((3, H)).astype(np.float32)
    x = _bf16(xv)
    xr = oracle.bf16_bits_to_f32(x).astype(np.float64)
    nw = (1.0 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    rw = np.zeros((E, H), np.float32)
    rw[np.arange(E), np.arange(E)] = 1.0
    got = oracle.gate_logits(x, nw, rw, 0.0)
    rms = np.sqrt(np.mean(xr * xr, axis=1, keepdims=True))
    ref = (xr[:, :E] / rms * nw[:E].astype(np.float64)).astype(np.float32)
    assert np.array_equal(got, ref)


def test_rmsnorm_scale_invariance_and_eps():
    H, E = 128, 8
    rng = np.random.default_rng(4)
    x = _bf16(rng.standard_normal((2, H)))
    x4 = _bf16(4.0 * oracle.bf16_bits_to_f32(x))            # exact in bf16 (power of two)
    nw = np.ones(H, np.float32)
    rw = rng.standard_normal((E, H)).astype(np.float32)
    a = oracle.gate_logits(x, nw, rw, 0.0)
    b = oracle.gate_logits(x4, nw, rw, 0.0)
    assert np.array_equal(a, b)
    # a large eps shrinks the logits: rms / sqrt(rms^2 + eps)
    xr = oracle.bf16_bits_to_f32(x).astype(np.float64)
    ms = np.mean(xr * xr, axis=1)
    c = oracle.gate_logits(x, nw, rw, 1.0)
    ratio = np.sqrt(ms / (ms + 1.0))
    assert np.allclose(c, a * ratio[:, None], rtol=1e-6, atol=1e-7)


def test_gate_routing_is_the_router_on_gate_logits():
    s = synth.Shape("gr", 9, 256, 128, 32, 4, renormalize=1, per_expert_scale=True, seed=41)
    p = synth.make_problem(s)
    ni = p.numpy_inputs()
    nw, rw, eps = synth.make_gate(s)
    lg = oracle.gate_logits(ni["x"], nw.numpy(), rw.numpy(), eps)
    assert 0.3 < float(np.std(lg)) < 3.0                     # logits of order one
    idx, w, _ = oracle.route(oracle.Config(**s.cfg()), lg, ni["per_expert_scale"])
    assert idx.shape == (9, 4) and np.all(w > 0)
