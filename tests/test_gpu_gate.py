"""Parity of the fused gate (RMSNorm + router matmul + router top-k, "mlx_native
ops/moe_gate.rs") against the oracle: logits within fp32-vs-fp64 accumulation error, the top-k
bit-exact against the oracle's router run on the GPU's own logits, and against the oracle's gate
except where two candidate logits lie within that error; logits independent of the batch; the
gate's routing feeds the layer exactly as router logits do; the weight transform (norm weight
folded into the router rows, split into three bf16 parts) bit for bit against torch on the CPU."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import GpuProblem, bits, check_routing, oracle_cfg

pytestmark = pytest.mark.gpu

CASES = {
    "decode": synth.SHAPES["decode"],                                         # softmax, per-expert scale
    "prefill64": synth.SHAPES["prefill"].with_tokens(64),                     # sigmoid, groups, H 7168
    "small": synth.Shape("gsmall", 37, 384, 128, 24, 3, renormalize=1, seed=42),
}
LOGIT_TOL = 3e-5          # |gpu - oracle| relative to max |logit|: fp32 sums over H terms


class _Acts:
    """The gate's inputs only (no expert weights): x, per-expert scale, and their numpy view."""

    def __init__(self, shape):
        self.x, _, self.per_expert_scale = synth.make_activations(shape)

    def numpy_inputs(self):
        return dict(x=self.x.view(torch.int16).numpy().view(np.uint16), logits=None,
                    per_expert_scale=None if self.per_expert_scale is None else self.per_expert_scale.numpy())


def _gate_inputs(shape, full=False):
    prob = synth.make_problem(shape) if full else _Acts(shape)
    nw, rw, eps = synth.make_gate(shape)
    return prob, nw, rw, eps


def _gate_weights(cfg, nw, rw):
    import mixture_experts_fp8_b200 as moe
    return moe.transform_gate_weights(cfg, nw.cuda(), rw.cuda())


@pytest.mark.parametrize("name", list(CASES))
def test_gate_logits_and_routing(name):
    import mixture_experts_fp8_b200 as moe
    shape = CASES[name]
    prob, nw, rw, eps = _gate_inputs(shape)
    ni = prob.numpy_inputs()
    cfg = moe.Config(**shape.cfg())
    x = prob.x.cuda()
    pes = None if prob.per_expert_scale is None else prob.per_expert_scale.cuda()
    lg, idx, w = moe.gate(cfg, x, _gate_weights(cfg, nw, rw), eps, per_expert_scale=pes)
    torch.cuda.synchronize()
    lg = lg.cpu().numpy()
    ref = oracle.gate_logits(ni["x"], nw.numpy(), rw.numpy(), eps)
    err = np.max(np.abs(lg - ref)) / np.max(np.abs(ref))
    assert err <= LOGIT_TOL, err
    # the router on the GPU's own logits: exactly the oracle's router on them
    gni = dict(ni, logits=lg)
    check_routing(shape, gni, idx.cpu().numpy(), w.cpu().numpy())
    # against the oracle's gate: equal except where the k-th and (k+1)-th choices are closer
    # than the logit error
    ridx, _, tie = oracle.route(oracle_cfg(shape), ref, ni["per_expert_scale"])
    gidx = idx.cpu().numpy()
    diff = np.where(np.any(ridx != gidx, axis=1))[0]
    for t in diff:
        s = np.sort(ref[t])[::-1]
        close = np.min(np.abs(np.diff(s))) <= 4 * LOGIT_TOL * np.max(np.abs(ref))
        assert close or tie[t], f"token {t}: routing differs without a near tie"
    assert diff.size <= max(1, shape.num_tokens // 50)


def test_gate_logits_do_not_depend_on_the_batch():
    import mixture_experts_fp8_b200 as moe
    shape = CASES["small"]
    prob, nw, rw, eps = _gate_inputs(shape)
    cfg = moe.Config(**shape.cfg())
    x = prob.x.cuda()
    gw = _gate_weights(cfg, nw, rw)
    lg, _, _ = moe.gate(cfg, x, gw, eps)
    sel = torch.tensor([36, 0, 5, 5, 17], device="cuda")
    cs = moe.Config(**replace(shape, num_tokens=5).cfg())
    ls, _, _ = moe.gate(cs, x[sel].contiguous(), gw, eps)
    torch.cuda.synchronize()
    assert torch.equal(ls, lg[sel])


def test_gate_routing_drives_the_layer_like_router_logits():
    import mixture_experts_fp8_b200 as moe
    shape = CASES["decode"]
    prob, nw, rw, eps = _gate_inputs(shape, full=True)
    gp = GpuProblem(prob)
    lg, idx, w = moe.gate(gp.cfg, gp.d.x, _gate_weights(gp.cfg, nw, rw), eps,
                          per_expert_scale=gp.d.per_expert_scale)
    y1 = bits(gp.forward(topk_idx=idx, topk_weights=w))
    y2 = bits(gp.forward(logits=lg))
    assert gp.status() == 0
    assert np.array_equal(y1, y2)


def test_gate_logits_same_for_any_batch_size():
    """A 2400-token batch runs 19 token tiles in several waves of clusters, a 4-token batch one
    tile: every logit is still the same eight shares of H added in the same order, so a token's
    logits are bit-identical either way."""
    import mixture_experts_fp8_b200 as moe
    shape = synth.Shape("gtiles", 2400, 256, 128, 256, 8, renormalize=1, seed=43)
    prob, nw, rw, eps = _gate_inputs(shape)
    cfg = moe.Config(**shape.cfg())
    x = prob.x.cuda()
    gw = _gate_weights(cfg, nw, rw)
    lg, _, _ = moe.gate(cfg, x, gw, eps)
    sel = torch.tensor([2399, 0, 1234, 7], device="cuda")
    cs = moe.Config(**replace(shape, num_tokens=4).cfg())
    ls, _, _ = moe.gate(cs, x[sel].contiguous(), gw, eps)
    torch.cuda.synchronize()
    assert torch.equal(ls, lg[sel])
    ref = oracle.gate_logits(prob.numpy_inputs()["x"][[2399, 0, 1234, 7]], nw.numpy(), rw.numpy(), eps)
    assert np.max(np.abs(ls.cpu().numpy() - ref)) / np.max(np.abs(ref)) <= LOGIT_TOL


@pytest.mark.parametrize("E,H", [(24, 384), (256, 7168)])
def test_gate_weight_transform_bits(E, H):
    """w' = fl32(norm_w * router_w) and its parts hi = rn_bf16(w'), mid = rn_bf16(w' - hi),
    lo = rn_bf16(w' - hi - mid), against the same three roundings done by torch on the CPU."""
    import mixture_experts_fp8_b200 as moe
    shape = synth.Shape("gsplit", 4, H, 128, E, 2, renormalize=1, seed=44)
    nw, rw, _ = synth.make_gate(shape)
    cfg = moe.Config(**shape.cfg())
    gw = _gate_weights(cfg, nw, rw)
    torch.cuda.synchronize()
    got = gw.cpu().view(torch.bfloat16).view(3, E, H)
    w = nw[None, :] * rw                                  # one fp32 rounding per element
    hi = w.to(torch.bfloat16)
    r1 = w - hi.float()
    mid = r1.to(torch.bfloat16)
    lo = (r1 - mid.float()).to(torch.bfloat16)
    for q, ref in enumerate((hi, mid, lo)):
        assert torch.equal(got[q].view(torch.int16), ref.view(torch.int16)), q
    # the parts carry w' to within 2^-24 of its magnitude
    back = hi.double() + mid.double() + lo.double()
    assert torch.all((back - w.double()).abs() <= w.double().abs() * 2.0 ** -24)


def test_gate_handles_every_tail():
    """T not a multiple of the 128-token tile, E not a multiple of the 64-expert tile, and H with
    fewer 64-column steps than the cluster has CTAs (some shares are empty)."""
    import mixture_experts_fp8_b200 as moe
    shape = synth.Shape("gtail", 129, 384, 128, 72, 4, renormalize=1, seed=45)
    prob, nw, rw, eps = _gate_inputs(shape)
    cfg = moe.Config(**shape.cfg())
    lg, idx, w = moe.gate(cfg, prob.x.cuda(), _gate_weights(cfg, nw, rw), eps)
    torch.cuda.synchronize()
    ref = oracle.gate_logits(prob.numpy_inputs()["x"], nw.numpy(), rw.numpy(), eps)
    lg = lg.cpu().numpy()
    assert np.all(np.isfinite(lg))
    assert np.max(np.abs(lg - ref)) / np.max(np.abs(ref)) <= LOGIT_TOL
    check_routing(shape, dict(prob.numpy_inputs(), logits=lg), idx.cpu().numpy(), w.cpu().numpy())
