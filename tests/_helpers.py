"""Shared helpers for the parity tests: run the CUDA path through the C ABI and the oracle on
the same seeded inputs, and compare.

Tolerance on the layer output y (bf16), from the fp8 arithmetic: the kernels accumulate in fp32
where the oracle uses fp64, so a requantized E4M3 code can flip by one step where the SwiGLU
product sits on a rounding boundary; y is rounded to bf16 on both sides.  Accepted when
    max |y - r| <= 2e-2 * rms(r)   and   sum |y - r| / sum |r| <= 5e-3.
Routing weights: |w - w_ref| <= 2e-6 * max(1, |w_ref|) (fp32 exp/sum order differ).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

Y_MAX_REL_RMS = 2e-2
Y_MEAN_REL = 5e-3
W_TOL = 2e-6


def y_metrics(y_bits: np.ndarray, r_bits: np.ndarray) -> dict:
    y = oracle.bf16_bits_to_f32(y_bits).astype(np.float64)
    r = oracle.bf16_bits_to_f32(r_bits).astype(np.float64)
    d = np.abs(y - r)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    return dict(max_abs=float(d.max()) if d.size else 0.0, rms=rms,
                max_rel_rms=float(d.max() / rms) if rms > 0 else 0.0,
                mean_rel=float(d.sum() / max(np.abs(r).sum(), 1e-300)),
                bit_equal_frac=float(np.mean(y_bits == r_bits)) if d.size else 1.0,
                finite=bool(np.all(np.isfinite(y))))


def assert_y_close(y_bits, r_bits, what=""):
    m = y_metrics(y_bits, r_bits)
    assert m["finite"], f"{what}: non-finite output"
    assert m["max_rel_rms"] <= Y_MAX_REL_RMS, f"{what}: {m}"
    assert m["mean_rel"] <= Y_MEAN_REL, f"{what}: {m}"
    return m


def oracle_cfg(shape: synth.Shape) -> oracle.Config:
    return oracle.Config(**shape.cfg())


def lib_cfg(shape: synth.Shape):
    import mixture_experts_fp8_b200 as moe
    return moe.Config(**shape.cfg())


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


class GpuProblem:
    """A problem on cuda:0 with transformed weights and a workspace."""

    def __init__(self, prob: synth.Problem, device="cuda"):
        import mixture_experts_fp8_b200 as moe
        self.moe = moe
        self.prob = prob
        self.shape = prob.shape
        self.cfg = lib_cfg(prob.shape)
        self.d = prob.to(device) if prob.x.device.type != "cuda" else prob
        self.weights = moe.transform_weights(self.cfg, self.d.w13, self.d.w13_scale, self.d.w2,
                                             self.d.w2_scale)
        self.workspace = moe.new_workspace(self.cfg, device)
        self.workspace.zero_()
        self.layout = moe.workspace_layout(self.cfg)

    def forward(self, topk_idx=None, topk_weights=None, x=None, logits=None, cfg=None, workspace=None,
                expert_counts=None):
        d = self.d
        cfg = cfg or self.cfg
        x = d.x if x is None else x
        if topk_idx is None:
            logits = d.logits if logits is None else logits
        y = self.moe.forward(cfg, x, self.weights, router_logits=logits if topk_idx is None else None,
                             per_expert_scale=d.per_expert_scale if topk_idx is None else None,
                             topk_idx=topk_idx, topk_weights=topk_weights, w13_bias=d.w13_bias,
                             w2_bias=d.w2_bias, workspace=self.workspace if workspace is None else workspace,
                             expert_counts=expert_counts)
        torch.cuda.synchronize()
        return y

    def ws_region(self, name, dtype, count):
        off = self.layout[name]
        nbytes = count * torch.tensor([], dtype=dtype).element_size()
        return self.workspace[off:off + nbytes].view(dtype)

    def ws_scales(self, name, kdim):
        """Scales of workspace region `name` (stored [kdim/128][scale_rows] 4-byte words) as
        [A, kdim/g]: fp32 for recipe 0, UE8M0 bytes for recipe 1."""
        SR = self.layout["scale_rows"]
        nb = kdim // 128
        A = self.shape.num_tokens * (self.shape.top_k + self.shape.shared_experts)
        words = self.ws_region(name, torch.int32, nb * SR).cpu().numpy().reshape(nb, SR)[:, :A]
        if self.shape.recipe == 0:
            return np.ascontiguousarray(words.view(np.float32).T)
        b = np.ascontiguousarray(words).view(np.uint8).reshape(nb, A, 4)
        return np.ascontiguousarray(b.transpose(1, 0, 2).reshape(A, nb * 4))

    def status(self) -> int:
        return self.moe.read_status(self.workspace)


def oracle_inputs(prob: synth.Problem) -> dict:
    return prob.numpy_inputs()


def oracle_y(prob: synth.Problem, ni: dict, tokens=None, topk_idx=None, topk_w=None):
    c = oracle_cfg(prob.shape)
    if topk_idx is not None:
        return oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"], topk_idx=topk_idx,
                              topk_weights=topk_w, b13=ni["b13"], b2=ni["b2"], tokens=tokens)
    return oracle.forward(c, ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"], logits=ni["logits"],
                          per_expert_scale=ni["per_expert_scale"], b13=ni["b13"], b2=ni["b2"], tokens=tokens)


def check_routing(shape, ni, idx_gpu: np.ndarray, w_gpu: np.ndarray):
    """Expert ids bit-exact, except tokens the oracle flags as near ties in the group choice;
    for those the GPU's ids must be a valid selection (distinct, descending logits)."""
    c = oracle_cfg(shape)
    idx, w, tie = oracle.route(c, ni["logits"], ni["per_expert_scale"])
    same = np.all(idx == idx_gpu, axis=1)
    bad = np.where(~same & (tie == 0))[0]
    assert bad.size == 0, f"routing differs on {bad.size} tokens, first {bad[:5]}"
    m = same
    tol = W_TOL * np.maximum(1.0, np.abs(w[m]))
    dw = np.abs(w_gpu[m] - w[m])
    assert np.all(dw <= tol), f"routing weights differ by up to {dw.max()}"
    for t in np.where(~same)[0]:
        ids = idx_gpu[t]
        assert len(set(ids.tolist())) == shape.top_k
        sel = ni["logits"][t, ids]
        assert np.all(sel[:-1] >= sel[1:])
    return int((~same).sum()), int(tie.sum())
