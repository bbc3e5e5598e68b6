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


GROUP_TIE_REL = 1e-5   # the oracle's near-tie band on group scores (relative)


def _better(l, a, b):
    """Is expert a ahead of expert b: larger logit, ties to the lower index."""
    return l[a] > l[b] or (l[a] == l[b] and a < b)


def _top_k_in(l, experts, k):
    """The k best of `experts` by (logit descending, index ascending)."""
    return sorted(experts, key=lambda e: (-float(l[e]), e))[:k]


def near_tie_choice_ok(cfg, l, gscore, ids):
    """Is `ids` a valid selection for one token whose group choice is a near tie?

    Valid means: some set S of k_group groups exists such that
      * every group clearly above the k_group-th best group score (outside the relative 1e-5
        band) is in S, and no group clearly below it is;
      * ids are exactly the top_k experts inside S, in descending logit order with ties to the
        lower index.
    Returns (ok, reason)."""
    E, G, K, kg = cfg.num_experts, cfg.group_count, cfg.top_k, cfg.k_group
    gs = E // G
    ids = [int(i) for i in ids]
    if len(set(ids)) != K or min(ids) < 0 or max(ids) >= E:
        return False, "ids not distinct or out of range"
    order = sorted(range(G), key=lambda g: (-float(gscore[g]), g))
    tau = float(gscore[order[kg - 1]])

    def band(g):
        return abs(float(gscore[g]) - tau) <= GROUP_TIE_REL * max(abs(float(gscore[g])), abs(tau))

    forced = {g for g in range(G) if float(gscore[g]) > tau and not band(g)}
    allowed = forced | {g for g in range(G) if band(g)}
    used = {e // gs for e in ids}
    if not used <= allowed:
        return False, f"groups {sorted(used - allowed)} score clearly below the k_group-th best"
    req = forced | used
    if len(req) > kg:
        return False, f"ids span {len(req)} groups with the forced ones, more than k_group={kg}"
    members = [e for g in req for e in range(g * gs, (g + 1) * gs)]
    if _top_k_in(l, members, K) != ids:
        return False, "ids are not the top_k (descending, ties to the lower index) of their groups"
    # fill S up to k_group groups from the band with groups none of whose experts would enter
    # the top_k (each loses to the k-th selected expert)
    fill = [g for g in sorted(allowed - req)
            if not any(_better(l, e, ids[-1]) for e in range(g * gs, (g + 1) * gs))]
    if len(req) + len(fill) < kg:
        return False, "no tie-consistent set of k_group groups yields these ids"
    return True, ""


def check_routing(shape, ni, idx_gpu: np.ndarray, w_gpu: np.ndarray):
    """Expert ids bit-exact, except on tokens the oracle flags as near ties in the group choice
    (their k_group-th and (k_group+1)-th fp32 group scores within 1e-5 relative).  For those the
    GPU's ids must be a tie-consistent selection (near_tie_choice_ok) and its weights must be the
    oracle's weights for the GPU's ids.  Weights of every other token within W_TOL of the oracle's.
    Returns (tokens whose ids differ from the oracle's, tokens the oracle flags)."""
    c = oracle_cfg(shape)
    logits = ni["logits"]
    idx, w, tie = oracle.route(c, logits, ni["per_expert_scale"])
    same = np.all(idx == idx_gpu, axis=1)
    bad = np.where(~same & (tie == 0))[0]
    assert bad.size == 0, f"routing differs on {bad.size} tokens, first {bad[:5]}"
    tol = W_TOL * np.maximum(1.0, np.abs(w[same]))
    dw = np.abs(w_gpu[same] - w[same])
    assert np.all(dw <= tol), f"routing weights differ by up to {dw.max()}"
    diff = np.where(~same)[0]
    if diff.size:
        gscore = oracle.group_scores(c, logits)
        for t in diff:
            ok, why = near_tie_choice_ok(c, logits[t], gscore[t], idx_gpu[t])
            assert ok, f"token {t}: GPU ids {idx_gpu[t].tolist()} invalid under the near tie: {why}"
        sub = shape.with_tokens(int(diff.size))
        pes = ni["per_expert_scale"]
        w_alt = oracle.route_weights(oracle_cfg(sub), logits[diff], idx_gpu[diff], pes)
        dw = np.abs(w_gpu[diff] - w_alt)
        assert np.all(dw <= W_TOL * np.maximum(1.0, np.abs(w_alt))), \
            f"near-tie tokens: weights differ from the oracle's weights of the GPU's ids by up to {dw.max()}"
    return int((~same).sum()), int(tie.sum())
