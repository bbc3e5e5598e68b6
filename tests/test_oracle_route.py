"""Pins for the oracle's routing (CPU only).

Sources: "MindIE-SD Fused MoE" -- parameter table (top_k in [1, num_experts]; group_count,
k_group, group_select_mode, routing_method, renormalize, routed_scaling_factor), routing
selection (grouped routing constraints; sigmoid outputs normalized weights) and the custom
routing function example (softmax -> topk -> renormalize); "mlx_native ops/moe_gate.rs"
(top-K, softmax over the selected, per_expert_scale).

The pins: the custom routing example re-run with torch (a library definition), an exhaustive
search over expert and group subsets on tiny inputs, closed-form weight identities, and the
pages' constraint lists as negative cases.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle


def cfg(**kw):
    base = dict(num_tokens=1, hidden=128, inter=128, num_experts=8, top_k=2)
    base.update(kw)
    return oracle.Config(**base)


def test_softmax_matches_custom_routing_example():
    """softmax -> topk -> renormalize, as the page's custom routing function does it."""
    rng = np.random.default_rng(0)
    T, E, K = 300, 64, 6
    logits = rng.standard_normal((T, E)).astype(np.float32)
    for renorm in (0, 1):
        c = cfg(num_tokens=T, num_experts=E, top_k=K, renormalize=renorm)
        idx, w, _ = oracle.route(c, logits)
        g = torch.from_numpy(logits).double()
        r = g.softmax(dim=-1).topk(K, dim=-1)
        tw, ti = r.values, r.indices
        if renorm:
            tw = tw / tw.sum(dim=-1, keepdim=True)
        assert np.array_equal(idx, ti.numpy().astype(np.int32))
        assert np.allclose(w, tw.numpy(), rtol=0, atol=1e-7)


def test_decode_reading_topk_then_softmax():
    """moe_gate: top-K by score, then softmax over the selected logits, then per-expert scale;
    equal to softmax routing with renormalize."""
    rng = np.random.default_rng(1)
    T, E, K = 50, 128, 8
    logits = rng.standard_normal((T, E)).astype(np.float32)
    pes = (rng.random(E) + 0.5).astype(np.float32)
    idx, w, _ = oracle.route(cfg(num_tokens=T, num_experts=E, top_k=K, renormalize=1), logits, pes)
    sel = np.take_along_axis(logits, idx, 1).astype(np.float64)
    ref = torch.from_numpy(sel).softmax(-1).numpy() * pes[idx]
    assert np.allclose(w, ref, rtol=0, atol=2e-7)


def _key_order(vals):
    return sorted(range(len(vals)), key=lambda e: (-vals[e], e))


def test_exhaustive_subsets_tiny():
    """On tiny inputs with deliberate ties, the chosen set is the k-subset whose sorted
    (value desc, index asc) keys are lexicographically best among ALL k-subsets."""
    rng = np.random.default_rng(2)
    for trial in range(200):
        E = int(rng.integers(1, 8))
        K = int(rng.integers(1, E + 1))
        l = rng.integers(-2, 3, E).astype(np.float32)          # many ties
        idx, _, _ = oracle.route(cfg(num_experts=E, top_k=K), l[None, :])
        best = None
        for sub in itertools.combinations(range(E), K):
            key = sorted(((-l[e], e) for e in sub))
            if best is None or key < best[0]:
                best = (key, sub)
        expect = [e for _, e in best[0]]
        assert list(idx[0]) == expect


def _group_scores_fp32(s, G, mode):
    s = torch.from_numpy(s.astype(np.float32)).reshape(G, -1)
    if mode == 0:
        return s.max(dim=-1).values.numpy()
    return s.topk(2, dim=-1).values.sum(dim=-1).numpy()


@pytest.mark.parametrize("routing", [0, 1])
@pytest.mark.parametrize("mode", [0, 1])
def test_grouped_routing_exhaustive(routing, mode):
    rng = np.random.default_rng(3 + routing + 2 * mode)
    E, G = 16, 4
    for trial in range(100):
        kg = int(rng.integers(1, G + 1))
        K = int(rng.integers(1, kg * (E // G) + 1))
        l = rng.standard_normal(E).astype(np.float32)
        c = cfg(num_experts=E, top_k=K, routing=routing, group_count=G, k_group=kg,
                group_select_mode=mode, renormalize=1)
        idx, w, tie = oracle.route(c, l[None, :])
        if routing == 1:
            s = torch.sigmoid(torch.from_numpy(l)).numpy()
        else:
            s = torch.from_numpy(l).softmax(-1).numpy()
        gsc = _group_scores_fp32(s, G, mode)
        if tie[0]:
            continue
        # exhaustive over group subsets: best is the lexicographically best sorted key list
        best = min(itertools.combinations(range(G), kg),
                   key=lambda sub: sorted((-gsc[g], g) for g in sub))
        eligible = [e for g in best for e in range(g * (E // G), (g + 1) * (E // G))]
        expect = sorted(eligible, key=lambda e: (-l[e], e))[:K]
        assert list(idx[0]) == expect


def test_sigmoid_weights_normalized_and_scaled():
    rng = np.random.default_rng(4)
    T, E, K = 100, 256, 8
    logits = (rng.standard_normal((T, E)) + rng.normal(0, 0.1, E)).astype(np.float32)
    c = cfg(num_tokens=T, num_experts=E, top_k=K, routing=1, group_count=8, k_group=4,
            group_select_mode=1, renormalize=1, routed_scaling_factor=2.5)
    idx, w, _ = oracle.route(c, logits)
    assert np.allclose(w.sum(1), 2.5, rtol=1e-6)
    s = 1 / (1 + np.exp(-np.take_along_axis(logits, idx, 1).astype(np.float64)))
    assert np.allclose(w, 2.5 * s / s.sum(1, keepdims=True), rtol=0, atol=1e-6)
    # the k experts are distinct, in descending logit order
    for t in range(T):
        assert len(set(idx[t])) == K
        sel = logits[t, idx[t]]
        assert np.all(sel[:-1] >= sel[1:])
        # all selected experts lie in at most k_group groups
        assert len(set(idx[t] // 32)) <= 4


def test_softmax_without_renormalize_gives_full_probabilities():
    rng = np.random.default_rng(5)
    T, E, K = 40, 256, 8
    logits = rng.standard_normal((T, E)).astype(np.float32)
    idx, w, _ = oracle.route(cfg(num_tokens=T, num_experts=E, top_k=K), logits)
    p = torch.from_numpy(logits).double().softmax(-1).numpy()
    assert np.allclose(w, np.take_along_axis(p, idx, 1), rtol=0, atol=1e-8)
    assert np.all(w.sum(1) < 1.0)


def test_per_expert_scale_and_rsf_applied_last():
    rng = np.random.default_rng(6)
    T, E, K = 30, 32, 4
    logits = rng.standard_normal((T, E)).astype(np.float32)
    pes = (rng.random(E) + 0.5).astype(np.float32)
    base = cfg(num_tokens=T, num_experts=E, top_k=K, renormalize=1)
    i0, w0, _ = oracle.route(base, logits)
    i1, w1, _ = oracle.route(oracle.Config(**{**base.__dict__, "routed_scaling_factor": 3.0}),
                             logits, pes)
    assert np.array_equal(i0, i1)
    assert np.allclose(w1, w0.astype(np.float64) * pes[i0] * 3.0, rtol=1e-6, atol=0)


def test_ties_go_to_lower_index_in_descending_slots():
    l = np.array([[1.0, 3.0, 3.0, 2.0, 3.0]], np.float32)
    idx, _, _ = oracle.route(cfg(num_experts=5, top_k=4), l)
    assert list(idx[0]) == [1, 2, 4, 3]


@pytest.mark.parametrize("kw,rc", [
    (dict(top_k=0), oracle.EINVAL),
    (dict(top_k=9), oracle.EINVAL),                       # top_k in [1, num_experts]
    (dict(num_experts=0), oracle.EINVAL),
    (dict(hidden=192), oracle.EUNSUPPORTED),              # hidden % 128 (MATE Current Limits)
    (dict(inter=64), oracle.EUNSUPPORTED),
    (dict(group_count=3), oracle.EUNSUPPORTED),           # num_experts % group_count
    (dict(group_count=2, k_group=3), oracle.EUNSUPPORTED),  # k_group in [1, group_count]
    (dict(group_count=4, k_group=1, top_k=3), oracle.EUNSUPPORTED),  # top_k > experts in groups
    (dict(num_experts=8, group_count=8, group_select_mode=1), oracle.EUNSUPPORTED),  # >= 2 / group
    (dict(num_experts=257, top_k=1), oracle.EUNSUPPORTED),
])
def test_constraints(kw, rc):
    assert oracle.check_cfg(cfg(**kw)) == rc


def test_valid_configs_accepted():
    assert oracle.check_cfg(cfg()) == oracle.OK
    assert oracle.check_cfg(cfg(num_experts=256, top_k=8, group_count=8, k_group=4,
                                group_select_mode=1, hidden=7168, inter=2048)) == oracle.OK
