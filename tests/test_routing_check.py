"""The parity check's acceptance rule for near-tie group choices (CPU only).

"MindIE-SD Fused MoE", routing selection: with grouped routing the k_group best groups are kept
and top_k experts are chosen inside them.  When two groups score (almost) the same at the
k_group-th place, an fp32 implementation may keep either; the parity check then accepts the
GPU's ids only if they are the top_k of a tie-consistent group set, and their weights only if
they are the oracle's weights for those ids.  A constructed exact tie shows that the check
accepts the other tied group and rejects choices that a looser check (distinct ids in
descending logit order) would let through.
"""
import numpy as np
import pytest

import oracle
import synth
from _helpers import check_routing, near_tie_choice_ok

# 16 experts in 4 groups of 4, keep 2 groups, top-2, sigmoid with the group max as its score
SHAPE = synth.Shape("tie", 1, 128, 128, 16, 2, routing=1, renormalize=1, group_count=4, k_group=2,
                    group_select_mode=0)
# group 0 leads; groups 1 and 2 tie exactly at max logit 1.0; group 3 is clearly behind (0.9)
LOGITS = np.array([[3.0, -1.0, -1.0, -1.0,
                    1.0, 0.5, -1.0, -1.0,
                    -1.0, 1.0, 0.2, -1.0,
                    0.9, 0.8, -1.0, -1.0]], np.float32)


def _cfg():
    return oracle.Config(**SHAPE.cfg())


def _loose_ok(ids):
    """The looser rule: distinct ids in descending logit order."""
    sel = LOGITS[0, ids]
    return len(set(ids.tolist())) == len(ids) and bool(np.all(sel[:-1] >= sel[1:]))


def _check(ids, w=None):
    ids = np.array([ids], np.int32)
    if w is None:
        w = oracle.route_weights(_cfg(), LOGITS, ids)
    return check_routing(SHAPE, {"logits": LOGITS, "per_expert_scale": None}, ids, w)


def test_oracle_flags_the_tie_and_takes_the_lower_group():
    idx, _, tie = oracle.route(_cfg(), LOGITS)
    assert tie[0] == 1
    assert idx[0].tolist() == [0, 4]        # groups {0, 1}: the lower index wins the tie


def test_group_scores_are_the_sigmoid_group_max():
    g = oracle.group_scores(_cfg(), LOGITS)[0]
    s = 1.0 / (1.0 + np.exp(-LOGITS[0].astype(np.float64)))
    np.testing.assert_allclose(g, s.reshape(4, 4).max(axis=1), rtol=1e-6)


def test_route_weights_of_the_oracle_choice_equal_route():
    idx, w, _ = oracle.route(_cfg(), LOGITS)
    assert np.array_equal(oracle.route_weights(_cfg(), LOGITS, idx), w)


def test_other_tied_group_is_accepted():
    assert _check([0, 9]) == (1, 1)         # groups {0, 2}


@pytest.mark.parametrize("ids, why", [
    ([0, 12], "below"),                      # group 3 is not tied
    ([0, 10], "top_k"),                      # group 2, but not its best expert
    ([4, 9], "groups"),                      # leaves out the leading group 0
])
def test_invalid_choices_pass_the_loose_rule_but_are_rejected(ids, why):
    assert _loose_ok(np.array(ids))
    with pytest.raises(AssertionError, match=why):
        _check(ids)


def test_wrong_weights_for_a_valid_tied_choice_are_rejected():
    ids = np.array([[0, 9]], np.int32)
    w = oracle.route_weights(_cfg(), LOGITS, ids)
    w[0, 1] += 1e-4
    with pytest.raises(AssertionError, match="weights"):
        _check(ids[0].tolist(), w)


def test_choice_spanning_too_many_groups_is_rejected():
    # top-3 with k_group 2: experts from groups 0, 1 and 2 cannot come from 2 groups
    shape = synth.Shape("tie3", 1, 128, 128, 16, 3, routing=1, renormalize=1, group_count=4,
                        k_group=2, group_select_mode=0)
    c = oracle.Config(**shape.cfg())
    g = oracle.group_scores(c, LOGITS)[0]
    ok, why = near_tie_choice_ok(c, LOGITS[0], g, [0, 4, 9])
    assert not ok and "groups" in why
    ok, _ = near_tie_choice_ok(c, LOGITS[0], g, [0, 4, 9][:2] + [5])
    assert ok                               # groups {0, 1}: 0, 4, 5


def _closed_form_weights(logits, ids, routing, renormalize, pes, rsf):
    """The weight rule written out in fp64 ("MindIE-SD Fused MoE", routing parameters): softmax
    over every expert, or over the chosen ones when renormalized; sigmoid scores always divided by
    their sum; then the per-expert scale, then the routed scaling factor."""
    l = logits.astype(np.float64)
    if routing == 0:
        e = np.exp(l - l.max())
        w = e[ids] / (e[ids].sum() if renormalize else e.sum())
    else:
        s = 1.0 / (1.0 + np.exp(-l))
        w = s[ids] / s[ids].sum()
    if pes is not None:
        w = w * pes.astype(np.float64)[ids]
    return w * rsf


@pytest.mark.parametrize("routing,renormalize,use_pes,rsf", [
    (1, 1, False, 1.0), (1, 1, True, 2.5), (0, 1, False, 1.0), (0, 0, True, 1.0), (0, 1, True, 2.5)])
def test_route_weights_match_the_closed_form_for_a_choice_the_oracle_would_not_make(routing, renormalize,
                                                                                    use_pes, rsf):
    shape = synth.Shape("w", 1, 128, 128, 16, 3, routing=routing, renormalize=renormalize,
                        routed_scaling_factor=rsf)
    c = oracle.Config(**shape.cfg())
    pes = np.linspace(0.5, 1.5, 16).astype(np.float32) if use_pes else None
    ids = np.array([[9, 2, 13]], np.int32)          # not the top 3 of LOGITS
    w = oracle.route_weights(c, LOGITS, ids, pes)
    np.testing.assert_allclose(w[0], _closed_form_weights(LOGITS[0], ids[0], routing, renormalize, pes, rsf),
                               rtol=2e-6)


def test_group_scores_top2_sum():
    """group_select_mode 1: a group scores the sum of its two best sigmoid scores."""
    shape = synth.Shape("g1", 1, 128, 128, 16, 2, routing=1, renormalize=1, group_count=4, k_group=2,
                        group_select_mode=1)
    g = oracle.group_scores(oracle.Config(**shape.cfg()), LOGITS)[0]
    s = np.sort(1.0 / (1.0 + np.exp(-LOGITS[0].astype(np.float64))).reshape(4, 4), axis=1)
    np.testing.assert_allclose(g, s[:, -1] + s[:, -2], rtol=1e-6)
