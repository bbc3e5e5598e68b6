"""Expert parallelism through the library on one GPU ("MindIE-SD Fused MoE", execution flow:
dispatch, mlp, combine).  The dispatch plan is checked bit for bit against a stable sort by
destination rank.  Then R ranks are emulated in one process: each routes its own tokens and
dispatches them, the all-to-all is a copy of row blocks on the device, each computes the rows it
received with its own experts' weights, the rows go back, and each combines.  Every rank's y must
equal the single-GPU forward of the whole problem on those tokens, bit for bit (a row's result
depends only on its own codes and its expert's weights), and must match the oracle's forward of
those tokens within the layer's tolerance; each rank's expert-side rows must match the oracle's
expert_rows on the rows it received.  No kernel waits on another: the ranks run one after the
other.  An expert id out of range is reported, not sent, and adds nothing in the combine."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import Y_MAX_REL_RMS, Y_MEAN_REL, assert_y_close, bits, oracle_y

pytestmark = pytest.mark.gpu

SHAPES = {
    "tiny_r0": synth.Shape("ep_tiny", 32, 256, 256, 8, 2, renormalize=1, biases=True, seed=60),
    "groups_mx": synth.Shape("ep_grp", 48, 512, 256, 32, 4, routing=1, renormalize=1, group_count=4, k_group=2,
                             group_select_mode=1, routed_scaling_factor=2.5, recipe=1, per_expert_scale=True,
                             seed=61),
    "w4a8": synth.Shape("ep_w4", 40, 512, 256, 16, 4, renormalize=1, recipe=2, biases=True, seed=62),
    "decode": synth.SHAPES["decode"],
}


def _lib():
    import mixture_experts_fp8_b200 as moe
    return moe


@pytest.mark.parametrize("ranks", [1, 2, 4])
def test_dispatch_plan_matches_a_stable_sort_by_rank(ranks):
    moe = _lib()
    shape = SHAPES["decode"]
    d = synth.make_problem(shape).to("cuda")
    cfg = moe.Config(**shape.cfg())
    ws = moe.new_workspace(cfg, "cuda")
    idx, _ = moe.route(cfg, d.logits, per_expert_scale=d.per_expert_scale)
    counts, send_x, send_e, slot_pos = moe.ep_dispatch(cfg, ranks, d.x, idx, ws)
    torch.cuda.synchronize()
    assert moe.read_status(ws) == moe.MOE_OK
    flat = idx.cpu().numpy().reshape(-1)
    e_loc = shape.num_experts // ranks
    order = np.argsort(flat // e_loc, kind="stable")
    assert np.array_equal(counts.cpu().numpy(), np.bincount(flat // e_loc, minlength=ranks))
    assert np.array_equal(send_e.cpu().numpy(), flat[order] % e_loc)
    pos = np.empty_like(order)
    pos[order] = np.arange(order.size)
    assert np.array_equal(slot_pos.cpu().numpy().reshape(-1), pos)
    xs = d.x.view(torch.int16).cpu().numpy()
    assert np.array_equal(send_x.view(torch.int16).cpu().numpy(), xs[order // shape.top_k])


def _emulate(shape, ranks):
    """y of every emulated rank, and the single-GPU forward of the whole problem."""
    moe = _lib()
    prob = synth.make_problem(shape)
    d = prob.to("cuda")
    full = moe.Config(**shape.cfg())
    ws_full = moe.new_workspace(full, "cuda")
    w_full = moe.transform_weights(full, d.w13, d.w13_scale, d.w2, d.w2_scale)
    y_ref = moe.forward(full, d.x, w_full, router_logits=d.logits, per_expert_scale=d.per_expert_scale,
                        w13_bias=d.w13_bias, w2_bias=d.w2_bias, workspace=ws_full)

    T = shape.num_tokens // ranks
    E_loc = shape.num_experts // ranks
    cfg = replace(full, num_tokens=T)
    plans = []
    for r in range(ranks):                                     # each rank: route + dispatch
        sl = slice(r * T, (r + 1) * T)
        ws = moe.new_workspace(cfg, "cuda")
        idx, w = moe.route(cfg, d.logits[sl].contiguous(), per_expert_scale=d.per_expert_scale)
        counts, send_x, send_e, slot_pos = moe.ep_dispatch(cfg, ranks, d.x[sl].contiguous(), idx, ws)
        torch.cuda.synchronize()
        assert moe.read_status(ws) == moe.MOE_OK
        plans.append(dict(w=w, counts=counts.cpu().tolist(), send_x=send_x, send_e=send_e, slot_pos=slot_pos))
    starts = [np.concatenate([[0], np.cumsum(p["counts"])]) for p in plans]
    sides = []                                                 # (rank, rows, local ids, o) per expert side
    o_back = [torch.empty((T * shape.top_k, shape.hidden), dtype=torch.float32, device="cuda") for _ in plans]
    for q in range(ranks):                                     # each rank: the rows sent to it
        blocks = [(r, int(starts[r][q]), int(starts[r][q + 1])) for r in range(ranks)]
        rows = torch.cat([plans[r]["send_x"][a:b] for r, a, b in blocks])
        rows_e = torch.cat([plans[r]["send_e"][a:b] for r, a, b in blocks])
        n = rows.shape[0]
        if n == 0:
            continue
        es = slice(q * E_loc, (q + 1) * E_loc)
        from mixture_experts_fp8_b200.ep import rows_config
        cq = rows_config(cfg, ranks, n)
        wq = moe.transform_weights(cq, d.w13[es].contiguous(), d.w13_scale[es].contiguous(), d.w2[es].contiguous(),
                                   d.w2_scale[es].contiguous())
        ws_q = moe.new_workspace(cq, "cuda")
        o = moe.forward_rows(cq, rows.contiguous(), rows_e.contiguous(), wq,
                             w13_bias=None if d.w13_bias is None else d.w13_bias[es].contiguous(),
                             w2_bias=None if d.w2_bias is None else d.w2_bias[es].contiguous(), workspace=ws_q)
        torch.cuda.synchronize()
        assert moe.read_status(ws_q) == moe.MOE_OK
        sides.append((q, rows, rows_e, o))
        off = 0
        for r, a, b in blocks:                                 # back to the senders' positions
            o_back[r][a:b] = o[off:off + (b - a)]
            off += b - a
    ys = []
    for r in range(ranks):                                     # each rank: combine
        ys.append(moe.combine_rows(cfg, o_back[r], plans[r]["slot_pos"], plans[r]["w"]))
    torch.cuda.synchronize()
    return torch.cat(ys), y_ref, prob, sides


@pytest.mark.parametrize("name,ranks", [("tiny_r0", 1), ("tiny_r0", 2), ("groups_mx", 4), ("w4a8", 2),
                                        ("decode", 2), ("decode", 8)])
def test_emulated_ranks_match_the_single_gpu_forward(name, ranks):
    y, y_ref, _, _ = _emulate(SHAPES[name], ranks)
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))


@pytest.mark.parametrize("name,ranks", [("tiny_r0", 2), ("groups_mx", 4), ("w4a8", 2), ("decode", 8)])
def test_emulated_ranks_match_the_oracle(name, ranks):
    """Every rank's y against the oracle's forward of the same tokens, and every expert side's
    rows against the oracle's expert_rows on the rows that rank received."""
    shape = SHAPES[name]
    y, _, prob, sides = _emulate(shape, ranks)
    ni = prob.numpy_inputs()
    assert_y_close(bits(y), oracle_y(prob, ni), f"{name} over {ranks} ranks")
    E_loc = shape.num_experts // ranks
    ocfg = oracle.Config(**shape.cfg())
    for q, rows, rows_e, o in sides:
        es = slice(q * E_loc, (q + 1) * E_loc)
        c = replace(ocfg, num_tokens=int(rows.shape[0]), top_k=1, num_experts=E_loc, routing=0, renormalize=0,
               group_count=1, k_group=1, group_select_mode=0, routed_scaling_factor=1.0)
        ref = oracle.expert_rows(c, rows.view(torch.int16).cpu().numpy().view(np.uint16), rows_e.cpu().numpy(),
                                 ni["w13"][es], ni["w13s"][es], ni["w2"][es], ni["w2s"][es],
                                 None if ni["b13"] is None else ni["b13"][es],
                                 None if ni["b2"] is None else ni["b2"][es])
        got = o.double().cpu().numpy()
        d = np.abs(got - ref)
        rms = float(np.sqrt(np.mean(ref * ref)))
        assert d.max() <= Y_MAX_REL_RMS * rms, (name, q, d.max() / rms)
        assert d.sum() / np.abs(ref).sum() <= Y_MEAN_REL, (name, q)


def test_out_of_range_expert_is_reported_not_sent_and_adds_nothing():
    """An expert id outside [0, E): the dispatch reports MOE_ERR_BOUNDS, does not send the slot and
    leaves its position at -1; the combine over the rows that did come back adds nothing for it
    and reports it in the status word it is given."""
    moe = _lib()
    shape = SHAPES["tiny_r0"]
    d = synth.make_problem(shape).to("cuda")
    cfg = moe.Config(**shape.cfg())
    ws = moe.new_workspace(cfg, "cuda")
    idx, w = moe.route(cfg, d.logits)
    idx[3, 1] = shape.num_experts + 5                          # token 3, slot 1: no such expert
    counts, send_x, send_e, slot_pos = moe.ep_dispatch(cfg, 2, d.x, idx, ws)
    torch.cuda.synchronize()
    assert moe.read_status(ws) == moe.MOE_ERR_BOUNDS
    A = shape.num_tokens * shape.top_k
    assert int(counts.sum()) == A - 1
    assert int(slot_pos[3, 1]) == -1
    n = A - 1
    o = torch.ones((n, shape.hidden), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    w1 = torch.ones_like(w)
    y = moe.combine_rows(cfg, o, slot_pos, w1, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == moe.MOE_ERR_BOUNDS
    yf = y.float().cpu()
    assert torch.all(yf[3] == 1.0)                             # only slot 0's row of ones
    assert torch.all(yf[torch.arange(shape.num_tokens) != 3] == float(shape.top_k))


def test_forward_rows_rejects_more_than_one_slot():
    moe = _lib()
    cfg = moe.Config(num_tokens=4, hidden=256, inter=256, num_experts=4, top_k=2)
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    e = torch.zeros(4, dtype=torch.int32, device="cuda")
    w = tuple(torch.zeros(n, dtype=torch.uint8, device="cuda") for n in moe.transformed_weights_size(cfg))
    with pytest.raises(moe.MoeError):
        moe.forward_rows(cfg, x, e, w)


class _OneRank:
    """The all-to-all of a single rank: every row stays home."""

    @staticmethod
    def all_to_all_single(out, inp, out_splits=None, in_splits=None, group=None):
        out.copy_(inp)


@pytest.mark.parametrize("name", ["tiny_r0", "w4a8"])
def test_ep_step_through_the_library_ops_equals_the_forward(name):
    """ep_step with its default device steps (the library ops, which keep one expert-side
    workspace from call to call) at one rank: the same bits as the fused forward, for the whole
    batch and then for a smaller one through the kept workspace."""
    moe = _lib()
    from mixture_experts_fp8_b200 import ep
    shape = SHAPES[name]
    d = synth.make_problem(shape).to("cuda")
    full = moe.Config(**shape.cfg())
    w = moe.transform_weights(full, d.w13, d.w13_scale, d.w2, d.w2_scale)
    for T in (shape.num_tokens, shape.num_tokens // 2, shape.num_tokens):
        cfg = replace(full, num_tokens=T)
        x, logits = d.x[:T].contiguous(), d.logits[:T].contiguous()
        y_ep, stats = ep.ep_step(cfg, 1, x, logits, w, _OneRank(), per_expert_scale=d.per_expert_scale,
                                 w13_bias_local=d.w13_bias, w2_bias_local=d.w2_bias)
        y_f = moe.forward(cfg, x, w, router_logits=logits, per_expert_scale=d.per_expert_scale,
                          w13_bias=d.w13_bias, w2_bias=d.w2_bias)
        torch.cuda.synchronize()
        assert stats["sent"] == [T * shape.top_k] and stats["received"] == [T * shape.top_k]
        assert torch.equal(y_ep.view(torch.int16), y_f.view(torch.int16)), f"{name}, {T} tokens"
    kept = ep._library_ops()._rows_ws
    assert len(kept) == 1
    need = moe.workspace_size(ep.rows_config(full, 1, shape.num_tokens * shape.top_k))
    assert next(iter(kept.values())).numel() >= need
