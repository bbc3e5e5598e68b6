"""Expert parallelism on the CPU: the oracle's two sides of the exchange pinned to closed forms,
then the exchange logic of mixture_experts_fp8_b200.ep run by two gloo ranks with the oracle's
steps, bit-identical to the single-process oracle forward ("MindIE-SD Fused MoE", execution
flow: dispatch, mlp, combine; the dynamic dispatcher's all-to-all)."""
import json
import os
import socket
from dataclasses import asdict, replace

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth



def _ocfg(cfg) -> oracle.Config:
    return oracle.Config(**asdict(cfg))


# ------------------------------------------------------------------------------ oracle pins
@pytest.mark.parametrize("recipe", [0, 1, 2])
def test_expert_rows_with_zero_down_weights_is_the_down_bias(recipe):
    """W2 = 0: every row's output is its own expert's b2, exactly, whatever x and W13 are
    (pins the row -> expert indexing and the bias)."""
    shape = synth.Shape("eprows", 6, 256, 128, 4, 1, recipe=recipe, biases=True, seed=50)
    ni = synth.make_problem(shape).numpy_inputs()
    w2 = np.zeros_like(ni["w2"])
    e = np.array([3, 0, 2, 2, 1, 3], np.int32)
    o = oracle.expert_rows(oracle.Config(**shape.cfg()), ni["x"], e, ni["w13"], ni["w13s"], w2, ni["w2s"],
                           ni["b13"], ni["b2"])
    b2 = oracle.bf16_bits_to_f32(ni["b2"]).astype(np.float64)
    assert np.array_equal(o, b2[e])


def test_expert_rows_rejects_an_expert_outside_the_rank():
    shape = synth.Shape("eprows", 2, 256, 128, 4, 1, seed=51)
    ni = synth.make_problem(shape).numpy_inputs()
    with pytest.raises(ValueError):
        oracle.expert_rows(oracle.Config(**shape.cfg()), ni["x"], np.array([0, 4], np.int32), ni["w13"],
                           ni["w13s"], ni["w2"], ni["w2s"])


def test_combine_rows_closed_form():
    """Rows of small integers and power-of-two weights: every sum is exact and fits bf16, so y is
    known exactly; positions may come in any order."""
    T, K, H = 3, 2, 8
    o = np.arange(T * K * H, dtype=np.float64).reshape(T * K, H) % 7 - 3
    pos = np.array([[5, 0], [3, 4], [1, 2]], np.int32)
    w = np.array([[0.5, 0.25], [1.0, 2.0], [0.125, 4.0]], np.float32)
    y = oracle.combine_rows(o, pos, w)
    exact = np.stack([w[t, 0] * o[pos[t, 0]] + w[t, 1] * o[pos[t, 1]] for t in range(T)]).astype(np.float32)
    assert np.array_equal(oracle.bf16_bits_to_f32(y), exact)


# ------------------------------------------------------------------------------ exchange logic
class OracleOps:
    """The device steps of ep.ep_step done by the oracle (rows in fp64, y as bf16 bits)."""

    rows_dtype = "float64"

    def route(self, cfg, logits, pes):
        idx, w, _ = oracle.route(_ocfg(cfg), logits.numpy(), None if pes is None else pes.numpy())
        return torch.from_numpy(idx), torch.from_numpy(w)

    def dispatch(self, cfg, ranks, x, topk_idx, workspace):
        idx = topk_idx.numpy().reshape(-1)
        e_loc = cfg.num_experts // ranks
        dest = idx // e_loc
        order = np.argsort(dest, kind="stable")               # send order: by rank, then slot
        counts = np.bincount(dest, minlength=ranks).astype(np.int32)
        pos = np.empty_like(order)
        pos[order] = np.arange(order.size)
        send_x = x[torch.from_numpy(order // cfg.top_k)]
        send_e = torch.from_numpy((idx[order] % e_loc).astype(np.int32))
        return (torch.from_numpy(counts), send_x, send_e,
                torch.from_numpy(pos.astype(np.int32).reshape(cfg.num_tokens, cfg.top_k)))

    def rows(self, cfg_rows, rows, expert_of_row, weights_local, b13, b2):
        x = rows.view(torch.int16).numpy().view(np.uint16)
        o = oracle.expert_rows(_ocfg(cfg_rows), x, expert_of_row.numpy(), *weights_local, b13, b2)
        return torch.from_numpy(o)

    def combine(self, cfg, o_rows, slot_pos, topk_weights, status=None):
        return torch.from_numpy(oracle.combine_rows(o_rows.numpy(), slot_pos.numpy(), topk_weights.numpy()))

    def new_workspace(self, cfg, device):
        return None


CASES = {
    # softmax top-2 over 8 experts
    "softmax": synth.Shape("ep_sm", 32, 256, 128, 8, 2, renormalize=1, seed=52),
    # sigmoid with 4 groups of 4 (keep 2), per-expert scale, biases, MXFP8
    "groups": synth.Shape("ep_grp", 24, 256, 128, 16, 4, routing=1, renormalize=1, group_count=4, k_group=2,
                          group_select_mode=1, routed_scaling_factor=2.5, recipe=1, per_expert_scale=True,
                          biases=True, seed=53),
    # every token prefers rank 0's experts: rank 1 receives no rows
    "one_sided": synth.Shape("ep_one", 16, 256, 128, 8, 2, renormalize=1, logit_bias_std=0.0, seed=54),
}


def _problem(name):
    shape = CASES[name]
    prob = synth.make_problem(shape)
    if name == "one_sided":       # logits of experts 4..7 far below the rest
        prob.logits[:, 4:] -= 100.0
    return shape, prob


def _rank(rank, world, port, name, out_dir):
    import datetime

    import torch.distributed as dist

    import mixture_experts_fp8_b200 as moe
    from mixture_experts_fp8_b200 import ep

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        shape, prob = _problem(name)
        ni = prob.numpy_inputs()
        T = shape.num_tokens // world                              # this rank's tokens
        sl = slice(rank * T, (rank + 1) * T)
        e_loc = shape.num_experts // world
        es = slice(rank * e_loc, (rank + 1) * e_loc)
        cfg = replace(moe.Config(**shape.cfg()), num_tokens=T)
        local = (ni["w13"][es], ni["w13s"][es], ni["w2"][es], ni["w2s"][es])
        b13 = None if ni["b13"] is None else ni["b13"][es]
        b2 = None if ni["b2"] is None else ni["b2"][es]
        y, stats = ep.ep_step(cfg, world, prob.x[sl].contiguous(), prob.logits[sl].contiguous(), local, dist,
                              ops=OracleOps(), per_expert_scale=prob.per_expert_scale, w13_bias_local=b13,
                              w2_bias_local=b2)
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y.numpy())
        with open(os.path.join(out_dir, f"s{rank}.json"), "w") as f:
            json.dump(stats, f)
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("name", list(CASES))
def test_two_rank_exchange_matches_the_single_process_forward(name, tmp_path):
    mp.spawn(_rank, args=(2, _free_port(), name, str(tmp_path)), nprocs=2, join=True)
    shape, prob = _problem(name)
    ni = prob.numpy_inputs()
    ref = oracle.forward(oracle.Config(**shape.cfg()), ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"],
                         logits=ni["logits"], per_expert_scale=ni["per_expert_scale"], b13=ni["b13"], b2=ni["b2"])
    y = np.concatenate([np.load(tmp_path / f"y{r}.npy") for r in range(2)])
    assert np.array_equal(y, ref)
    stats = [json.load(open(tmp_path / f"s{r}.json")) for r in range(2)]
    T = shape.num_tokens // 2
    assert all(sum(s["sent"]) == T * shape.top_k for s in stats)
    # what rank a sends to rank b is what rank b receives from rank a
    assert all(stats[a]["sent"][b] == stats[b]["received"][a] for a in range(2) for b in range(2))
    if name == "one_sided":
        assert sum(stats[1]["received"]) == 0


def test_one_rank_with_the_benchmark_local_exchange():
    """World size 1 (what bench.py --ep runs without torchrun): every row stays home, through
    bench.LocalExchange; the result is the single-process forward."""
    import bench

    import mixture_experts_fp8_b200 as moe
    from mixture_experts_fp8_b200 import ep

    shape, prob = _problem("groups")
    ni = prob.numpy_inputs()
    cfg = moe.Config(**shape.cfg())
    y, stats = ep.ep_step(cfg, 1, prob.x, prob.logits, (ni["w13"], ni["w13s"], ni["w2"], ni["w2s"]),
                          bench.LocalExchange(), ops=OracleOps(), per_expert_scale=prob.per_expert_scale,
                          w13_bias_local=ni["b13"], w2_bias_local=ni["b2"])
    ref = oracle.forward(oracle.Config(**shape.cfg()), ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"],
                         logits=ni["logits"], per_expert_scale=ni["per_expert_scale"], b13=ni["b13"], b2=ni["b2"])
    assert np.array_equal(y.numpy(), ref)
    assert stats["sent"] == stats["received"] == [shape.num_tokens * shape.top_k]


def test_library_ops_keep_one_growing_expert_side_workspace():
    """The expert side's workspace is kept across steps: reused while the step's problem fits,
    replaced by a larger one when it does not, never shrunk (host logic, a fake library)."""
    from mixture_experts_fp8_b200 import ep

    class FakeMoe:
        def __init__(self):
            self.made = []

        def workspace_size(self, cfg):
            return 1000 * cfg.num_tokens

        def new_workspace(self, cfg, device):
            ws = torch.empty(self.workspace_size(cfg), dtype=torch.uint8, device=device)
            self.made.append(ws.numel())
            return ws

    import mixture_experts_fp8_b200 as moe
    cfg = moe.Config(**synth.SHAPES["tiny"].cfg())
    fake = FakeMoe()
    ops = ep.LibraryOps(fake)
    sizes = [ops.rows_workspace(ep.rows_config(cfg, 1, n), "cpu").numel() for n in [40, 12, 40, 64, 8, 64]]
    assert fake.made == [40000, 64000]
    assert sizes == [40000, 40000, 40000, 64000, 64000, 64000]
