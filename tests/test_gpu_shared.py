"""Parity of the shared expert (one more expert, index num_experts, that every token uses with
weight 1; "metrale_model_layers fp8_grouped_tc_w8a8.rs", run_fp8_grouped_w8a8) against the
oracle: the permutation with the shared slot bit for bit, and y within the layer tolerance, on
every GEMM kernel (narrow, wide, MXFP8), both permutation paths, and 256 routed experts plus the
shared one.  Plus a plumbing check: a shared expert whose down projection is zero leaves y's bits
as they are without it."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import GpuProblem, assert_y_close, bits, oracle_cfg, oracle_inputs, oracle_y

pytestmark = pytest.mark.gpu

_E257 = synth.Shape("e257", 512, 512, 256, 256, 8, routing=1, renormalize=1, group_count=8, k_group=4,
                    group_select_mode=1, routed_scaling_factor=2.5, logit_bias_std=0.1, seed=33,
                    shared_experts=1)
CASES = {
    "tiny_sh": replace(synth.SHAPES["tiny"], name="tiny_sh", shared_experts=1),               # narrow
    "decode_sh": replace(synth.SHAPES["decode"], name="decode_sh", shared_experts=1),         # narrow, full size
    "wide_sh": synth.Shape("wide_sh", 300, 256, 256, 2, 2, renormalize=1, biases=True, seed=31,
                           shared_experts=1),                                                   # wide
    "mx_sh": synth.Shape("mx_sh", 96, 256, 384, 8, 2, renormalize=1, recipe=1, biases=True, seed=32,
                         shared_experts=1),                                                     # MXFP8, swap-AB
    "w4_sh": synth.Shape("w4_sh", 96, 256, 384, 8, 2, renormalize=1, recipe=2, biases=True, seed=34,
                         shared_experts=1),                                                     # W4A8, swap-AB
    "w4_sh_wide": synth.Shape("w4_sh_wide", 400, 256, 384, 8, 2, renormalize=1, recipe=2, biases=True,
                              seed=35, shared_experts=1),                                       # W4A8, wide
    "e257_narrow": _E257,                                                                       # 3-kernel permute
    "e257_wide": replace(_E257, name="e257_wide", num_tokens=2048),                             # 3-kernel, wide
}


@pytest.fixture(scope="module")
def problems():
    cache = {}

    def get(name):
        if name not in cache:
            prob = synth.make_problem(CASES[name])
            cache[name] = (GpuProblem(prob), oracle_inputs(prob), prob)
        return cache[name]
    return get


def _slots(idx: np.ndarray, E: int) -> np.ndarray:
    """[T, k] routed ids -> [T, k + 1] slot experts, the shared expert (E) last."""
    return np.concatenate([idx, np.full((idx.shape[0], 1), E, idx.dtype)], axis=1)


@pytest.mark.parametrize("name", list(CASES))
def test_shared_permutation_bit_exact(problems, name):
    gp, ni, _ = problems(name)
    s = gp.shape
    T, E = s.num_tokens, s.num_experts
    A = T * (s.top_k + 1)
    idx, w, _ = oracle.route(oracle_cfg(s), ni["logits"], ni["per_expert_scale"])
    counts_out = torch.zeros(E + 1, dtype=torch.int32, device="cuda")
    gp.forward(topk_idx=torch.from_numpy(idx).cuda(), topk_weights=torch.from_numpy(w).cuda(),
               expert_counts=counts_out)
    assert gp.status() == 0
    counts, offsets, row_src, row_of = oracle.permute(_slots(idx, E), E + 1)
    assert counts[E] == T
    assert np.array_equal(counts_out.cpu().numpy(), counts)
    assert np.array_equal(gp.ws_region("offsets", torch.int32, E + 2).cpu().numpy(), offsets)
    assert np.array_equal(gp.ws_region("row_src", torch.int32, A).cpu().numpy(), row_src)
    assert np.array_equal(gp.ws_region("row_of", torch.int32, A).cpu().numpy(), row_of.ravel())
    tiles = gp.ws_region("tile_start", torch.int32, E + 2).cpu().numpy()
    assert np.array_equal(np.diff(tiles), (counts + 127) // 128)


@pytest.mark.parametrize("name", list(CASES))
def test_shared_forward_matches_oracle(problems, name):
    gp, ni, prob = problems(name)
    T = gp.shape.num_tokens
    y = bits(gp.forward())
    assert gp.status() == 0
    tok = np.arange(T, dtype=np.int32) if T <= 96 else np.linspace(0, T - 1, 96).astype(np.int32)
    r = oracle_y(prob, ni, tokens=tok)
    assert_y_close(y[tok], r, name)


@pytest.mark.parametrize("name", ["tiny_sh", "wide_sh", "mx_sh", "w4_sh", "w4_sh_wide"])
def test_zero_shared_down_projection_keeps_bits(problems, name):
    """Shared expert with w2 = 0 (and no biases): y has the bits of the layer without it."""
    s = replace(CASES[name], biases=False)
    p1 = synth.make_problem(s)
    p1.w2[s.num_experts].zero_()
    y1 = bits(GpuProblem(p1).forward())
    y0 = bits(GpuProblem(synth.make_problem(replace(s, shared_experts=0))).forward())
    assert np.array_equal(y0, y1)
