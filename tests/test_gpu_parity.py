"""GPU parity: the CUDA path (called through the C ABI) against the oracle, on the same seeded
inputs, for every step of the layer.

  routing        expert ids bit-exact (near-tie group choices excepted and checked for
                 validity), weights within 2e-6
  permutation    counts, offsets, row_src, row_of bit-exact
  quantization   E4M3 codes and scales of every permuted row bit-exact
  output y       within the fp8 tolerance of tests/_helpers.py

Sizes: the tiny problem and small ragged problems in full (several tiles, ragged tails, empty
experts); the four full-size problems with routing, permutation and quantization in full and y
on seeded token samples (a row's bits do not depend on the other rows).  The W4A8 recipe (E2M1
weights) runs on the decode and prefill shapes, the small random problems and the edge shapes.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import (GpuProblem, assert_y_close, bits, check_routing, oracle_cfg, oracle_inputs,
                      oracle_y)

pytestmark = pytest.mark.gpu

FULL = ["tiny", "decode", "prefill", "skewed", "large", "decode_w4a8", "prefill_w4a8"]
SAMPLE_TOKENS = {"tiny": None, "decode": None, "skewed": 384, "prefill": 128, "large": 256,
                 "decode_w4a8": None, "prefill_w4a8": 128}
ON_GPU = ("prefill", "large", "prefill_w4a8")     # inputs drawn on the device (their size)


@pytest.fixture(scope="module")
def problems():
    cache = {}

    def get(name):
        if name not in cache:
            dev = "cuda" if name in ON_GPU else "cpu"
            prob = synth.make_problem(name, device=dev)
            gp = GpuProblem(prob)
            cache[name] = (gp, oracle_inputs(prob))
        return cache[name]
    return get


def _sample(T, n, seed):
    if n is None or n >= T:
        return None
    rng = np.random.default_rng(seed)
    s = np.sort(rng.choice(T, n, replace=False)).astype(np.int32)
    s[0], s[-1] = 0, T - 1
    return s


@pytest.mark.parametrize("name", FULL)
def test_routing(problems, name):
    gp, ni = problems(name)
    d = gp.d
    idx, w = gp.moe.route(gp.cfg, d.logits, d.per_expert_scale)
    torch.cuda.synchronize()
    nd, nt = check_routing(gp.shape, ni, idx.cpu().numpy(), w.cpu().numpy())
    print(f"{name}: {nd} tokens differ in routing (near ties flagged: {nt})")


@pytest.mark.parametrize("name", FULL)
def test_permutation_and_quantization(problems, name):
    gp, ni = problems(name)
    shape = gp.shape
    T, K, E, H = shape.num_tokens, shape.top_k, shape.num_experts, shape.hidden
    A = T * K
    # routing from the oracle, so the permutation is checked on exactly its input
    idx, w, _ = oracle.route(oracle_cfg(shape), ni["logits"], ni["per_expert_scale"])
    counts_out = torch.zeros(E, dtype=torch.int32, device="cuda")
    gp.forward(topk_idx=torch.from_numpy(idx).cuda(), topk_weights=torch.from_numpy(w).cuda(),
               expert_counts=counts_out)
    assert gp.status() == 0
    counts, offsets, row_src, row_of = oracle.permute(idx, E)
    assert np.array_equal(counts_out.cpu().numpy(), counts)
    assert np.array_equal(gp.ws_region("counts", torch.int32, E).cpu().numpy(), counts)
    assert np.array_equal(gp.ws_region("offsets", torch.int32, E + 1).cpu().numpy(), offsets)
    assert np.array_equal(gp.ws_region("row_src", torch.int32, A).cpu().numpy(), row_src)
    assert np.array_equal(gp.ws_region("row_of", torch.int32, A).cpu().numpy(), row_of.ravel())
    tiles = gp.ws_region("tile_start", torch.int32, E + 1).cpu().numpy()
    assert np.array_equal(np.diff(tiles), (counts + 127) // 128)

    # quantized activations, in permuted order
    xq = gp.ws_region("xq", torch.uint8, A * H).cpu().numpy().reshape(A, H)
    xs = gp.ws_scales("xs", H)
    tok = _sample(T, 512, 5)
    tok = np.arange(T) if tok is None else tok
    q_ref, s_ref = oracle.quantize_tokens(ni["x"][tok], shape.recipe)
    for j in range(K):
        rows = row_of[tok, j]
        assert np.array_equal(xq[rows], q_ref), f"E4M3 codes differ (slot {j})"
        assert np.array_equal(xs[rows], s_ref), f"scales differ (slot {j})"


@pytest.mark.parametrize("hidden", [128, 384, 640, 896])
@pytest.mark.parametrize("recipe", [0, 1])
def test_quantization_odd_widths(hidden, recipe):
    """Rows whose width is not a multiple of the quantizer's 256-column chunks (a half chunk at
    the end), several chunk pairs per row, and more routed slots than a warp has lanes: every
    permuted row's codes and scales bit for bit."""
    shape = synth.Shape("q_odd", 37, hidden, 128, 48, 40, renormalize=1, recipe=recipe, seed=81)
    prob = synth.make_problem(shape)
    gp = GpuProblem(prob)
    ni = oracle_inputs(prob)
    idx, w, _ = oracle.route(oracle_cfg(shape), ni["logits"], None)
    gp.forward(topk_idx=torch.from_numpy(idx).cuda(), topk_weights=torch.from_numpy(w).cuda())
    assert gp.status() == 0
    T, K, H = shape.num_tokens, shape.top_k, shape.hidden
    _, _, _, row_of = oracle.permute(idx, shape.num_experts)
    xq = gp.ws_region("xq", torch.uint8, T * K * H).cpu().numpy().reshape(T * K, H)
    xs = gp.ws_scales("xs", H)
    q_ref, s_ref = oracle.quantize_tokens(ni["x"], recipe)
    for j in range(K):
        assert np.array_equal(xq[row_of[:, j]], q_ref), f"codes differ (slot {j})"
        assert np.array_equal(xs[row_of[:, j]], s_ref), f"scales differ (slot {j})"


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "skewed", "large", "prefill_w4a8"])
def test_gate_up_swiglu_codes(problems, name):
    """The gate+up GEMM's requantized SwiGLU products (E4M3 codes and scales) against the
    oracle's, per routed row: codes may differ by one step where the fp32 and fp64 sums straddle a
    rounding boundary, so nearly all must be equal and none may differ by more than one code."""
    gp, ni = problems(name)
    shape = gp.shape
    T, K, I = shape.num_tokens, shape.top_k, shape.inter
    A = T * K
    idx, w, _ = oracle.route(oracle_cfg(shape), ni["logits"], ni["per_expert_scale"])
    gp.forward(topk_idx=torch.from_numpy(idx).cuda(), topk_weights=torch.from_numpy(w).cuda())
    _, _, _, row_of = oracle.permute(idx, shape.num_experts)
    aq = gp.ws_region("act_q", torch.uint8, A * I).cpu().numpy().reshape(A, I)
    as_ = gp.ws_scales("act_s", I)
    tok = _sample(T, 32, 3)
    tok = np.arange(min(T, 32)) if tok is None else tok
    _, rq, rs = oracle.forward(oracle_cfg(shape), ni["x"], ni["w13"], ni["w13s"], ni["w2"], ni["w2s"],
                               topk_idx=idx, topk_weights=w, b13=ni["b13"], b2=ni["b2"], tokens=tok,
                               want_act=True)
    gq = aq[row_of[tok]]                      # [n, K, I]
    gs = as_[row_of[tok]]
    eq = np.mean(gq == rq)
    dec = lambda c: torch.from_numpy(np.ascontiguousarray(c)).view(torch.float8_e4m3fn).float().numpy()
    print(f"{name}: act code equality {eq:.5f}")
    assert eq > 0.99, eq
    if shape.recipe == 0:
        assert np.allclose(gs, rs, rtol=1e-4, atol=0)
    else:
        assert np.mean(gs == rs) > 0.99
    # where codes differ they are neighbours
    diff = gq != rq
    if diff.any():
        a, b = dec(gq[diff]), dec(rq[diff])
        assert np.all(np.abs(a - b) <= np.maximum(np.abs(a), np.abs(b)) * 0.13 + 2.0 ** -9)


@pytest.mark.parametrize("name", FULL)
def test_forward_output(problems, name):
    gp, ni = problems(name)
    shape = gp.shape
    y = gp.forward()
    assert gp.status() == 0
    idx_g = gp.ws_region("topk_idx", torch.int32, shape.num_tokens * shape.top_k).cpu().numpy()
    w_g = gp.ws_region("topk_weights", torch.float32, shape.num_tokens * shape.top_k).cpu().numpy()
    idx_g = idx_g.reshape(shape.num_tokens, shape.top_k)
    w_g = w_g.reshape(shape.num_tokens, shape.top_k)
    tok = _sample(shape.num_tokens, SAMPLE_TOKENS[name], 11)
    # Near-tie tokens: the GPU's choice of experts must be valid (check_routing), and the oracle
    # then follows it.
    nd, nt = check_routing(shape, ni, idx_g, w_g)
    if nd:
        r = oracle_y(gp.prob, ni, tokens=tok, topk_idx=idx_g, topk_w=w_g)
    else:
        r = oracle_y(gp.prob, ni, tokens=tok)
    yb = bits(y)
    yb = yb if tok is None else yb[tok]
    m = assert_y_close(yb, r, name)
    print(f"{name}: {m}")


@pytest.mark.parametrize("seed,recipe", [(s, None) for s in range(8)] + [(s, 2) for s in range(8, 12)] +
                         [(s, "grouped") for s in range(12, 18)])
def test_forward_random_small(seed, recipe):
    if recipe == "grouped":
        shape = synth.random_grouped_shape(seed)
    else:
        shape = synth.random_shape(seed) if recipe is None else synth.random_shape(seed, recipe=recipe)
    prob = synth.make_problem(shape)
    gp = GpuProblem(prob)
    ni = oracle_inputs(prob)
    y = gp.forward()
    assert gp.status() == 0
    T, K = shape.num_tokens, shape.top_k
    idx_g = gp.ws_region("topk_idx", torch.int32, T * K).cpu().numpy().reshape(T, K)
    w_g = gp.ws_region("topk_weights", torch.float32, T * K).cpu().numpy().reshape(T, K)
    nd, _ = check_routing(shape, ni, idx_g, w_g)
    r = oracle_y(prob, ni, topk_idx=idx_g, topk_w=w_g) if nd else oracle_y(prob, ni)
    assert_y_close(bits(y), r, shape.name)


@pytest.mark.parametrize("over", [
    dict(num_tokens=1, num_experts=1, top_k=1),
    dict(num_tokens=300, num_experts=2, top_k=2),          # every expert > 2 row tiles
    dict(num_tokens=129, num_experts=1, top_k=1),           # ragged second row tile
    dict(num_tokens=40, num_experts=16, top_k=16),          # top_k = E
    dict(num_tokens=50, hidden=384, inter=640, num_experts=5, top_k=2),   # 3 K stages, odd N tiles
    dict(num_tokens=33, hidden=128, inter=128, num_experts=64, top_k=3),  # many empty experts
])
@pytest.mark.parametrize("recipe", [0, 1, 2])
def test_forward_edge_shapes(over, recipe):
    base = synth.Shape("edge", 8, 256, 256, 4, 2, renormalize=1, recipe=recipe, seed=77, biases=True)
    from dataclasses import replace
    shape = replace(base, **over)
    prob = synth.make_problem(shape)
    gp = GpuProblem(prob)
    y = gp.forward()
    assert gp.status() == 0
    assert_y_close(bits(y), oracle_y(prob, oracle_inputs(prob)), str(over))
