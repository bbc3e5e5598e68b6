"""moe_forward_static_workspace: the forward for callers that may not allocate device memory.

Some callers run inside a host framework that owns every byte of device memory (a serving
engine's pre-reserved pool, or a plugin interface that hands its kernels no scratch buffer);
they cannot call cudaMalloc, which can synchronize the device and can fail under memory pressure.
This entry point takes the same inputs and outputs as moe_forward but keeps its scratch in a
fixed 16 MiB array inside the library.  Its output must match moe_forward's (same kernels) within
the tolerance the other parity tests use, on two calls in a row (the array keeps the previous
call's contents).  This file is named to be collected last, and passes alone or after the rest.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_fp8_b200 as moe
import synth
from _helpers import GpuProblem, assert_y_close, bits

pytestmark = pytest.mark.gpu


def _call(gp, y):
    """Call the new entry point directly through the C ABI."""
    c = gp.cfg.c()
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    d = gp.d
    rc = moe.lib().moe_forward_static_workspace(
        ctypes.byref(c), P(d.x), P(d.logits), P(d.per_expert_scale), None, None,
        *[P(w) for w in gp.weights], P(d.w13_bias), P(d.w2_bias), P(y), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc


@pytest.mark.parametrize("name", ["decode", "tiny"])
def test_static_workspace_matches_moe_forward_twice(name):
    gp = GpuProblem(synth.make_problem(name))
    ref = bits(gp.forward())
    for _ in range(2):
        y = torch.full((gp.shape.num_tokens, gp.shape.hidden), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call(gp, y) == moe.MOE_OK, moe.lib().moe_last_error()
        assert_y_close(bits(y), ref, f"{name} static workspace")


def test_static_workspace_rejects_problems_that_do_not_fit():
    gp = GpuProblem(synth.make_problem(synth.SHAPES["tiny"].with_tokens(16)))
    big = moe.Config(**{**gp.cfg.__dict__, "num_tokens": 4096, "top_k": 8, "hidden": 2048})
    assert moe.workspace_size(big) > 16 << 20
    c = big.c()
    rc = moe.lib().moe_forward_static_workspace(ctypes.byref(c), *([ctypes.c_void_p(16)] * 13), None)
    assert rc == moe.MOE_ERR_UNSUPPORTED
    assert b"16777216" in moe.lib().moe_last_error()
