"""Failure detection on the GPU without a fault: bounded waits and bounds checks report through
the status word; the context stays usable afterwards."""
import numpy as np
import pytest
import torch

import mixture_experts_fp8_b200 as moe
import synth
from _helpers import GpuProblem, bits

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    st = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    moe.selftest_bounded_wait(st, 2000)
    torch.cuda.synchronize()
    assert int(st.item()) == moe.MOE_ERR_TIMEOUT
    # the context is still usable
    assert float(torch.ones(4, device="cuda").sum().item()) == 4.0


def test_out_of_range_expert_id_sets_bounds_status():
    gp = GpuProblem(synth.make_problem("tiny"))
    T, K = gp.shape.num_tokens, gp.shape.top_k
    idx, w = moe.route(gp.cfg, gp.d.logits)
    bad = idx.clone()
    bad[3, 1] = gp.shape.num_experts + 5        # checked on the device, never dereferenced
    bad[7, 0] = -2
    gp.forward(topk_idx=bad, topk_weights=w)
    assert gp.status() == moe.MOE_ERR_BOUNDS
    # a good call afterwards clears the status and works
    y = gp.forward(topk_idx=idx, topk_weights=w)
    assert gp.status() == 0
    assert np.all(np.isfinite(y.float().cpu().numpy()))


def test_invalid_arguments_launch_nothing():
    gp = GpuProblem(synth.make_problem("tiny"))
    with pytest.raises(moe.MoeError) as e:
        moe.forward(gp.cfg, gp.d.x, gp.weights, router_logits=gp.d.logits,
                    workspace=gp.workspace[: gp.workspace.numel() // 2])
    assert e.value.code == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError):
        moe.forward(gp.cfg, gp.d.x, gp.weights)                      # neither logits nor ids
