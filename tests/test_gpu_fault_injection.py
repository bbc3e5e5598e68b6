"""Failure detection inside the GEMMs, without a GPU fault: the debug library
(libmoefp8_debug.so, the same sources built with MOE_FAULT_INJECTION) drops the first K stage of
the gate+up GEMM's producer in CTA 0 when a fault is armed from the host.  The MMA role's bounded
wait then runs out; every role leaves, the status word reads MOE_ERR_TIMEOUT, and the next call
works.  One problem per GEMM kernel: narrow (swap-AB), wide, MXFP8.  The injected runs happen in a
child process that loads the debug library; with no fault armed, that library's output must equal
the release library's bit for bit."""
import json
import os
import subprocess
import sys
import numpy as np
import pytest

import synth
from _helpers import GpuProblem, bits

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (kernel the library picks, shape)
CASES = [
    ("narrow", synth.Shape("fi_narrow", 16, 256, 256, 8, 2, renormalize=1, seed=5)),
    ("wide", synth.Shape("fi_wide", 300, 256, 256, 2, 2, renormalize=1, seed=6, biases=True)),
    ("mx", synth.Shape("fi_mx", 64, 256, 256, 8, 2, renormalize=1, recipe=1, seed=7)),
]

CHILD = r"""
import json, sys, numpy as np, torch
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
import mixture_experts_fp8_b200 as moe
from mixture_experts_fp8_b200 import build as b
moe.LIB_PATH = b.build(debug=True)
import synth
from _helpers import GpuProblem, bits
out = {}
for name, fields in CASES:
    gp = GpuProblem(synth.make_problem(synth.Shape(**fields)))
    y0 = bits(gp.forward()); s0 = gp.status()
    moe.debug_inject_fault(moe.MOE_FAULT_SKIP_STAGE)
    gp.forward(); s1 = gp.status()
    y2 = bits(gp.forward()); s2 = gp.status()
    np.save(OUTDIR + "/" + name + ".npy", y0)
    out[name] = [s0, s1, s2, bool(np.array_equal(y0, y2))]
print(json.dumps(out))
"""


def test_injected_stage_loss_times_out_and_recovers(tmp_path):
    cases = [(n, s.__dict__) for n, s in CASES]
    code = f"ROOT = {ROOT!r}\nOUTDIR = {str(tmp_path)!r}\nCASES = {cases!r}\n" + CHILD
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    import mixture_experts_fp8_b200 as moe
    for name, shape in CASES:
        s0, s1, s2, same = res[name]
        assert s0 == 0, name                         # debug library, no fault armed
        assert s1 == moe.MOE_ERR_TIMEOUT, name       # the armed fault is detected, not hung
        assert s2 == 0 and same, name                # the next call is clean and identical
        # the release library (this process) gives the same bits as the debug library
        y_rel = bits(GpuProblem(synth.make_problem(shape)).forward())
        assert np.array_equal(y_rel, np.load(tmp_path / f"{name}.npy")), name


def test_release_library_refuses_fault_injection():
    import mixture_experts_fp8_b200 as moe
    with pytest.raises(moe.MoeError) as e:
        moe.debug_inject_fault(moe.MOE_FAULT_SKIP_STAGE)
    assert e.value.code == moe.MOE_ERR_UNSUPPORTED
