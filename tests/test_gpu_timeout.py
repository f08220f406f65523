"""Failure detection on the GPU without a GPU fault.

A debug flag makes the producer warp issue no loads, so the MMA and
promotion warps' bounded waits run out.  The kernel must then record
DG_ERR_TIMEOUT in the device status word and return (no hang, no trap), and
the CUDA context must stay usable: a normal call afterwards in the same
process still matches the oracle.  Runs in a child process because the wait
limit is read once per process from DG_WAIT_TIMEOUT_CYCLES (here ~2 ms).
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, time
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import torch, numpy as np
import moe_grouped_gemm_fp32_b200 as dg
import oracle, workloads as W
from gpu_util import DeviceProblem, compare, to_f64, valid_mask
dg.dg_get_device_status(clear=True)
for name, prob in [("swap+split", W.make_dense(128, 256, 512, seed=1)),
                   ("normal", W.make_dense(512, 512, 512, seed=2)),
                   ("masked", W.make_masked([3, 0, 70], 128, 256, 512, seed=3))]:
    dp = DeviceProblem(prob)
    dg.dg_debug_set_flags(1)
    t0 = time.time()
    dp.run()
    torch.cuda.synchronize()
    dt = time.time() - t0
    code = dg.dg_get_device_status(clear=True)
    assert code & 0xFF == 6, (name, hex(code))
    assert dt < 30, dt
    dg.dg_debug_set_flags(0)
    dp.run()
    torch.cuda.synchronize()
    compare(to_f64(dp.d), oracle.solve(prob), valid_mask(prob))
    assert dg.dg_get_device_status(clear=True) == 0
    print(name, "timeout reported", hex(code), "in %.3f s; recovered" % dt)
print("OK")
"""


def test_bounded_wait_reports_timeout_and_context_survives():
    env = dict(os.environ, DG_WAIT_TIMEOUT_CYCLES="4000000")
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "OK" in r.stdout
