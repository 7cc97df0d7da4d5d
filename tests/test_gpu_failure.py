"""Failure detection on the GPU without a fault: a bounded device-side wait that runs out is
reported through the device status word, and the context stays usable afterwards."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, ensure_built, max_abs_rel, to_device, to_np
from nested_mamba2_selective_b200 import MatMambaError, mm_device_status, mm_selftest_wait_timeout, ssd_scan, synth

pytestmark = pytest.mark.gpu

MM_ERR_SHAPE, MM_ERR_TIMEOUT = 2, 7


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def test_wait_that_runs_out_sets_timeout_status_and_context_survives(orc):
    assert mm_device_status() == 0
    mm_selftest_wait_timeout(20000)  # a 20 ms limit on a barrier nothing arrives on
    assert mm_device_status() == MM_ERR_TIMEOUT
    assert mm_device_status() == 0  # reading the word clears it
    # the next call on the same context runs and is correct
    inp = synth.long_memory(synth.ssd_inputs(1, 300, 4, 64, 128, 1, "bf16", seed=209))
    g = dict(x=to_device(inp["x"], "bf16"), B=to_device(inp["B"], "bf16"), C=to_device(inp["C"], "bf16"),
             dt=torch.from_numpy(inp["dt"]).cuda(), A=torch.from_numpy(inp["A"]).cuda(),
             D=torch.from_numpy(inp["D"]).cuda())
    y = ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk=256)
    torch.cuda.synchronize()
    assert mm_device_status() == 0
    ref, _ = orc.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])
    assert max_abs_rel(to_np(y), ref) <= TOL["bf16"]
