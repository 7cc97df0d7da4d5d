"""GPU parity of the recurrent step (ssd_step) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, dims_of, ensure_built, make_block, max_abs_rel, to_device, to_np
from nested_mamba2_selective_b200 import matmamba_block_fwd, ssd_step, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_timeouts():
    yield
    from nested_mamba2_selective_b200 import mm_device_status
    assert mm_device_status() == 0, "a kernel's bounded wait gave up"
W = synth.WORKLOADS["decode_b256_1p4b"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


@pytest.fixture(scope="module")
def block():
    return make_block(W)


def states(batch, seed):
    dims = dims_of(W)
    return synth.states(batch, dims.nheads, W.d_head, W.d_state, W.d_inner + 2 * W.d_state, W.d_conv, "bf16", seed)


@pytest.mark.parametrize("m", [2048, 1024, 512])
def test_steps_match_oracle_and_leave_inactive_state(orc, block, m):
    wt, p64 = block
    dims = dims_of(W)
    s_np, c_np = states(4, seed=300 + m)
    s_gpu, c_gpu = torch.from_numpy(s_np).cuda(), to_device(c_np, "bf16")
    s_ref, c_ref = s_np.astype(np.float64), c_np.astype(np.float64)
    d, h = orc.width(dims, m)
    E = W.d_inner
    for step in range(3):
        u = synth.activations((4, W.d_model), "bf16", seed=310 + step)
        out = ssd_step(wt, s_gpu, c_gpu, to_device(u, "bf16"), m)
        torch.cuda.synchronize()
        ref = orc.block_step(dims, p64, u, m, s_ref, c_ref)
        assert max_abs_rel(to_np(out), ref) <= TOL["bf16"]
    assert max_abs_rel(to_np(s_gpu[:, :h]), s_ref[:, :h]) <= TOL["bf16"]
    active = list(range(d)) + list(range(E, E + 2 * W.d_state))
    assert max_abs_rel(to_np(c_gpu[:, active]), c_ref[:, active]) <= TOL["bf16"]
    np.testing.assert_array_equal(s_gpu[:, h:].cpu().numpy(), s_np[:, h:])
    np.testing.assert_array_equal(to_np(c_gpu[:, d:E]), c_np[:, d:E].astype(np.float64))


@pytest.mark.parametrize("m", [2048, 512])
def test_64_consecutive_steps_match_oracle(orc, block, m):
    """64 recurrent tokens in a row on 4 sequences from a prefilled random state: the state carried
    through the GPU's own updates stays on the oracle's trajectory (every step's output and the
    final states are compared)."""
    wt, p64 = block
    dims = dims_of(W)
    s_np, c_np = states(4, seed=340 + m)
    s_gpu, c_gpu = torch.from_numpy(s_np).cuda(), to_device(c_np, "bf16")
    s_ref, c_ref = s_np.astype(np.float64), c_np.astype(np.float64)
    d, h = orc.width(dims, m)
    us = synth.activations((64, 4, W.d_model), "bf16", seed=350 + m)
    worst = 0.0
    for step in range(64):
        out = ssd_step(wt, s_gpu, c_gpu, to_device(us[step], "bf16"), m)
        ref = orc.block_step(dims, p64, us[step], m, s_ref, c_ref)
        worst = max(worst, max_abs_rel(to_np(out), ref))
    assert worst <= TOL["bf16"], worst
    assert max_abs_rel(to_np(s_gpu[:, :h]), s_ref[:, :h]) <= TOL["bf16"]
    E = W.d_inner
    active = list(range(d)) + list(range(E, E + 2 * W.d_state))
    assert max_abs_rel(to_np(c_gpu[:, active]), c_ref[:, active]) <= TOL["bf16"]


def test_full_batch_step_sampled(orc, block):
    """256 sequences in one launch; the oracle checks three of them (sequences are independent)."""
    wt, p64 = block
    dims = dims_of(W)
    s_np, c_np = states(W.batch, seed=320)
    s_gpu, c_gpu = torch.from_numpy(s_np).cuda(), to_device(c_np, "bf16")
    u = synth.activations((W.batch, W.d_model), "bf16", seed=321)
    out = ssd_step(wt, s_gpu, c_gpu, to_device(u, "bf16"), 2048)
    torch.cuda.synchronize()
    rows = [0, 101, 255]
    s_ref, c_ref = s_np[rows].astype(np.float64), c_np[rows].astype(np.float64)
    ref = orc.block_step(dims, p64, u[rows], 2048, s_ref, c_ref)
    assert max_abs_rel(to_np(out[rows]), ref) <= TOL["bf16"]
    assert max_abs_rel(to_np(s_gpu[rows]), s_ref) <= TOL["bf16"]


@pytest.mark.parametrize("m", [2048, 512])
def test_prefill_then_step_equals_longer_prefill(block, m):
    wt, _ = block
    dims = dims_of(W)
    u = to_device(synth.activations((2, 201, W.d_model), "bf16", seed=330), "bf16")
    H, rows = dims.nheads, W.d_inner + 2 * W.d_state
    s = torch.zeros((2, H, 64, 128), device="cuda")
    c = torch.zeros((2, rows, 3), device="cuda", dtype=torch.bfloat16)
    matmamba_block_fwd(wt, u[:, :200].contiguous(), m, 256, ssm_state_out=s, conv_state_out=c)
    step = ssd_step(wt, s, c, u[:, 200].contiguous(), m)
    full = matmamba_block_fwd(wt, u, m, 256)
    torch.cuda.synchronize()
    assert max_abs_rel(to_np(step), to_np(full[:, 200])) <= TOL["bf16"]


def test_unaligned_conv_state_gives_the_same_steps(orc, block):
    """A conv state that starts 2 bytes past an 8-byte boundary takes the one-channel-per-thread roll
    instead of the vector one.  Both do the same arithmetic in the same order, so the conv and SSM
    states agree bit for bit; the outputs (summed over K slices in arrival order) both match the
    oracle."""
    wt, p64 = block
    dims = dims_of(W)
    m = 1024
    s_np, c_np = states(4, seed=377)
    runs = []
    for offset in (0, 1):
        buf = torch.zeros(c_np.size + 4, dtype=torch.bfloat16, device="cuda")
        c_gpu = buf[offset:offset + c_np.size].view(c_np.shape)
        c_gpu.copy_(to_device(c_np, "bf16"))
        s_gpu = torch.from_numpy(s_np).cuda()
        outs = []
        for step in range(3):
            u = synth.activations((4, W.d_model), "bf16", seed=380 + step)
            outs.append(ssd_step(wt, s_gpu, c_gpu, to_device(u, "bf16"), m))
        torch.cuda.synchronize()
        runs.append((torch.stack(outs), s_gpu, c_gpu.clone()))
    assert torch.equal(runs[0][1], runs[1][1])
    assert torch.equal(runs[0][2], runs[1][2])
    s_ref, c_ref = s_np.astype(np.float64), c_np.astype(np.float64)
    for step in range(3):
        u = synth.activations((4, W.d_model), "bf16", seed=380 + step)
        ref = orc.block_step(dims, p64, u, m, s_ref, c_ref)
        for run in runs:
            assert max_abs_rel(to_np(run[0][step]), ref) <= TOL["bf16"]
