"""GPU parity of the block forward (matmamba_block_fwd) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, dims_of, ensure_built, make_block, max_abs_rel, to_device, to_np
from nested_mamba2_selective_b200 import (BlockWeights, MatMambaError, matmamba_block_fwd, matmamba_block_fwd_host,
                                          matmamba_block_workspace, synth)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_timeouts():
    yield
    from nested_mamba2_selective_b200 import mm_device_status
    assert mm_device_status() == 0, "a kernel's bounded wait gave up"


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def run_block(orc, w, wt, p64, u, m, chunk, **kw):
    ud = to_device(u, w.dtype)
    out = matmamba_block_fwd(wt, ud, m, chunk, **kw)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("m", [64, 32, 16])
def test_block_tiny_f32_every_width(orc, m):
    """Single block, fp32, b1 L64 d_model 64 (4 heads of 32, d_state 16, chunk 16)."""
    w = synth.WORKLOADS["block_tiny_f32"]
    wt, p64 = make_block(w)
    u = synth.activations((w.batch, w.seqlen, w.d_model), "f32", seed=w.seed + 10)
    dims = dims_of(w)
    H, P, N = dims.nheads, w.d_head, w.d_state
    rows = w.d_inner + 2 * N
    s_out = torch.zeros((1, H, P, N), device="cuda")
    c_out = torch.zeros((1, rows, 3), device="cuda")
    out = run_block(orc, w, wt, p64, u, m, w.chunk, ssm_state_out=s_out, conv_state_out=c_out)
    s_ref = np.zeros((1, H, P, N))
    c_ref = np.zeros((1, rows, 3))
    ref = orc.block_fwd(dims, p64, u, m, ssm_state_out=s_ref, conv_state_out=c_ref)
    assert max_abs_rel(to_np(out), ref) <= TOL["f32"]
    h = orc.width(dims, m)[1]
    assert max_abs_rel(to_np(s_out)[:, :h], s_ref[:, :h]) <= TOL["f32"]
    assert max_abs_rel(to_np(c_out), c_ref) <= TOL["f32"]


@pytest.mark.parametrize("m", [768, 736, 384, 192, 96])
def test_block_130m_reduced_batch(orc, m):
    """130M-class block (d_model 768, 24 heads of 64, d_state 128) on b2 L640: several chunks
    and a ragged tail (640 = 2*256 + 128).  m = 736 is a width outside the trained set that still
    gives whole heads (23, an odd count), as Mix'n'Match allows."""
    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, p64 = make_block(w)
    u = synth.activations((2, 640, w.d_model), "bf16", seed=w.seed + 20)
    out = run_block(orc, w, wt, p64, u, m, w.chunk)
    ref = orc.block_fwd(dims_of(w), p64, u, m)
    err = max_abs_rel(to_np(out), ref)
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("m", [768, 96])
def test_block_130m_full_size_whole_rows(orc, m):
    """Full workload (b8 L2048) in the launch configuration the benchmark times; the oracle checks
    batch rows 0 and 7 over all 2048 tokens (rows are independent), so every 128-token scan block,
    segment and GEMM tile row of those sequences is compared."""
    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, p64 = make_block(w)
    u = synth.activations((w.batch, w.seqlen, w.d_model), "bf16", seed=w.seed + 30)
    out = run_block(orc, w, wt, p64, u, m, w.chunk)
    assert torch.isfinite(out.float()).all()
    on = to_np(out)
    for row in (0, 7):
        ref = orc.block_fwd(dims_of(w), p64, u[row:row + 1], m)
        assert max_abs_rel(on[row:row + 1], ref) <= TOL["bf16"], row


def sliced_weights(wt: BlockWeights, d, h):
    E, GN = wt.d_inner, wt.ngroups * wt.d_state
    W = wt.W_in
    cat = torch.cat
    return BlockWeights(wt.d_model, d, wt.d_head, wt.d_state, wt.ngroups, wt.d_conv, wt.norm_eps,
                        cat([W[0:d], W[E:E + d], W[2 * E:2 * E + 2 * GN], W[2 * E + 2 * GN:2 * E + 2 * GN + h]]).contiguous(),
                        cat([wt.conv_w[0:d], wt.conv_w[E:E + 2 * GN]]).contiguous(),
                        cat([wt.conv_b[0:d], wt.conv_b[E:E + 2 * GN]]).contiguous(),
                        wt.dt_bias[:h].contiguous(), wt.A[:h].contiguous(), wt.D[:h].contiguous(),
                        wt.norm_w[:d].contiguous(), wt.W_out[:, :d].contiguous())


@pytest.mark.parametrize("m", [384, 192])
def test_width_view_is_bit_identical_to_sliced_copy(m):
    """The strided prefix view of the full weights gives exactly the output of a full-width run
    on explicitly sliced contiguous copies."""
    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, _ = make_block(w)
    u = to_device(synth.activations((2, 512, w.d_model), "bf16", seed=5), "bf16")
    d, h = m * 2, m * 2 // 64
    a = matmamba_block_fwd(wt, u, m, 256)
    b = matmamba_block_fwd(sliced_weights(wt, d, h), u, w.d_model, 256)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("m", [768, 192])
def test_block_states_out_and_untouched_regions(orc, m):
    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, p64 = make_block(w)
    dims = dims_of(w)
    H, P, N, E = dims.nheads, w.d_head, w.d_state, w.d_inner
    rows = E + 2 * N
    u = synth.activations((2, 300, w.d_model), "bf16", seed=9)
    s_in_np, c_in_np = synth.states(2, H, P, N, rows, 4, "bf16", seed=10)
    s_in, c_in = torch.from_numpy(s_in_np).cuda(), to_device(c_in_np, "bf16")
    s_out = torch.full((2, H, P, N), 7.25, device="cuda")
    c_out = torch.full((2, rows, 3), -3.5, device="cuda", dtype=torch.bfloat16)
    out = run_block(orc, w, wt, p64, u, m, 256, ssm_state_in=s_in, conv_state_in=c_in, ssm_state_out=s_out,
                    conv_state_out=c_out)
    s_ref = np.zeros((2, H, P, N))
    c_ref = np.zeros((2, rows, 3))
    ref = orc.block_fwd(dims, p64, u, m, ssm_state_in=s_in_np, conv_state_in=c_in_np.astype(np.float64),
                        ssm_state_out=s_ref, conv_state_out=c_ref)
    d, h = orc.width(dims, m)
    assert max_abs_rel(to_np(out), ref) <= TOL["bf16"]
    assert max_abs_rel(to_np(s_out[:, :h]), s_ref[:, :h]) <= TOL["bf16"]
    active = list(range(d)) + list(range(E, rows))
    assert max_abs_rel(to_np(c_out[:, active]), c_ref[:, active]) <= TOL["bf16"]
    assert torch.all(s_out[:, h:] == 7.25)
    assert torch.all(c_out[:, d:E] == -3.5)


@pytest.mark.parametrize("batch,L", [(2, 256), (8, 300), (3, 129)])
def test_host_buffer_entry_point_matches_oracle(orc, batch, L):
    """matmamba_block_fwd_host pipelines sub-batches of sequences through copy streams; its output
    matches the oracle and the device entry point, and nothing is left of a previous result."""
    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, p64 = make_block(w)
    u_np = synth.activations((batch, L, w.d_model), "bf16", seed=12 + batch)
    u = to_device(u_np, "bf16")
    ref = matmamba_block_fwd(wt, u, 384, 256)
    u_host = u.cpu().pin_memory()
    out_host = torch.full_like(u_host, 77.0).pin_memory()
    ws = torch.empty(matmamba_block_workspace(wt, batch, L, 384, 256), dtype=torch.uint8, device="cuda")
    matmamba_block_fwd_host(wt, u_host, 384, 256, out_host, torch.empty_like(u), torch.empty_like(u), ws)
    got = out_host.double().numpy()
    assert max_abs_rel(got, orc.block_fwd(dims_of(w), p64, u_np, 384)) <= TOL["bf16"]
    assert max_abs_rel(got, to_np(ref)) <= TOL["bf16"]


def test_host_entry_point_from_two_threads():
    """Two host threads calling matmamba_block_fwd_host on one device, each with its own buffers and
    stream, get bit for bit what one thread gets: calls on one device take turns on its copy streams
    and events instead of interleaving their records and waits."""
    import threading

    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, _ = make_block(w)
    batch, L, m = 4, 384, 384
    jobs = []
    for k in range(2):
        u = to_device(synth.activations((batch, L, w.d_model), "bf16", seed=70 + k), "bf16")
        job = dict(u_host=u.cpu().pin_memory(), out_host=torch.empty_like(u.cpu()).pin_memory(),
                   u_dev=torch.empty_like(u), out_dev=torch.empty_like(u), results=[], errors=[],
                   ws=torch.empty(matmamba_block_workspace(wt, batch, L, m, 256), dtype=torch.uint8,
                                  device="cuda"))
        matmamba_block_fwd_host(wt, job["u_host"], m, 256, job["out_host"], job["u_dev"], job["out_dev"], job["ws"])
        job["ref"] = job["out_host"].clone()
        jobs.append(job)
    assert not torch.equal(jobs[0]["ref"], jobs[1]["ref"])

    def worker(job):
        try:
            torch.cuda.set_device(0)
            with torch.cuda.stream(torch.cuda.Stream()):
                for _ in range(6):
                    job["out_host"].fill_(0.0)
                    matmamba_block_fwd_host(wt, job["u_host"], m, 256, job["out_host"], job["u_dev"],
                                            job["out_dev"], job["ws"])
                    job["results"].append(job["out_host"].clone())
        except Exception as e:  # reported by the main thread
            job["errors"].append(repr(e))

    threads = [threading.Thread(target=worker, args=(job,)) for job in jobs]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads)
    torch.cuda.synchronize()
    for job in jobs:
        assert job["errors"] == []
        assert len(job["results"]) == 6
        for got in job["results"]:
            assert torch.equal(got, job["ref"])


def test_invalid_width_raises_and_launches_nothing():
    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, _ = make_block(w)
    u = to_device(synth.activations((1, 64, w.d_model), "bf16", seed=13), "bf16")
    out = torch.full_like(u, 5.0)
    for m in (100, 0, 800):
        with pytest.raises(MatMambaError) as ei:
            matmamba_block_fwd(wt, u, m, 256, out=out)
        assert ei.value.status == 1
    assert torch.all(out == 5.0)


def test_single_token_and_tiny_lengths(orc):
    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, p64 = make_block(w)
    for L in (1, 3, 129):
        u = synth.activations((3, L, w.d_model), "bf16", seed=40 + L)
        out = run_block(orc, w, wt, p64, u, 192, 256)
        assert max_abs_rel(to_np(out), orc.block_fwd(dims_of(w), p64, u, 192)) <= TOL["bf16"]


@pytest.mark.parametrize("L", [1, 2, 5])
def test_short_prefill_with_history_and_state_out(orc, L):
    """Prefills shorter than the conv window read the given history and shift it into the new state."""
    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, p64 = make_block(w)
    dims = dims_of(w)
    H, P, N, E = dims.nheads, w.d_head, w.d_state, w.d_inner
    rows = E + 2 * N
    u = synth.activations((2, L, w.d_model), "bf16", seed=60 + L)
    s_in_np, c_in_np = synth.states(2, H, P, N, rows, 4, "bf16", seed=61)
    s_out = torch.zeros((2, H, P, N), device="cuda")
    c_out = torch.zeros((2, rows, 3), device="cuda", dtype=torch.bfloat16)
    out = run_block(orc, w, wt, p64, u, 384, 256, ssm_state_in=torch.from_numpy(s_in_np).cuda(),
                    conv_state_in=to_device(c_in_np, "bf16"), ssm_state_out=s_out, conv_state_out=c_out)
    s_ref, c_ref = np.zeros((2, H, P, N)), np.zeros((2, rows, 3))
    ref = orc.block_fwd(dims, p64, u, 384, ssm_state_in=s_in_np, conv_state_in=c_in_np.astype(np.float64),
                        ssm_state_out=s_ref, conv_state_out=c_ref)
    d, h = orc.width(dims, 384)
    assert max_abs_rel(to_np(out), ref) <= TOL["bf16"]
    assert max_abs_rel(to_np(s_out[:, :h]), s_ref[:, :h]) <= TOL["bf16"]
    active = list(range(d)) + list(range(E, rows))
    assert max_abs_rel(to_np(c_out[:, active]), c_ref[:, active]) <= TOL["bf16"]


def test_repeated_calls_are_bit_identical():
    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, _ = make_block(w)
    u = to_device(synth.activations((4, 700, w.d_model), "bf16", seed=70), "bf16")
    a = matmamba_block_fwd(wt, u, 768, 256)
    b = matmamba_block_fwd(wt, u, 768, 256)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def guarded(shape, dtype, fill, pad=4096):
    """A tensor of `shape` inside a larger buffer whose other elements hold `fill`."""
    n = int(np.prod(shape))
    flat = torch.full((pad + n + pad,), fill, dtype=dtype, device="cuda")
    return flat, flat[pad:pad + n].view(*shape), (pad, pad + n)


def assert_outside_untouched(flat, span, fill):
    lo, hi = span
    assert torch.all(flat[:lo] == fill) and torch.all(flat[hi:] == fill), "write outside the output region"


@pytest.mark.parametrize("m,L", [(736, 300), (96, 131)])
def test_block_writes_nothing_outside_its_outputs(orc, m, L):
    """out, ssm_state_out and conv_state_out each sit inside a larger buffer filled with a sentinel;
    with a ragged length and an odd head count (23 or 3 heads) no byte outside the outputs (nor an
    inactive head or conv row) changes, and the outputs match the oracle."""
    w = synth.WORKLOADS["block_130m_b8_L2048"]
    wt, p64 = make_block(w)
    dims = dims_of(w)
    H, P, N, E = dims.nheads, w.d_head, w.d_state, w.d_inner
    rows = E + 2 * N
    u = synth.activations((3, L, w.d_model), "bf16", seed=80 + m)
    fo, out, so = guarded((3, L, w.d_model), torch.bfloat16, -7.0)
    fs, s_out, ss = guarded((3, H, P, N), torch.float32, 11.5)
    fc, c_out, sc = guarded((3, rows, 3), torch.bfloat16, -5.0)
    run_block(orc, w, wt, p64, u, m, 256, out=out, ssm_state_out=s_out, conv_state_out=c_out)
    d, h = orc.width(dims, m)
    s_ref, c_ref = np.zeros((3, H, P, N)), np.zeros((3, rows, 3))
    ref = orc.block_fwd(dims, p64, u, m, ssm_state_out=s_ref, conv_state_out=c_ref)
    assert max_abs_rel(to_np(out), ref) <= TOL["bf16"]
    assert max_abs_rel(to_np(s_out[:, :h]), s_ref[:, :h]) <= TOL["bf16"]
    active = list(range(d)) + list(range(E, rows))
    assert max_abs_rel(to_np(c_out[:, active]), c_ref[:, active]) <= TOL["bf16"]
    assert torch.all(s_out[:, h:] == 11.5) and torch.all(c_out[:, d:E] == -5.0)
    for flat, span, fill in ((fo, so, -7.0), (fs, ss, 11.5), (fc, sc, -5.0)):
        assert_outside_untouched(flat, span, fill)
