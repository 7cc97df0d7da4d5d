"""GPU parity of the standalone selective scan (ssd_scan) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, ensure_built, max_abs_rel, to_device, to_np
from nested_mamba2_selective_b200 import mm_device_status, ssd_scan, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


@pytest.fixture(autouse=True)
def _no_device_timeouts():
    yield
    assert mm_device_status() == 0, "a kernel's bounded wait gave up"


def upload(inp, dtype):
    return dict(x=to_device(inp["x"], dtype), B=to_device(inp["B"], dtype), C=to_device(inp["C"], dtype),
                dt=torch.from_numpy(inp["dt"]).cuda(), A=torch.from_numpy(inp["A"]).cuda(),
                D=torch.from_numpy(inp["D"]).cuda())


def oracle_scan(orc, inp, h, heads=None, b=None, L=None, init=None):
    """Oracle on heads `heads` (subset of [0,h)) of batch rows `b` over the first L tokens."""
    heads = list(range(h)) if heads is None else list(heads)
    bs = slice(None) if b is None else slice(b, b + 1)
    Ls = slice(None) if L is None else slice(0, L)
    x = inp["x"][bs, Ls][:, :, heads]
    dt = inp["dt"][bs, Ls][:, :, heads]
    return orc.ssd_scan(x, dt, inp["A"][heads], inp["B"][bs, Ls], inp["C"][bs, Ls], inp["D"][heads],
                        init_state=None if init is None else init[bs][:, heads], heads_per_group=len(heads))


@pytest.mark.parametrize("h", [24, 12])
@pytest.mark.parametrize("long_memory", [False, True])
def test_scan_reduced_length(orc, h, long_memory):
    """b2 L1000 (3 full chunks of 256 and a ragged tail), 24 heads of 64, d_state 128; the full
    head set and the 12-head prefix slice; long_memory keeps the carried state visible."""
    inp = synth.ssd_inputs(2, 1000, 24, 64, 128, 1, "bf16", seed=201)
    if long_memory:
        inp = synth.long_memory(inp)
    g = upload(inp, "bf16")
    fs = torch.zeros((2, h, 64, 128), device="cuda")
    y = ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], h=h, chunk=256, final_state=fs)
    torch.cuda.synchronize()
    ref, fs_ref = oracle_scan(orc, inp, h)
    assert max_abs_rel(to_np(y), ref) <= TOL["bf16"]
    assert max_abs_rel(to_np(fs), fs_ref) <= TOL["bf16"]


@pytest.mark.parametrize("h", [24, 12])
def test_scan_full_size_sampled(orc, h):
    """b4 L8192 h24 P64 N128 chunk 256 in one launch; the oracle checks batch row 3 on three
    heads over the whole sequence (heads are independent)."""
    w = synth.WORKLOADS["ssd_b4_L8192_h24"]
    inp = synth.ssd_inputs(w.batch, w.seqlen, w.nheads, w.d_head, w.d_state, 1, "bf16", seed=w.seed)
    g = upload(inp, "bf16")
    fs = torch.zeros((w.batch, h, 64, 128), device="cuda")
    y = ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], h=h, chunk=w.chunk, final_state=fs)
    torch.cuda.synchronize()
    heads = [0, h // 2 - 1, h - 1]
    ref, fs_ref = oracle_scan(orc, inp, h, heads=heads, b=3)
    assert max_abs_rel(to_np(y[3:4, :, heads]), ref) <= TOL["bf16"]
    assert max_abs_rel(to_np(fs[3:4, heads]), fs_ref) <= TOL["bf16"]
    assert torch.isfinite(y.float()).all()


def test_scan_f32_matches_oracle(orc):
    inp = synth.ssd_inputs(2, 77, 4, 32, 16, 1, "f32", seed=202)
    g = upload(inp, "f32")
    y = ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk=16)
    torch.cuda.synchronize()
    ref, _ = oracle_scan(orc, inp, 4)
    assert max_abs_rel(to_np(y), ref) <= TOL["f32"]


def test_scan_state_handoff(orc):
    """Scan [0, 700) then [700, 1000) from the returned state; compare with the oracle."""
    inp = synth.long_memory(synth.ssd_inputs(2, 1000, 8, 64, 128, 1, "bf16", seed=203))
    g = upload(inp, "bf16")
    fs1 = torch.zeros((2, 8, 64, 128), device="cuda")
    fs2 = torch.zeros_like(fs1)
    cut = {k: (v[:, :700].contiguous() if v.dim() >= 3 else v) for k, v in g.items()}
    rest = {k: (v[:, 700:].contiguous() if v.dim() >= 3 else v) for k, v in g.items()}
    y1 = ssd_scan(cut["x"], cut["dt"], cut["A"], cut["B"], cut["C"], cut["D"], chunk=256, final_state=fs1)
    y2 = ssd_scan(rest["x"], rest["dt"], rest["A"], rest["B"], rest["C"], rest["D"], chunk=256, init_state=fs1,
                  final_state=fs2)
    torch.cuda.synchronize()
    ref, fs_ref = oracle_scan(orc, inp, 8)
    assert max_abs_rel(to_np(torch.cat([y1, y2], 1)), ref) <= TOL["bf16"]
    assert max_abs_rel(to_np(fs2), fs_ref) <= TOL["bf16"]


@pytest.mark.parametrize("L", [1, 5, 128, 255, 257])
def test_scan_short_and_ragged_lengths(orc, L):
    inp = synth.long_memory(synth.ssd_inputs(3, L, 2, 64, 128, 1, "bf16", seed=204 + L))
    g = upload(inp, "bf16")
    y = ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk=256)
    torch.cuda.synchronize()
    ref, _ = oracle_scan(orc, inp, 2)
    assert max_abs_rel(to_np(y), ref) <= TOL["bf16"]


def test_scan_without_skip_term(orc):
    inp = synth.ssd_inputs(1, 300, 3, 64, 128, 1, "bf16", seed=205)
    g = upload(inp, "bf16")
    y = ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], None, chunk=256)
    torch.cuda.synchronize()
    ref, _ = orc.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], None)
    assert max_abs_rel(to_np(y), ref) <= TOL["bf16"]


def test_scan_two_groups(orc):
    """ngroups = 2: heads 0-1 read group 0, heads 2-3 group 1."""
    inp = synth.long_memory(synth.ssd_inputs(2, 300, 4, 64, 128, 2, "bf16", seed=206))
    g = upload(inp, "bf16")
    y = ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk=256, heads_per_group=2)
    torch.cuda.synchronize()
    ref, _ = orc.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], heads_per_group=2)
    assert max_abs_rel(to_np(y), ref) <= TOL["bf16"]


@pytest.mark.parametrize("chunk", [128, 256, 512])
def test_scan_chunk_parameter_does_not_change_the_result(orc, chunk):
    inp = synth.long_memory(synth.ssd_inputs(1, 700, 3, 64, 128, 1, "bf16", seed=207))
    g = upload(inp, "bf16")
    y = ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk=chunk)
    torch.cuda.synchronize()
    ref, _ = oracle_scan(orc, inp, 3)
    assert max_abs_rel(to_np(y), ref) <= TOL["bf16"]


def test_scan_steep_decay_blocks(orc):
    """Decay far stronger than 2^-100 across a 32-token block (dt A down to -96 per token) on some
    heads and token ranges, next to ordinary ones, and a stretch near that threshold: both ways of
    forming the decay matrix inside one block of 128 tokens, and the carried state across them."""
    inp = synth.ssd_inputs(2, 600, 6, 64, 128, 1, "bf16", seed=208)
    A = inp["A"].copy()
    A[:3] = -16.0
    A[3:] = -1.0
    dt = inp["dt"].copy()
    dt[:, 130:170, 0:3] = 6.0            # steep: about 138 (log2 units) per token on heads 0-2
    dt[:, 300:364, 3] = 3.2 / np.log2(np.e)  # about 3.2 per token on head 3: ~100 across a block
    dt[1, 40:41, 5] = 80.0               # one very steep token on head 5 of batch row 1
    inp = dict(inp, A=A, dt=dt.astype(np.float32))
    g = upload(inp, "bf16")
    fs = torch.zeros((2, 6, 64, 128), device="cuda")
    y = ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk=256, final_state=fs)
    torch.cuda.synchronize()
    ref, fs_ref = oracle_scan(orc, inp, 6)
    assert torch.isfinite(y.float()).all()
    yn, fsn = to_np(y), to_np(fs)
    for i in range(6):  # per head: the steep token's large output must not hide errors elsewhere
        assert max_abs_rel(yn[:, :, i], ref[:, :, i]) <= TOL["bf16"], i
        assert max_abs_rel(fsn[:, i], fs_ref[:, i]) <= TOL["bf16"], i


@pytest.mark.parametrize("h,L", [(5, 1000), (3, 131), (23, 384)])
def test_scan_writes_nothing_outside_its_outputs(orc, h, L):
    """y has a row pitch of h+1 heads (y_stride > h*P) and sits with the final state inside larger
    buffers filled with a sentinel; odd head counts and ragged lengths leave every byte outside the
    outputs, and the padding head of every row, unchanged."""
    b = 2
    inp = synth.long_memory(synth.ssd_inputs(b, L, h, 64, 128, 1, "bf16", seed=210 + h))
    g = upload(inp, "bf16")
    pad = 8192
    ny, ns = b * L * (h + 1) * 64, b * h * 64 * 128
    fy = torch.full((pad + ny + pad,), -9.0, dtype=torch.bfloat16, device="cuda")
    fsf = torch.full((pad + ns + pad,), 13.0, device="cuda")
    y = fy[pad:pad + ny].view(b, L, h + 1, 64)
    fs = fsf[pad:pad + ns].view(b, h, 64, 128)
    ssd_scan(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], h=h, chunk=256, y=y, final_state=fs)
    torch.cuda.synchronize()
    ref, fs_ref = oracle_scan(orc, inp, h)
    assert max_abs_rel(to_np(y[:, :, :h]), ref) <= TOL["bf16"]
    assert max_abs_rel(to_np(fs), fs_ref) <= TOL["bf16"]
    assert torch.all(y[:, :, h:] == -9.0), "write into the padding columns of a y row"
    for flat, fill in ((fy, -9.0), (fsf, 13.0)):
        assert torch.all(flat[:pad] == fill) and torch.all(flat[-pad:] == fill), "write outside an output"
