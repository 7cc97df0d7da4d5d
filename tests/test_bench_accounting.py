"""The algorithmic work that bench.py divides by each kernel's time (the roofline's numerator),
checked against the tensors and GEMM shapes it stands for.  CPU only: widths come from the library's
host-side width rule, tensor sizes from the seeded input recipes."""
import ctypes

import numpy as np
import pytest

import bench
from nested_mamba2_selective_b200 import _lib, build, synth


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def width_view(lib, m, d_model, d_inner):
    fake = ctypes.c_void_p(1 << 20)  # host-side validation never dereferences the weights
    p = _lib.BlockParamsC(d_model, d_inner, 64, 128, 1, 4, _lib.MM_BF16, 1e-5, *([fake] * 8))
    d, h = ctypes.c_int(), ctypes.c_int()
    assert lib.mm_width(ctypes.byref(p), m, ctypes.byref(d), ctypes.byref(h)) == 0
    return d.value, h.value


def test_scan_bytes_are_the_scan_operands():
    """x read and y written (bf16, the same shape), B and C read (bf16), dt read (fp32): once each."""
    b, L, h = 2, 48, 6
    inp = synth.ssd_inputs(b, L, h, 64, 128, 1, "bf16", seed=3)
    expect = 2 * inp["x"].size * 2 + (inp["B"].size + inp["C"].size) * 2 + inp["dt"].size * 4
    assert bench.scan_bytes(b * L, h) == expect
    # the standalone workload at 24 heads and at the 12-head prefix
    assert round(bench.scan_bytes(4 * 8192, 24) / 1e6, 1) == 221.2
    assert round(bench.scan_bytes(4 * 8192, 12) / 1e6, 1) == 119.0


@pytest.mark.parametrize("m", [768, 384, 192, 96, 736])
def test_block_work_matches_the_width_view(lib, m):
    """in_proj reads W_in rows z, x (d each), B, C (N each) and dt (h); out_proj is (T, d) x (d, D_m);
    the gated scan reads xBC, dt and z and writes the gated row and two sums of squares per head."""
    T, Dm, E, N = 16384, 768, 1536, 128
    d, h = width_view(lib, m, Dm, E)
    arrays = synth.block_params(Dm, E, 64, N, dtype="bf16", seed=1)
    rows = 2 * d + 2 * N + h
    assert rows <= arrays["W_in"].shape[0]
    w = bench.block_work(m, T)
    assert w["in_proj_conv"] == ("tensor", 2.0 * T * Dm * rows)
    assert w["out_proj_norm"] == ("tensor", 2.0 * T * d * Dm)
    xbc, dt, z = T * (d + 2 * N) * 2, T * h * 4, T * d * 2
    gated, parts = T * d * 2, T * 2 * h * 4
    assert w["ssd_scan_gate"] == ("hbm", xbc + dt + z + gated + parts)
    if m == 768:
        assert round(w["in_proj_conv"][1] / 1e9, 1) == 84.4
        assert round(w["ssd_scan_gate"][1] / 1e6, 1) == 164.1


@pytest.mark.parametrize("m", [2048, 1024, 512])
def test_decode_state_traffic_is_the_active_state(lib, m):
    """The gated state update reads and writes the active heads' fp32 state once per step."""
    Bt, Dm, E, P, N = 256, 2048, 4096, 64, 128
    d, h = width_view(lib, m, Dm, E)
    ssm, conv = synth.states(2, E // P, P, N, E + 2 * N, 4, "bf16", seed=5)
    state_bytes = ssm[:, :h].astype(np.float32).nbytes / 2 * Bt  # per sequence, for Bt sequences
    kind, nbytes = bench.decode_work(m, Bt)["step_scan_gate"]
    rest = Bt * ((d + 2 * N) * 2 + h * 4 + d * 2 + d * 2 + 2 * h * 4)  # xBC, dt, z read; row and sums written
    assert kind == "hbm" and nbytes == 2 * state_bytes + rest
    assert conv.shape[1] == E + 2 * N


def test_stage_table_fraction_is_work_over_time_over_peak():
    """A stage's fraction is its algorithmic work per launch over its mean launch time, against the
    peak of its bound (bf16 tensor FLOP/s or HBM GB/s)."""
    pk = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    stages = {"in_proj_conv": (4, 12, 0.4), "ssd_scan_gate": (2, 4, 0.2)}  # launches, kernels, total ms
    work = {"in_proj_conv": ("tensor", 50e9), "ssd_scan_gate": ("hbm", 250e6)}
    rows = bench.stage_table(stages, work, pk)
    assert rows["in_proj_conv"]["ms_per_launch"] == pytest.approx(0.1)
    assert rows["in_proj_conv"]["achieved"] == pytest.approx(500.0)  # 50 GFLOP in 0.1 ms
    assert rows["in_proj_conv"]["frac"] == pytest.approx(0.5)
    assert rows["ssd_scan_gate"]["achieved"] == pytest.approx(2500.0)  # 250 MB in 0.1 ms
    assert rows["ssd_scan_gate"]["frac"] == pytest.approx(0.5)
    assert rows["in_proj_conv"]["share"] == pytest.approx(2 / 3)
