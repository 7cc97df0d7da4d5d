"""GPU checks of the projection kernel (mm_linear) against an fp64 matmul of the same inputs."""
import numpy as np
import pytest
import torch

from gpu_util import ensure_built, max_abs_rel, to_np
from nested_mamba2_selective_b200 import mm_device_status, mm_linear, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_device_timeouts():
    yield
    from nested_mamba2_selective_b200 import mm_device_status
    assert mm_device_status() == 0, "a kernel's bounded wait gave up"


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


@pytest.mark.parametrize("M,K,N", [(1000, 768, 3352), (256, 2048, 8512), (130, 200, 72), (16384, 1536, 768),
                                   (7, 64, 16), (300, 4096, 2048)])
def test_linear_bf16(M, K, N):
    a = synth.activations((M, K), "bf16", seed=M + K)
    w = synth.activations((N, K), "bf16", seed=N + 7, std=0.05)
    out = mm_linear(torch.from_numpy(a).cuda().bfloat16(), torch.from_numpy(w).cuda().bfloat16())
    assert mm_device_status() == 0
    ref = a.astype(np.float64) @ w.astype(np.float64).T
    assert max_abs_rel(to_np(out), ref) <= 5e-3


@pytest.mark.parametrize("M,K,N", [(333, 768, 24), (512, 512, 256)])
def test_linear_fp32_out_and_accumulate(M, K, N):
    a = synth.activations((M, K), "bf16", seed=1)
    w = synth.activations((N, K), "bf16", seed=2, std=0.05)
    A, W = torch.from_numpy(a).cuda().bfloat16(), torch.from_numpy(w).cuda().bfloat16()
    base = torch.from_numpy(synth.activations((M, N), "f32", seed=3)).cuda()
    out = mm_linear(A, W, out=base.clone(), out_f32=True, accumulate=True)
    plain = mm_linear(A, W, out_f32=True)
    torch.cuda.synchronize()
    ref = a.astype(np.float64) @ w.astype(np.float64).T
    assert max_abs_rel(to_np(plain), ref) <= 1e-5
    assert max_abs_rel(to_np(out), ref + base.cpu().numpy()) <= 1e-5


def test_linear_fp32():
    a = synth.activations((100, 96), "f32", seed=4)
    w = synth.activations((40, 96), "f32", seed=5)
    out = mm_linear(torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert max_abs_rel(to_np(out), a.astype(np.float64) @ w.astype(np.float64).T) <= 1e-5


@pytest.mark.parametrize("out_f32", [False, True])
def test_linear_many_tiles_writes_every_tile_once(out_f32):
    """Twelve times more tiles than SMs: running CTAs take over the tiles of CTAs that have not
    started, and each tile must still be written (the output starts as NaN) with the plain value."""
    M, K, N = 8192, 768, 3352
    a = synth.activations((M, K), "bf16", seed=11)
    w = synth.activations((N, K), "bf16", seed=12, std=0.05)
    A, W = torch.from_numpy(a).cuda().bfloat16(), torch.from_numpy(w).cuda().bfloat16()
    out = torch.full((M, N), float("nan"), dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
    mm_linear(A, W, out=out, out_f32=out_f32)
    torch.cuda.synchronize()
    assert not torch.isnan(out).any()
    ref = a.astype(np.float64) @ w.astype(np.float64).T
    assert max_abs_rel(to_np(out), ref) <= (1e-5 if out_f32 else 5e-3)


@pytest.mark.parametrize("out_f32", [False, True])
def test_linear_cta_pairs_odd_row_blocks(out_f32):
    """Wide tiles with K >= 512 run on CTA pairs, each pair taking two 128-row blocks.  With 9 row
    blocks the last pair's second CTA gets rows past M: they must load as zeros and store nothing.
    The output sits inside a NaN-filled buffer: every row of it is written, and the 64 rows after
    it stay untouched."""
    M, K, N = 128 * 8 + 50, 768, 3352
    a = synth.activations((M, K), "bf16", seed=21)
    w = synth.activations((N, K), "bf16", seed=22, std=0.05)
    A, W = torch.from_numpy(a).cuda().bfloat16(), torch.from_numpy(w).cuda().bfloat16()
    full = torch.full((M + 64, N), float("nan"), dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
    mm_linear(A, W, out=full[:M], out_f32=out_f32)
    torch.cuda.synchronize()
    assert mm_device_status() == 0
    assert not torch.isnan(full[:M]).any()
    assert torch.isnan(full[M:]).all()
    ref = a.astype(np.float64) @ w.astype(np.float64).T
    assert max_abs_rel(to_np(full[:M]), ref) <= (1e-5 if out_f32 else 5e-3)
