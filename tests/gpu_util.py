"""Shared helpers of the GPU parity tests (no arithmetic of the method lives here)."""
import numpy as np
import torch

import oracle
from nested_mamba2_selective_b200 import BlockWeights, build, synth

# Tolerances on max|gpu - ref| / max|ref| per output tensor.
TOL = {"f32": 1e-4, "bf16": 2e-2}
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def ensure_built():
    build.build()


def max_abs_rel(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), "non-finite GPU output"
    return float(np.max(np.abs(gpu - ref)) / max(np.max(np.abs(ref)), 1e-30))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def dims_of(w: synth.Workload) -> oracle.Dims:
    return oracle.Dims(w.d_model, w.d_inner, w.d_head, w.d_state, w.ngroups, w.d_conv, 1e-5)


def make_block(w: synth.Workload, seed=None, d_model=None):
    """(device weights, fp64 oracle params) for the workload's block sizes."""
    arrays = synth.block_params(w.d_model, w.d_inner, w.d_head, w.d_state, w.ngroups, w.d_conv, dtype=w.dtype,
                                seed=w.seed if seed is None else seed)
    wt = BlockWeights.from_arrays(arrays, w.d_model, w.d_inner, w.d_head, w.d_state, w.ngroups, w.d_conv, 1e-5,
                                  dtype=TORCH_DTYPE[w.dtype])
    return wt, {k: v.astype(np.float64) for k, v in arrays.items()}


def to_device(a: np.ndarray, dtype: str):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().to(TORCH_DTYPE[dtype])
