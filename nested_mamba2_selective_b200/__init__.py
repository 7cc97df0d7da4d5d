"""MatMamba block at a Matryoshka width on B200 (sm_100a).

The computation runs in libmatmamba.so (C ABI in include/matmamba.h); this
package holds its CUDA sources (csrc/), the nvcc build step (build.py), a thin
ctypes binding with the C entry points' names (_lib.py) and the seeded
synthetic input recipes shared by tests and benchmarks (synth.py).
"""
from ._lib import (BlockWeights, MatMambaError, load, matmamba_block_fwd, matmamba_block_fwd_host,  # noqa: F401
                   matmamba_block_workspace, matmamba_stack_fwd, matmamba_stack_workspace, mm_trace_collect,
                   mm_device_status, mm_linear, mm_selftest_wait_timeout, mm_trace_enable, mm_width, ssd_scan,
                   ssd_scan_static, ssd_scan_workspace, ssd_step, ssd_step_workspace, status_string)
