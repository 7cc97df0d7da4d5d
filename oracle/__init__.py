"""fp64 CPU oracle (test infrastructure only; the product path never imports it)."""
from .oracle import (Dims, block_fwd, block_step, build, num_threads, rmsnorm_rows, ssd_scan,  # noqa: F401
                     stack_fwd, width)
