"""Host-side checks of the C ABI: the library loads, exports every declared symbol, and
validates widths, shapes and workspace sizes without touching a GPU."""
import ctypes
import os
import re

import pytest

from nested_mamba2_selective_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "matmamba.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.EXPORTS)


def params(dtype=_lib.MM_BF16, d_model=768, d_inner=1536, d_head=64, d_state=128, ngroups=1, d_conv=4):
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced by host-side validation
    return _lib.BlockParamsC(d_model, d_inner, d_head, d_state, ngroups, d_conv, dtype, 1e-5,
                             *([fake] * 8))


def test_width_rule_on_host(lib):
    p = params()
    d, h = ctypes.c_int(), ctypes.c_int()
    for m, dd, hh in ((768, 1536, 24), (384, 768, 12), (192, 384, 6), (96, 192, 3), (32, 64, 1), (736, 1472, 23)):
        assert lib.mm_width(ctypes.byref(p), m, ctypes.byref(d), ctypes.byref(h)) == 0
        assert (d.value, h.value) == (dd, hh)
    for m in (0, -1, 769, 1000, 16, 100):
        assert lib.mm_width(ctypes.byref(p), m, None, None) == 1


def test_param_validation(lib):
    assert lib.mm_width(ctypes.byref(params(d_inner=1530)), 768, None, None) == 2     # E % P
    assert lib.mm_width(ctypes.byref(params(dtype=7)), 768, None, None) == 3
    assert lib.mm_width(ctypes.byref(params(d_state=512)), 768, None, None) == 2
    assert lib.mm_width(None, 768, None, None) == 8
    p = params()
    p.W_out = None
    assert lib.mm_width(ctypes.byref(p), 768, None, None) == 8
    p = params()
    p.W_in = ctypes.c_void_p((1 << 20) + 2)
    assert lib.mm_width(ctypes.byref(p), 768, None, None) == 4


def test_workspace_queries_scale_with_width(lib):
    p = params()
    sizes = []
    for m in (768, 384, 192, 96):
        n = ctypes.c_size_t()
        assert lib.matmamba_block_workspace(ctypes.byref(p), 8, 2048, m, 256, ctypes.byref(n)) == 0
        sizes.append(n.value)
    assert sizes == sorted(sizes, reverse=True) and sizes[-1] > 0
    n = ctypes.c_size_t()
    assert lib.matmamba_block_workspace(ctypes.byref(p), 8, 2048, 100, 256, ctypes.byref(n)) == 1
    assert lib.ssd_scan_workspace(1, 4, 8192, 24, 64, 128, 1, 256, ctypes.byref(n)) == 0
    assert lib.ssd_step_workspace(ctypes.byref(p), 256, 768, ctypes.byref(n)) == 0 and n.value > 0


def test_rejected_calls_launch_nothing(lib):
    """Invalid arguments return before any CUDA call, so they work without a device."""
    p = params()
    fake = ctypes.c_void_p(1 << 20)
    assert lib.matmamba_block_fwd(ctypes.byref(p), fake, 2, 16, 100, 256, fake, None, None, None, None, fake, 1 << 30,
                                  None) == 1
    assert lib.matmamba_block_fwd(ctypes.byref(p), fake, 2, 16, 768, 256, fake, None, None, None, None, fake, 16,
                                  None) == 5
    assert lib.matmamba_block_fwd(ctypes.byref(p), fake, 0, 16, 768, 256, fake, None, None, None, None, fake, 1 << 30,
                                  None) == 2
    assert lib.ssd_scan(9, fake, 64, fake, 1, fake, fake, 128, fake, 128, None, 1, 64, 1, 64, 128, 1, 1, 256, None, 0,
                        fake, 64, None, None, 0, None) == 3
    assert lib.ssd_scan(1, ctypes.c_void_p((1 << 20) + 8), 64, fake, 1, fake, fake, 128, fake, 128, None, 1, 64, 1, 64,
                        128, 1, 1, 256, None, 0, fake, 64, None, None, 0, None) == 4


def test_batch_and_token_limits_are_checked_on_the_host(lib):
    """At most 65535 sequences (they go on a grid's y or z dimension) and fewer than 2^31 tokens per
    call: queries and calls beyond that return MM_ERR_SHAPE before anything is launched."""
    p = params()
    n = ctypes.c_size_t()
    assert lib.matmamba_block_workspace(ctypes.byref(p), 65535, 16, 768, 256, ctypes.byref(n)) == 0
    assert lib.matmamba_block_workspace(ctypes.byref(p), 65536, 16, 768, 256, ctypes.byref(n)) == 2
    assert lib.matmamba_block_workspace(ctypes.byref(p), 1024, 1 << 21, 768, 256, ctypes.byref(n)) == 2
    assert lib.ssd_scan_workspace(1, 65535, 64, 24, 64, 128, 1, 256, ctypes.byref(n)) == 0
    assert lib.ssd_scan_workspace(1, 65536, 64, 24, 64, 128, 1, 256, ctypes.byref(n)) == 2
    assert lib.ssd_step_workspace(ctypes.byref(p), 65535, 768, ctypes.byref(n)) == 0
    assert lib.ssd_step_workspace(ctypes.byref(p), 65536, 768, ctypes.byref(n)) == 2
    fake = ctypes.c_void_p(1 << 20)
    assert lib.matmamba_block_fwd(ctypes.byref(p), fake, 65536, 1, 768, 256, fake, None, None, None, None, fake,
                                  1 << 40, None) == 2
    assert lib.ssd_scan(1, fake, 64, fake, 1, fake, fake, 128, fake, 128, None, 65536, 1, 1, 64, 128, 1, 1, 256,
                        None, 0, fake, 64, None, fake, 1 << 40, None) == 2
    assert lib.ssd_step(ctypes.byref(p), fake, fake, fake, 65536, 768, fake, fake, 1 << 40, None) == 2
    assert lib.matmamba_block_fwd_host(ctypes.byref(p), fake, 65536, 1, 768, 256, fake, fake, fake, fake, 1 << 40,
                                       None) == 2


def test_overlapping_state_buffers_are_rejected(lib):
    """A final state that shares bytes with the initial state is refused before any launch; disjoint
    buffers pass validation (and would launch, so they are not called here)."""
    base = 1 << 24
    x, dt, a_, bc, y = (ctypes.c_void_p(base + i * (1 << 22)) for i in range(5))
    init = ctypes.c_void_p(base + 8 * (1 << 22))
    for shift in (0, 64, (1 << 15) - 4):    # same start, inside, last float of the first head
        final = ctypes.c_void_p(init.value + shift)
        assert lib.ssd_scan(1, x, 64, dt, 1, a_, bc, 128, bc, 128, None, 1, 64, 1, 64, 128, 1, 1, 256, init,
                            64 * 128, y, 64, final, None, 0, None) == 2
    p = params()
    fake = ctypes.c_void_p(1 << 20)
    s_in = ctypes.c_void_p(1 << 26)
    s_out = ctypes.c_void_p((1 << 26) + 4096)
    assert lib.matmamba_block_fwd(ctypes.byref(p), fake, 2, 16, 768, 256, fake, s_in, None, s_out, None, fake,
                                  1 << 30, None) == 2


def test_status_strings(lib):
    for s in range(10):
        assert lib.mm_status_string(s)
    assert lib.mm_version() >= 100


def test_selftest_rejects_limits_out_of_range_on_the_host():
    from nested_mamba2_selective_b200 import _lib
    lib = _lib.load()
    for bad in (0, 2_000_000):
        assert lib.mm_selftest_wait_timeout(bad, None) == 2  # MM_ERR_SHAPE, before any launch
