"""Thin Python binding of libmatmamba.so (argument marshalling only).

Every function here checks tensor placement and dtypes, passes raw device
pointers and the current CUDA stream to the C ABI declared in
include/matmamba.h, and raises MatMambaError on a non-zero status.  All
arithmetic runs in the library's CUDA kernels; PyTorch only provides device
memory and streams.  There is no fallback: a missing library raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmatmamba.so")

MM_F32, MM_BF16 = 0, 1
_DTYPES = {torch.float32: MM_F32, torch.bfloat16: MM_BF16}
_TORCH = {MM_F32: torch.float32, MM_BF16: torch.bfloat16}


class MatMambaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = " [%s]" % load().mm_last_cuda_error().decode() if status == 6 else ""
        super().__init__("%s failed: %s (status %d)%s" % (where, status_string(status), status, detail))


class BlockParamsC(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("d_inner", ctypes.c_int), ("d_head", ctypes.c_int),
                ("d_state", ctypes.c_int), ("ngroups", ctypes.c_int), ("d_conv", ctypes.c_int),
                ("dtype", ctypes.c_int), ("norm_eps", ctypes.c_float),
                ("W_in", ctypes.c_void_p), ("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p),
                ("dt_bias", ctypes.c_void_p), ("A", ctypes.c_void_p), ("D", ctypes.c_void_p),
                ("norm_w", ctypes.c_void_p), ("W_out", ctypes.c_void_p)]


_vp, _i, _i64, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_pp = ctypes.POINTER(BlockParamsC)
_SIGS = {
    "mm_status_string": ([_i], ctypes.c_char_p),
    "mm_last_cuda_error": ([], ctypes.c_char_p),
    "mm_version": ([], _i),
    "mm_device_status": ([_vp], _i),
    "mm_width": ([_pp, _i, ctypes.POINTER(_i), ctypes.POINTER(_i)], _i),
    "matmamba_block_workspace": ([_pp, _i, _i, _i, _i, ctypes.POINTER(_sz)], _i),
    "matmamba_block_fwd": ([_pp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _i),
    "matmamba_block_fwd_host": ([_pp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp], _i),
    "ssd_scan_workspace": ([_i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_sz)], _i),
    "ssd_scan": ([_i, _vp, _i64, _vp, _i64, _vp, _vp, _i64, _vp, _i64, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                  _vp, _i64, _vp, _i64, _vp, _vp, _sz, _vp], _i),
    "ssd_scan_static": ([_i, _vp, _i64, _vp, _i64, _vp, _vp, _i64, _vp, _i64, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                         _vp, _i64, _vp, _i64, _vp, _vp], _i),
    "mm_selftest_wait_timeout": ([ctypes.c_uint, _vp], _i),
    "ssd_step_workspace": ([_pp, _i, _i, ctypes.POINTER(_sz)], _i),
    "ssd_step": ([_pp, _vp, _vp, _vp, _i, _i, _vp, _vp, _sz, _vp], _i),
    "matmamba_stack_workspace": ([_pp, _i, ctypes.POINTER(_i), _i, _i, _i, ctypes.POINTER(_sz)], _i),
    "matmamba_stack_fwd": ([_pp, ctypes.POINTER(_vp), _f, _i, ctypes.POINTER(_i), _vp, _i, _i, _i, _vp, _vp, _sz,
                            _vp], _i),
    "mm_linear": ([_i, _vp, _i64, _i, _i, _vp, _i64, _i, _vp, _i64, _i, _i, _vp], _i),
    "mm_trace_enable": ([_i], _i),
    "mm_trace_collect": ([_vp, _i, ctypes.POINTER(_i), ctypes.POINTER(_i)], _i),
}
EXPORTS = tuple(_SIGS)
_lib = None


def load() -> ctypes.CDLL:
    """Load libmatmamba.so from the package directory (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmatmamba.so is not built; run nested_mamba2_selective_b200.build.build()")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes, fn.restype = args, res
        _lib = lib
    return _lib


def mm_device_status(stream=None) -> int:
    """Synchronize the stream and return (then clear) the device status word."""
    return int(load().mm_device_status(_stream(stream)))


def status_string(status: int) -> str:
    return load().mm_status_string(int(status)).decode()


def _check(rc: int, where: str):
    if rc:
        raise MatMambaError(rc, where)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _workspace(nbytes: int, device, workspace=None):
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError("workspace too small: need %d bytes" % nbytes)
        return workspace
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


@dataclass
class BlockWeights:
    """Full-width block parameters on the device (see include/matmamba.h for shapes)."""
    d_model: int
    d_inner: int
    d_head: int
    d_state: int
    ngroups: int
    d_conv: int
    norm_eps: float
    W_in: torch.Tensor
    conv_w: torch.Tensor
    conv_b: torch.Tensor
    dt_bias: torch.Tensor
    A: torch.Tensor
    D: torch.Tensor
    norm_w: torch.Tensor
    W_out: torch.Tensor

    @property
    def dtype(self) -> torch.dtype:
        return self.W_in.dtype

    @property
    def nheads(self) -> int:
        return self.d_inner // self.d_head

    def c_struct(self) -> BlockParamsC:
        for k in ("dt_bias", "A", "D"):
            if getattr(self, k).dtype != torch.float32:
                raise ValueError("%s must be float32" % k)
        for k in ("conv_w", "conv_b", "norm_w", "W_out"):
            if getattr(self, k).dtype != self.dtype:
                raise ValueError("%s must match W_in's dtype" % k)
        return BlockParamsC(self.d_model, self.d_inner, self.d_head, self.d_state, self.ngroups, self.d_conv,
                            _DTYPES[self.dtype], self.norm_eps,
                            *[_ptr(getattr(self, k)) for k in ("W_in", "conv_w", "conv_b", "dt_bias", "A", "D",
                                                                "norm_w", "W_out")])

    @staticmethod
    def from_arrays(arrays: dict, d_model, d_inner, d_head, d_state, ngroups=1, d_conv=4, norm_eps=1e-5,
                    dtype=torch.bfloat16, device="cuda"):
        """Upload float32 numpy arrays (values exact in ``dtype``) to the device."""
        t = {}
        for k, v in arrays.items():
            dt = torch.float32 if k in ("dt_bias", "A", "D") else dtype
            t[k] = torch.from_numpy(v).to(device=device).to(dt).contiguous()
        return BlockWeights(d_model, d_inner, d_head, d_state, ngroups, d_conv, norm_eps, **t)


def mm_width(w: BlockWeights, m_i: int):
    d, h = ctypes.c_int(), ctypes.c_int()
    _check(load().mm_width(ctypes.byref(w.c_struct()), int(m_i), ctypes.byref(d), ctypes.byref(h)), "mm_width")
    return d.value, h.value


def matmamba_block_workspace(w: BlockWeights, batch: int, L: int, m_i: int, chunk: int = 256) -> int:
    n = ctypes.c_size_t()
    _check(load().matmamba_block_workspace(ctypes.byref(w.c_struct()), batch, L, int(m_i), chunk, ctypes.byref(n)),
           "matmamba_block_workspace")
    return n.value


def matmamba_block_fwd(w: BlockWeights, u: torch.Tensor, m_i: int, chunk: int = 256, out=None, ssm_state_in=None,
                       conv_state_in=None, ssm_state_out=None, conv_state_out=None, workspace=None, stream=None):
    """out (b, L, d_model) = block at width m_i applied to u (b, L, d_model)."""
    if u.dim() != 3 or u.shape[2] != w.d_model or u.dtype != w.dtype:
        raise ValueError("u must be (batch, L, d_model) in the weights' dtype")
    b, L, _ = u.shape
    if out is None:
        out = torch.empty_like(u)
    ws = _workspace(matmamba_block_workspace(w, b, L, m_i, chunk), u.device, workspace)
    rc = load().matmamba_block_fwd(ctypes.byref(w.c_struct()), _ptr(u), b, L, int(m_i), int(chunk), _ptr(out),
                                   _ptr(ssm_state_in), _ptr(conv_state_in), _ptr(ssm_state_out),
                                   _ptr(conv_state_out), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "matmamba_block_fwd")
    return out


def matmamba_block_fwd_host(w: BlockWeights, u_host: torch.Tensor, m_i: int, chunk: int, out_host: torch.Tensor,
                            u_dev: torch.Tensor, out_dev: torch.Tensor, workspace: torch.Tensor, stream=None):
    """Host-buffer variant: copies u_host in, runs the block, copies the result to out_host, waits."""
    b, L, _ = u_host.shape
    rc = load().matmamba_block_fwd_host(ctypes.byref(w.c_struct()), ctypes.c_void_p(u_host.data_ptr()), b, L,
                                        int(m_i), int(chunk), ctypes.c_void_p(out_host.data_ptr()), _ptr(u_dev),
                                        _ptr(out_dev), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "matmamba_block_fwd_host")
    return out_host


def mm_linear(A: torch.Tensor, W: torch.Tensor, out=None, out_f32: bool = False, accumulate: bool = False,
              stream=None):
    """out (M, N) (+)= A (M, K) . W (N, K)^T through the library's projection kernel."""
    M, K = A.shape
    N = W.shape[0]
    if W.shape[1] != K or W.dtype != A.dtype:
        raise ValueError("W must be (N, K) in A's dtype")
    if out is None:
        out = torch.zeros((M, N), dtype=torch.float32 if out_f32 else A.dtype, device=A.device)
    rc = load().mm_linear(_DTYPES[A.dtype], _ptr(A), K, M, K, _ptr(W), K, N, _ptr(out), out.shape[1],
                          int(out_f32), int(accumulate), _stream(stream))
    _check(rc, "mm_linear")
    return out


def ssd_scan_workspace(dtype, batch, L, h, P, N, G=1, chunk=256) -> int:
    n = ctypes.c_size_t()
    _check(load().ssd_scan_workspace(_DTYPES[dtype], batch, L, h, P, N, G, chunk, ctypes.byref(n)),
           "ssd_scan_workspace")
    return n.value


def ssd_scan(x, dt, A, B, C, D=None, h=None, chunk=256, heads_per_group=None, init_state=None, final_state=None,
             y=None, workspace=None, stream=None):
    """Selective scan.  x (b, L, H_x, P) with heads [0, h) used, dt (b, L, H_dt) fp32, A/D (>= h) fp32,
    B/C (b, L, G, N).  Returns y (b, L, h, P) in x's dtype (or writes the given y, which may be wider)."""
    b, L, Hx, P = x.shape
    G, N = B.shape[2], B.shape[3]
    h = Hx if h is None else h
    hpg = heads_per_group if heads_per_group is not None else -(-h // G)
    if y is None:
        y = torch.empty((b, L, h, P), dtype=x.dtype, device=x.device)
    st_stride = 0
    for s in (init_state, final_state):
        if s is not None:
            st_stride = s.shape[1] * s.shape[2] * s.shape[3]
    ws = _workspace(ssd_scan_workspace(x.dtype, b, L, h, P, N, G, chunk), x.device, workspace)
    rc = load().ssd_scan(_DTYPES[x.dtype], _ptr(x), Hx * P, _ptr(dt), dt.shape[2], _ptr(A), _ptr(B), G * N, _ptr(C),
                         G * N, _ptr(D), b, L, h, P, N, G, hpg, int(chunk), _ptr(init_state), st_stride, _ptr(y),
                         y.shape[2] * y.shape[3], _ptr(final_state), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "ssd_scan")
    return y


def ssd_scan_static(x, dt, A, B, C, D=None, h=None, chunk=256, heads_per_group=None, init_state=None,
                    final_state=None, y=None, stream=None):
    """ssd_scan with the library's own fixed scratch array instead of a workspace (no allocation
    inside the call; calls on one device must not overlap on the GPU)."""
    b, L, Hx, P = x.shape
    G, N = B.shape[2], B.shape[3]
    h = Hx if h is None else h
    hpg = heads_per_group if heads_per_group is not None else -(-h // G)
    if y is None:
        y = torch.empty((b, L, h, P), dtype=x.dtype, device=x.device)
    st_stride = 0
    for s in (init_state, final_state):
        if s is not None:
            st_stride = s.shape[1] * s.shape[2] * s.shape[3]
    rc = load().ssd_scan_static(_DTYPES[x.dtype], _ptr(x), Hx * P, _ptr(dt), dt.shape[2], _ptr(A), _ptr(B), G * N,
                                _ptr(C), G * N, _ptr(D), b, L, h, P, N, G, hpg, int(chunk), _ptr(init_state),
                                st_stride, _ptr(y), y.shape[2] * y.shape[3], _ptr(final_state), _stream(stream))
    _check(rc, "ssd_scan_static")
    return y


def mm_selftest_wait_timeout(timeout_us=20000, stream=None):
    """Run the failure-path self-test: a kernel whose bounded wait gives up after timeout_us and
    records MM_ERR_TIMEOUT in the device status word (read it with mm_device_status)."""
    _check(load().mm_selftest_wait_timeout(int(timeout_us), _stream(stream)), "mm_selftest_wait_timeout")


def ssd_step_workspace(w: BlockWeights, batch: int, m_i: int) -> int:
    n = ctypes.c_size_t()
    _check(load().ssd_step_workspace(ctypes.byref(w.c_struct()), batch, int(m_i), ctypes.byref(n)),
           "ssd_step_workspace")
    return n.value


def ssd_step(w: BlockWeights, ssm_state, conv_state, u_t, m_i: int, out_t=None, workspace=None, stream=None):
    """One recurrent token: u_t (b, d_model) -> out_t; ssm_state / conv_state updated in place."""
    b = u_t.shape[0]
    if out_t is None:
        out_t = torch.empty_like(u_t)
    ws = _workspace(ssd_step_workspace(w, b, m_i), u_t.device, workspace)
    rc = load().ssd_step(ctypes.byref(w.c_struct()), _ptr(ssm_state), _ptr(conv_state), _ptr(u_t), b, int(m_i),
                         _ptr(out_t), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "ssd_step")
    return out_t


def _stack_structs(layers):
    arr = (BlockParamsC * len(layers))()
    for i, w in enumerate(layers):
        arr[i] = w.c_struct()
    return arr


def matmamba_stack_workspace(layers, m_per_layer, batch: int, L: int, chunk: int = 256) -> int:
    n = ctypes.c_size_t()
    ms = (ctypes.c_int * len(layers))(*[int(m) for m in m_per_layer])
    _check(load().matmamba_stack_workspace(_stack_structs(layers), len(layers), ms, batch, L, chunk, ctypes.byref(n)),
           "matmamba_stack_workspace")
    return n.value


class TraceEntryC(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("stages", ctypes.c_int), ("kernels", ctypes.c_int),
                ("total_ms", ctypes.c_double)]


def mm_trace_enable(capacity: int):
    """Start (capacity > 0) or stop (0) per-stage CUDA-event tracing inside the library."""
    _check(load().mm_trace_enable(int(capacity)), "mm_trace_enable")


def mm_trace_collect():
    """Per-stage totals since the last collect: ({name: (stages, kernels, total_ms)}, kernel launches)."""
    arr = (TraceEntryC * 64)()
    n, k = ctypes.c_int(), ctypes.c_int()
    _check(load().mm_trace_collect(ctypes.cast(arr, ctypes.c_void_p), 64, ctypes.byref(n), ctypes.byref(k)),
           "mm_trace_collect")
    return {arr[i].name.decode(): (arr[i].stages, arr[i].kernels, arr[i].total_ms) for i in range(n.value)}, k.value


def matmamba_stack_fwd(layers, prenorm_w, u, m_per_layer, chunk: int = 256, prenorm_eps: float = 1e-5, out=None,
                       workspace=None, stream=None):
    """Pre-norm residual stack of len(layers) blocks, layer l at width m_per_layer[l]."""
    b, L, _ = u.shape
    if out is None:
        out = torch.empty_like(u)
    n = len(layers)
    ms = (ctypes.c_int * n)(*[int(m) for m in m_per_layer])
    pw = (ctypes.c_void_p * n)(*[t.data_ptr() for t in prenorm_w])
    ws = _workspace(matmamba_stack_workspace(layers, m_per_layer, b, L, chunk), u.device, workspace)
    rc = load().matmamba_stack_fwd(_stack_structs(layers), pw, float(prenorm_eps), n, ms, _ptr(u), b, L, int(chunk),
                                   _ptr(out), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "matmamba_stack_fwd")
    return out
