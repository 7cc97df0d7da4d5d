"""fp64 CPU oracle for the MatMamba block at a Matryoshka width (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this module; the product path
(``nested_mamba2_selective_b200``) never does.

The arithmetic lives in ``oracle.c`` (plain C, fp64, sequential recurrence);
this file only builds it with gcc, marshals numpy arrays through ctypes, and
composes the per-block oracle into the stacked model and the one-token
recurrent step:

* stack: "MatMamba: A Matryoshka State Space Model", stacking paragraph -- a
  model f_i is L blocks M_i stacked.  The pages give no residual form; the
  reading taken is the pre-norm residual u <- u + M_i(RMSNorm(u) * w_l), with
  no final norm.
* decode step: "Mamba: Linear-Time Sequence Modeling with Selective State
  Spaces" (summary page), strengths list -- linear-time recurrent inference
  with no KV cache.  One step is the block on a single token with the SSM state
  and the last d_conv-1 pre-conv inputs carried across calls.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into oracle/liboracle.so (gcc, fp64, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
               _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Dims(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("d_inner", ctypes.c_int), ("d_head", ctypes.c_int),
                ("d_state", ctypes.c_int), ("ngroups", ctypes.c_int), ("d_conv", ctypes.c_int),
                ("norm_eps", ctypes.c_double)]


_dp = ctypes.POINTER(ctypes.c_double)


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.orc_width.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                  ctypes.POINTER(ctypes.c_int)]
        lib.orc_ssd_scan.argtypes = [ctypes.c_int] * 7 + [_dp] * 6 + [_dp, _dp, _dp]
        lib.orc_rmsnorm_rows.argtypes = [ctypes.c_int, ctypes.c_int, _dp, _dp, ctypes.c_double, _dp]
        lib.orc_block_fwd.argtypes = ([ctypes.POINTER(_Dims)] + [_dp] * 8 + [ctypes.c_int] * 3 + [_dp]
                                      + [_dp] * 2 + [_dp] * 3 + [_dp] * 5)
        lib.orc_num_threads.argtypes = []
        _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_dp)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


@dataclass(frozen=True)
class Dims:
    d_model: int
    d_inner: int
    d_head: int
    d_state: int
    ngroups: int = 1
    d_conv: int = 4
    norm_eps: float = 1e-5

    @property
    def nheads(self) -> int:
        return self.d_inner // self.d_head

    def _c(self) -> _Dims:
        return _Dims(self.d_model, self.d_inner, self.d_head, self.d_state, self.ngroups, self.d_conv,
                     self.norm_eps)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def width(dims: Dims, m: int):
    """(d_i, h_i) for width m, or None when m is not a valid Matryoshka width."""
    d, h = ctypes.c_int(), ctypes.c_int()
    if _load().orc_width(ctypes.byref(dims._c()), int(m), ctypes.byref(d), ctypes.byref(h)):
        return None
    return d.value, h.value


def ssd_scan(x, dt, A, B, C, D=None, init_state=None, heads_per_group=None, want_state=True):
    """Sequential scan.  x (b,L,h,P), dt (b,L,h), A (h), B/C (b,L,G,N), D (h) or None,
    init_state (b,h,P,N) or None.  Returns (y, final_state)."""
    x, dt, A, B, C, D, init_state = map(_f64, (x, dt, A, B, C, D, init_state))
    b, L, h, P = x.shape
    G, N = B.shape[2], B.shape[3]
    hpg = heads_per_group if heads_per_group is not None else max(1, -(-h // G))
    y = np.zeros_like(x)
    fs = np.zeros((b, h, P, N)) if want_state else None
    rc = _load().orc_ssd_scan(b, L, h, P, N, G, hpg, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                              _ptr(init_state), _ptr(y), _ptr(fs))
    if rc:
        raise ValueError("oracle ssd_scan rejected the shapes")
    return y, fs


def rmsnorm_rows(v, w, eps):
    v, w = _f64(v), _f64(w)
    out = np.empty_like(v)
    rows, cols = v.reshape(-1, v.shape[-1]).shape
    _load().orc_rmsnorm_rows(rows, cols, _ptr(v), _ptr(w), float(eps), _ptr(out))
    return out


def block_fwd(dims: Dims, p: dict, u, m: int, ssm_state_in=None, conv_state_in=None,
              ssm_state_out=None, conv_state_out=None, trace: bool = False):
    """Block forward at width m.  p holds full-width fp64 arrays W_in, conv_w, conv_b,
    dt_bias, A, D, norm_w, W_out.  ssm_state_out / conv_state_out, when given, are
    fp64 arrays updated in place (only the active heads / conv rows).
    Returns out, or (out, trace dict) with trace=True."""
    wd = width(dims, m)
    if wd is None:
        raise ValueError("invalid Matryoshka width %d" % m)
    d, h = wd
    u = _f64(u)
    b, L, Dm = u.shape
    out = np.zeros((b, L, Dm))
    GN = dims.ngroups * dims.d_state
    tr = None
    if trace:
        tr = dict(z=np.zeros((b, L, d)), xbc=np.zeros((b, L, d + 2 * GN)), dt=np.zeros((b, L, h)),
                  y=np.zeros((b, L, d)), nrm=np.zeros((b, L, d)))
    args = [_f64(p[k]) for k in ("W_in", "conv_w", "conv_b", "dt_bias", "A", "D", "norm_w", "W_out")]
    for a_out in (ssm_state_out, conv_state_out):
        assert a_out is None or (a_out.dtype == np.float64 and a_out.flags["C_CONTIGUOUS"])
    rc = _load().orc_block_fwd(
        ctypes.byref(dims._c()), *[_ptr(a) for a in args], b, L, int(m), _ptr(u),
        _ptr(_f64(ssm_state_in)), _ptr(_f64(conv_state_in)),
        _ptr(out), _ptr(ssm_state_out), _ptr(conv_state_out),
        *[_ptr(tr[k]) if tr else None for k in ("z", "xbc", "dt", "y", "nrm")])
    if rc:
        raise ValueError("oracle block_fwd rejected the shapes")
    return (out, tr) if trace else out


def block_step(dims: Dims, p: dict, u_t, m: int, ssm_state, conv_state):
    """One recurrent token for every sequence: u_t (b, d_model).  ssm_state (b,H,P,N) and
    conv_state (b, E+2GN, d_conv-1) are fp64 arrays updated in place (active part only)."""
    u_t = _f64(u_t)
    s_in, c_in = ssm_state.copy(), conv_state.copy()
    out = block_fwd(dims, p, u_t[:, None, :], m, ssm_state_in=s_in, conv_state_in=c_in,
                    ssm_state_out=ssm_state, conv_state_out=conv_state)
    return out[:, 0, :]


def stack_fwd(dims: Dims, nlayers: int, layer_params, prenorm_w, u, m_per_layer, prenorm_eps=1e-5):
    """Pre-norm residual stack: u <- u + block_l(RMSNorm(u) * w_l) for l in range(nlayers).
    layer_params(l) -> dict of fp64 arrays; prenorm_w(l) -> (d_model,) fp64 array."""
    x = _f64(u).copy()
    for l in range(nlayers):
        nrm = rmsnorm_rows(x, prenorm_w(l), prenorm_eps)
        x = x + block_fwd(dims, layer_params(l), nrm, int(m_per_layer[l]))
    return x
