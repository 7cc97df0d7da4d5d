"""Pins for the fp64 oracle: every check here is independent of the oracle's own code.

Each test compares the oracle with something the pages or the mathematics fix:
a hand-computed worked example, closed forms (geometric series), the unrolled
O(L^2) matrix form of the recurrence, library routines (np.convolve, matmul,
logaddexp, expit, cumsum), a chunked restatement with cumulative-sum decays,
and invariants (nesting of the sub-block, causality, linearity, scale
invariance of RMSNorm, prefill/step equivalence).  A dropped term, a wrong
sign or index, or a transposed operand in the oracle fails at least one test.
"""
import json
import os

import numpy as np
import pytest
from scipy.special import expit

from nested_mamba2_selective_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- independent restatements

def quadratic_form_scan(x, dt, A, B, C, D=None, init_state=None, hpg=None):
    """Unrolled recurrence: y_t = sum_{s<=t} exp(A sum_{r=s+1..t} dt_r) (C_t.B_s) dt_s x_s
    + exp(A sum_{r<=t} dt_r) C_t^T H_0 + D x_t, each decay summed explicitly."""
    b, L, h, P = x.shape
    N = B.shape[-1]
    hpg = hpg or -(-h // B.shape[2])
    y = np.zeros((b, L, h, P))
    fs = np.zeros((b, h, P, N))
    for bb in range(b):
        for i in range(h):
            g = i // hpg
            H0 = init_state[bb, i].T if init_state is not None else np.zeros((N, P))
            for t in range(L):
                acc = np.zeros(P)
                for s in range(t + 1):
                    decay = np.exp(A[i] * np.sum(dt[bb, s + 1:t + 1, i]))
                    acc += decay * np.dot(C[bb, t, g], B[bb, s, g]) * dt[bb, s, i] * x[bb, s, i]
                acc += np.exp(A[i] * np.sum(dt[bb, :t + 1, i])) * (C[bb, t, g] @ H0)
                if D is not None:
                    acc += D[i] * x[bb, t, i]
                y[bb, t, i] = acc
            Hl = np.exp(A[i] * np.sum(dt[bb, :, i])) * H0
            for s in range(L):
                Hl = Hl + np.exp(A[i] * np.sum(dt[bb, s + 1:, i])) * dt[bb, s, i] * np.outer(B[bb, s, g], x[bb, s, i])
            fs[bb, i] = Hl.T
    return y, fs


def chunked_scan(x, dt, A, B, C, D, Q, hpg=None):
    """Chunked restatement: intra-chunk (L o C B^T)(dt x) with L from chunk-local cumulative sums,
    plus exp(cs_t) C_t^T H_prev, and H <- exp(cs_end) H + sum_s exp(cs_end - cs_s) dt_s B_s x_s^T."""
    b, L, h, P = x.shape
    N = B.shape[-1]
    hpg = hpg or -(-h // B.shape[2])
    y = np.zeros((b, L, h, P))
    for bb in range(b):
        for i in range(h):
            g = i // hpg
            H = np.zeros((N, P))
            for c0 in range(0, L, Q):
                idx = np.arange(c0, min(c0 + Q, L))
                cs = np.cumsum(dt[bb, idx, i] * A[i])
                Lm = np.tril(np.exp(cs[:, None] - cs[None, :]))
                G_ = C[bb, idx, g] @ B[bb, idx, g].T
                Xdt = dt[bb, idx, i][:, None] * x[bb, idx, i]
                yc = (Lm * G_) @ Xdt + np.exp(cs)[:, None] * (C[bb, idx, g] @ H) + D[i] * x[bb, idx, i]
                y[bb, idx, i] = yc
                w = np.exp(cs[-1] - cs) * dt[bb, idx, i]
                H = np.exp(cs[-1]) * H + B[bb, idx, g].T @ (w[:, None] * x[bb, idx, i])
    return y


def small_scan_inputs(seed, b=2, L=13, h=3, P=4, N=5, G=1):
    rng = np.random.default_rng(seed)
    return dict(x=rng.standard_normal((b, L, h, P)), dt=np.exp(rng.uniform(np.log(1e-2), np.log(0.5), (b, L, h))),
                A=-np.exp(rng.uniform(0, np.log(4), h)), B=rng.standard_normal((b, L, G, N)),
                C=rng.standard_normal((b, L, G, N)), D=rng.standard_normal(h))


def rel_err(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# ---------------------------------------------------------------- scan pins

def test_scan_hand_worked_example(orc):
    """Worked by hand (tests/golden/scan_hand.json): a = e^{dt A} = 1/2, B = 1, C = 2, x = 1,
    D = 1/4: H_t = H_{t-1}/2 + 1 -> 1, 1.5, 1.75, 1.875; y = 2 H + 0.25."""
    with open(os.path.join(GOLDEN, "scan_hand.json")) as f:
        g = json.load(f)
    L = len(g["y"])
    x = np.ones((1, L, 1, 1))
    dt = np.full((1, L, 1), g["dt"])
    A = np.array([g["A"]])
    B = np.full((1, L, 1, 1), g["B"])
    C = np.full((1, L, 1, 1), g["C"])
    y, fs = orc.ssd_scan(x, dt, A, B, C, np.array([g["D"]]))
    np.testing.assert_allclose(y[0, :, 0, 0], g["y"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(fs[0, 0, 0, 0], g["final_state"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("G,hpg,h", [(1, 3, 3), (2, 2, 4)])
@pytest.mark.parametrize("with_init", [False, True])
def test_scan_equals_unrolled_matrix_form(orc, G, hpg, h, with_init):
    inp = small_scan_inputs(1 + G + with_init, h=h, G=G)
    rng = np.random.default_rng(7)
    init = rng.standard_normal((2, h, 4, 5)) if with_init else None
    y, fs = orc.ssd_scan(**inp, init_state=init, heads_per_group=hpg)
    yq, fq = quadratic_form_scan(**inp, init_state=init, hpg=hpg)
    assert rel_err(y, yq) < 1e-12
    assert rel_err(fs, fq) < 1e-12


def test_scan_closed_form_constant_inputs(orc):
    """Constant x, B, C, dt: y_t = (C.B) dt (1 - a^t)/(1 - a) x + D x, a = e^{dt A}, t 1-based."""
    L, P, N = 40, 3, 6
    rng = np.random.default_rng(3)
    xv, Bv, Cv = rng.standard_normal(P), rng.standard_normal(N), rng.standard_normal(N)
    dtv, Av, Dv = 0.07, -2.5, 0.3
    x = np.broadcast_to(xv, (1, L, 1, P)).copy()
    B = np.broadcast_to(Bv, (1, L, 1, N)).copy()
    C = np.broadcast_to(Cv, (1, L, 1, N)).copy()
    dt = np.full((1, L, 1), dtv)
    y, _ = orc.ssd_scan(x, dt, np.array([Av]), B, C, np.array([Dv]))
    a = np.exp(dtv * Av)
    t = np.arange(1, L + 1)[:, None]
    expect = (Cv @ Bv) * dtv * (1 - a ** t) / (1 - a) * xv[None, :] + Dv * xv[None, :]
    assert rel_err(y[0, :, 0], expect) < 1e-13


def test_scan_A_zero_is_cumulative_sum(orc):
    inp = small_scan_inputs(11)
    inp["A"] = np.zeros(3)
    y, _ = orc.ssd_scan(**inp)
    x, dt, B, C, D = inp["x"], inp["dt"], inp["B"][:, :, 0], inp["C"][:, :, 0], inp["D"]
    outer = dt[..., None, None] * np.einsum("btn,bthp->bthnp", B, x)      # (b,L,h,N,P)
    Hs = np.cumsum(outer, axis=1)
    expect = np.einsum("btn,bthnp->bthp", C, Hs) + D[None, None, :, None] * x
    assert rel_err(y, expect) < 1e-12


@pytest.mark.parametrize("zero", ["B", "C"])
def test_scan_B_or_C_zero_leaves_skip_term(orc, zero):
    inp = small_scan_inputs(12)
    inp[zero] = np.zeros_like(inp[zero])
    y, _ = orc.ssd_scan(**inp)
    np.testing.assert_array_equal(y, inp["D"][None, None, :, None] * inp["x"])


def test_scan_memoryless_limit(orc):
    """dt*A -> -inf: no memory, y_t = dt_t (C_t.B_t) x_t + D x_t."""
    inp = small_scan_inputs(13)
    inp["A"] = np.full(3, -1e4)
    y, _ = orc.ssd_scan(**inp)
    cb = np.einsum("btn,btn->bt", inp["C"][:, :, 0], inp["B"][:, :, 0])
    expect = (inp["dt"] * cb[..., None])[..., None] * inp["x"] + inp["D"][None, None, :, None] * inp["x"]
    assert rel_err(y, expect) < 1e-13


@pytest.mark.parametrize("Q", [1, 2, 4, 16, 24])
def test_scan_chunk_invariance(orc, Q):
    inp = small_scan_inputs(14, L=24)
    y, _ = orc.ssd_scan(**inp)
    yc = chunked_scan(**inp, Q=Q)
    assert rel_err(yc, y) < 1e-12


def test_scan_linear_causal_batch_independent(orc):
    inp = small_scan_inputs(15)
    y1, _ = orc.ssd_scan(**inp)
    inp2 = dict(inp, x=2.5 * inp["x"])
    y2, _ = orc.ssd_scan(**inp2)
    assert rel_err(y2, 2.5 * y1) < 1e-13
    inp3 = {k: v.copy() for k, v in inp.items()}
    inp3["x"][:, 7:] += 1.0
    inp3["B"][:, 7:] -= 0.5
    y3, _ = orc.ssd_scan(**inp3)
    np.testing.assert_array_equal(y3[:, :7], y1[:, :7])
    one = {k: (v[1:2] if v.ndim >= 3 else v) for k, v in inp.items()}
    y4, _ = orc.ssd_scan(**one)
    np.testing.assert_array_equal(y4[0], y1[1])


def test_scan_state_handoff(orc):
    """Scanning [0, L1) then [L1, L) from the returned state equals one scan over [0, L)."""
    inp = small_scan_inputs(16, L=20)
    y, fs = orc.ssd_scan(**inp)
    cut = lambda a, s: a[:, s] if a.ndim >= 3 else a  # noqa: E731
    first = {k: cut(v, slice(0, 9)) for k, v in inp.items()}
    second = {k: cut(v, slice(9, 20)) for k, v in inp.items()}
    ya, sa = orc.ssd_scan(**first)
    yb, sb = orc.ssd_scan(**second, init_state=sa)
    assert rel_err(np.concatenate([ya, yb], 1), y) < 1e-13
    assert rel_err(sb, fs) < 1e-13


# ---------------------------------------------------------------- block pins

def tiny_dims(orc, G=1, eps=1e-5):
    return orc.Dims(d_model=16, d_inner=32, d_head=8, d_state=4, ngroups=G, d_conv=4, norm_eps=eps)


def tiny_params(dims, seed=5):
    p = synth.block_params(dims.d_model, dims.d_inner, dims.d_head, dims.d_state, dims.ngroups, dims.d_conv,
                           dtype="f32", seed=seed)
    p = {k: v.astype(np.float64) for k, v in p.items()}
    # spread the small init so every stage is exercised well away from zero
    for k in ("W_in", "W_out", "conv_w", "conv_b"):
        p[k] = p[k] * 25.0
    return p


@pytest.mark.parametrize("m", [16, 8, 4])
def test_block_stages_against_library_routines(orc, m):
    dims = tiny_dims(orc)
    p = tiny_params(dims)
    rng = np.random.default_rng(20 + m)
    u = rng.standard_normal((2, 11, 16))
    out, tr = orc.block_fwd(dims, p, u, m, trace=True)
    d, h = orc.width(dims, m)
    E, GN, K = dims.d_inner, dims.d_state, dims.d_conv
    W = p["W_in"]
    z = np.matmul(u, W[0:d].T)
    v = np.concatenate([np.matmul(u, W[E:E + d].T), np.matmul(u, W[2 * E:2 * E + 2 * GN].T)], -1)
    r = np.matmul(u, W[2 * E + 2 * GN:2 * E + 2 * GN + h].T)
    assert rel_err(tr["z"], z) < 1e-13
    rows = list(range(d)) + list(range(E, E + 2 * GN))
    conv = np.zeros_like(v)
    for bb in range(2):
        for c, row in enumerate(rows):
            conv[bb, :, c] = np.convolve(v[bb, :, c], p["conv_w"][row][::-1], mode="full")[:11] + p["conv_b"][row]
    xbc = conv * expit(conv)
    assert rel_err(tr["xbc"], xbc) < 1e-13
    dt = np.logaddexp(0.0, r + p["dt_bias"][:h])
    assert rel_err(tr["dt"], dt) < 1e-13
    x = xbc[..., :d].reshape(2, 11, h, dims.d_head)
    yq, _ = quadratic_form_scan(x, dt, p["A"][:h], xbc[..., d:d + GN][:, :, None], xbc[..., d + GN:][:, :, None],
                                p["D"][:h], hpg=dims.nheads)
    assert rel_err(tr["y"], yq.reshape(2, 11, d)) < 1e-12
    # gate + RMSNorm: n / norm_w is parallel to y*SiLU(z) and has RMS 1/sqrt(1 + eps/mean(q^2))
    q = tr["y"] * z * expit(z)
    ratio = tr["nrm"] / p["norm_w"][:d]
    scale = ratio / q
    assert np.max(np.abs(scale - scale[..., :1])) < 1e-12 * np.max(np.abs(scale))
    ms = np.mean(q * q, -1)
    np.testing.assert_allclose(np.sqrt(np.mean(ratio * ratio, -1)), 1 / np.sqrt(1 + dims.norm_eps / ms), rtol=1e-12)
    assert rel_err(out, np.matmul(tr["nrm"], p["W_out"][:, :d].T)) < 1e-13


def test_rmsnorm_unit_rms_and_scale_invariance(orc):
    rng = np.random.default_rng(30)
    v = rng.standard_normal((5, 33))
    w = np.ones(33)
    n = orc.rmsnorm_rows(v, w, 0.0)
    np.testing.assert_allclose(np.mean(n * n, -1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(orc.rmsnorm_rows(7.0 * v, w, 0.0), n, rtol=1e-13)
    w2 = rng.standard_normal(33)
    np.testing.assert_allclose(orc.rmsnorm_rows(v, w2, 0.0), n * w2, rtol=1e-13)


def test_rmsnorm_with_eps_closed_form(orc):
    """With eps > 0 the output keeps each row's direction and has RMS 1/sqrt(1 + eps/mean(v^2)): the
    textbook definition v / sqrt(mean(v^2) + eps), checked through that closed form."""
    rng = np.random.default_rng(31)
    v = rng.standard_normal((6, 40)) * np.array([1e-3, 0.1, 1.0, 3.0, 10.0, 0.02])[:, None]
    w = np.ones(40)
    for eps in (1e-5, 1e-2, 0.5):
        n = orc.rmsnorm_rows(v, w, eps)
        ms = np.mean(v * v, -1)
        np.testing.assert_allclose(np.sqrt(np.mean(n * n, -1)), 1.0 / np.sqrt(1.0 + eps / ms), rtol=1e-12)
        ratio = n / v
        np.testing.assert_allclose(ratio, np.broadcast_to(ratio[:, :1], ratio.shape), rtol=1e-12)
        assert np.all(ratio > 0)


def sliced_params(dims, p, d, h):
    E, GN = dims.d_inner, dims.ngroups * dims.d_state
    W = p["W_in"]
    return dict(
        W_in=np.concatenate([W[0:d], W[E:E + d], W[2 * E:2 * E + 2 * GN], W[2 * E + 2 * GN:2 * E + 2 * GN + h]]),
        conv_w=np.concatenate([p["conv_w"][0:d], p["conv_w"][E:E + 2 * GN]]),
        conv_b=np.concatenate([p["conv_b"][0:d], p["conv_b"][E:E + 2 * GN]]),
        dt_bias=p["dt_bias"][:h].copy(), A=p["A"][:h].copy(), D=p["D"][:h].copy(),
        norm_w=p["norm_w"][:d].copy(), W_out=np.ascontiguousarray(p["W_out"][:, :d]))


@pytest.mark.parametrize("m", [8, 4, 12])
def test_nesting_invariant(orc, m):
    """M_i on the full weights equals the full-width block on explicitly sliced weights (exact)."""
    dims = tiny_dims(orc)
    p = tiny_params(dims)
    u = np.random.default_rng(40 + m).standard_normal((2, 9, 16))
    d, h = orc.width(dims, m)
    sub = orc.Dims(dims.d_model, d, dims.d_head, dims.d_state, 1, dims.d_conv, dims.norm_eps)
    np.testing.assert_array_equal(orc.block_fwd(dims, p, u, m), orc.block_fwd(sub, sliced_params(dims, p, d, h), u, 16))


def test_width_rule(orc):
    dims = tiny_dims(orc)       # e = 2, d_head = 8: valid m are multiples of 4 up to 16
    assert orc.width(dims, 16) == (32, 4) and orc.width(dims, 4) == (8, 1) and orc.width(dims, 12) == (24, 3)
    for m in (0, -4, 2, 6, 17, 20):
        assert orc.width(dims, m) is None
    with pytest.raises(ValueError):
        orc.block_fwd(dims, tiny_params(dims), np.zeros((1, 2, 16)), 6)


def test_block_causal_and_batch_independent(orc):
    dims = tiny_dims(orc)
    p = tiny_params(dims)
    u = np.random.default_rng(50).standard_normal((3, 12, 16))
    o1 = orc.block_fwd(dims, p, u, 8)
    u2 = u.copy()
    u2[:, 6:] *= -3.0
    o2 = orc.block_fwd(dims, p, u2, 8)
    np.testing.assert_array_equal(o2[:, :6], o1[:, :6])
    np.testing.assert_array_equal(orc.block_fwd(dims, p, u[2:3], 8)[0], o1[2])


@pytest.mark.parametrize("m", [16, 8])
def test_prefill_then_step_equals_longer_prefill(orc, m):
    dims = tiny_dims(orc)
    p = tiny_params(dims)
    H, P, N = dims.nheads, dims.d_head, dims.d_state
    rows = dims.d_inner + 2 * N
    u = np.random.default_rng(60 + m).standard_normal((2, 10, 16))
    s = np.zeros((2, H, P, N))
    c = np.zeros((2, rows, 3))
    out9 = orc.block_fwd(dims, p, u[:, :9], m, ssm_state_out=s, conv_state_out=c)
    step = orc.block_step(dims, p, u[:, 9], m, s, c)
    s10 = np.zeros_like(s)
    c10 = np.zeros_like(c)
    out10 = orc.block_fwd(dims, p, u, m, ssm_state_out=s10, conv_state_out=c10)
    assert rel_err(step, out10[:, 9]) < 1e-12
    assert rel_err(out9, out10[:, :9]) < 1e-15
    assert rel_err(s, s10) < 1e-12
    np.testing.assert_array_equal(c, c10)
    # L steps from the zero state reproduce the prefill
    s0 = np.zeros_like(s)
    c0 = np.zeros_like(c)
    outs = np.stack([orc.block_step(dims, p, u[:, t], m, s0, c0) for t in range(10)], 1)
    assert rel_err(outs, out10) < 1e-12


def test_conv_state_holds_last_inputs(orc):
    """After a prefill the conv state holds the last d_conv-1 pre-conv inputs (oldest first); untouched
    rows (inactive x channels) keep their contents."""
    dims = tiny_dims(orc)
    p = tiny_params(dims)
    u = np.random.default_rng(70).standard_normal((1, 5, 16))
    c = np.full((1, dims.d_inner + 2 * dims.d_state, 3), 9.0)
    orc.block_fwd(dims, p, u, 8, conv_state_out=c)
    d = 16
    W = p["W_in"]
    v_x = np.matmul(u[0], W[dims.d_inner:dims.d_inner + d].T)
    np.testing.assert_allclose(c[0, :d].T, v_x[2:5], rtol=1e-13)
    assert np.all(c[0, d:dims.d_inner] == 9.0)


def test_stack_composition_and_mix_n_match(orc):
    dims = tiny_dims(orc)
    params = [tiny_params(dims, seed=80 + l) for l in range(3)]
    wts = [1.0 + 0.1 * np.random.default_rng(90 + l).standard_normal(16) for l in range(3)]
    u = np.random.default_rng(99).standard_normal((2, 7, 16))
    ms = [16, 4, 12]
    out = orc.stack_fwd(dims, 3, lambda l: params[l], lambda l: wts[l], u, ms)
    x = u.copy()
    for l in range(3):
        n = x / np.sqrt(np.mean(x * x, -1, keepdims=True) + 1e-5) * wts[l]
        x = x + orc.block_fwd(dims, params[l], n, ms[l])
    assert rel_err(out, x) < 1e-13


def test_stack_with_zero_output_projections_is_the_identity(orc):
    """All W_out = 0: every block adds exactly zero to the residual stream, so the stack returns its
    input bit for bit, whatever the other weights and widths (a dropped or doubled residual, or a
    residual added to the normed stream, fails)."""
    dims = tiny_dims(orc)
    params = []
    for l in range(4):
        p = tiny_params(dims, seed=120 + l)
        p["W_out"] = np.zeros_like(p["W_out"])
        params.append(p)
    wts = [1.0 + 0.3 * np.random.default_rng(130 + l).standard_normal(16) for l in range(4)]
    u = np.random.default_rng(140).standard_normal((2, 9, 16)) * 3.0
    out = orc.stack_fwd(dims, 4, lambda l: params[l], lambda l: wts[l], u, [16, 4, 12, 8])
    np.testing.assert_array_equal(out, u)
    # and a single non-zero W_out changes it: the pin is not vacuous
    params[2] = tiny_params(dims, seed=122)
    out2 = orc.stack_fwd(dims, 4, lambda l: params[l], lambda l: wts[l], u, [16, 4, 12, 8])
    assert np.max(np.abs(out2 - u)) > 1e-6


@pytest.mark.parametrize("name,expect", [("block_tiny_f32", 0.966), ("block_130m_b8_L2048", 0.997),
                                         ("stack48_1p4b_b4_L4096", 0.999)])
def test_projection_parameter_share(name, expect):
    """More than 95% of a block's parameters sit in the in/out projections."""
    w = synth.WORKLOADS[name]
    E, GN, H = w.d_inner, w.ngroups * w.d_state, w.d_inner // w.d_head
    proj = (2 * E + 2 * GN + H) * w.d_model + w.d_model * E
    rest = (E + 2 * GN) * (w.d_conv + 1) + 3 * H + E
    share = proj / (proj + rest)
    assert share > 0.95 and abs(share - expect) < 1e-3
