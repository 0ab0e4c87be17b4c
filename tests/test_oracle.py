"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: a value
worked by hand, a closed form, an identity the pages state, brute force on
a tiny input, or finite differences.  Together they are chosen so that a
plausible slip in the oracle (a dropped term, a wrong sign, a swapped B/C,
a wrong index or stride) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def rng(seed):
    return np.random.default_rng(seed)


def rand_case(seed, batch=2, dim=3, L=16, N=4, z=True, D=True, bias=True):
    r = rng(seed)
    c = dict(u=r.standard_normal((batch, dim, L)),
             delta=r.standard_normal((batch, dim, L)),
             A=-np.exp(r.standard_normal((dim, N))),
             B=r.standard_normal((batch, N, L)),
             C=r.standard_normal((batch, N, L)),
             D=r.uniform(0.5, 1.5, dim) if D else None,
             z=r.standard_normal((batch, dim, L)) if z else None,
             delta_bias=np.log(np.expm1(r.uniform(1e-3, 0.1, dim))) if bias else None)
    return c


# ----------------------------------------------------------------- forward pins

def test_golden_lti_impulse_kernel():
    """Impulse response = the LTI convolution kernel K (page-3 §2), worked by hand."""
    vals = {}
    with open(os.path.join(HERE, "golden", "lti_impulse_kernel.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, *v = line.split()
            vals[k] = np.array([float(x) for x in v])
    L = len(vals["u"])
    u = vals["u"].reshape(1, 1, L)
    delta = np.full((1, 1, L), vals["delta"][0])
    A = vals["A"].reshape(1, 1)
    B = np.full((1, 1, L), vals["B"][0])
    C = np.full((1, 1, L), vals["C"][0])
    out, last = oracle.fwd(u, delta, A, B, C, D=np.zeros(1), delta_softplus=False)
    np.testing.assert_allclose(out[0, 0], vals["y"], rtol=1e-14, atol=0)
    assert abs(last[0, 0, 0] - 0.75 * 0.5 ** (L - 1)) < 1e-15


def test_hand_unrolled_n1_l3():
    """N=1, L=3 with time-varying Δ, B, C, written out step by step."""
    x = [0.5, -1.0, 2.0]
    dt = [0.25, 1.0, 0.5]
    Bv = [2.0, -0.5, 1.0]
    Cv = [1.0, 3.0, -2.0]
    a, Dd = -1.5, 0.75
    h1 = dt[0] * Bv[0] * x[0]
    h2 = math.exp(dt[1] * a) * h1 + dt[1] * Bv[1] * x[1]
    h3 = math.exp(dt[2] * a) * h2 + dt[2] * Bv[2] * x[2]
    want = [Cv[0] * h1 + Dd * x[0], Cv[1] * h2 + Dd * x[1], Cv[2] * h3 + Dd * x[2]]
    out, last = oracle.fwd(np.array(x).reshape(1, 1, 3), np.array(dt).reshape(1, 1, 3),
                           np.array([[a]]), np.array(Bv).reshape(1, 1, 3),
                           np.array(Cv).reshape(1, 1, 3), D=np.array([Dd]),
                           delta_softplus=False)
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-15, atol=1e-15)
    assert abs(last[0, 0, 0] - h3) < 1e-15


def test_hand_unrolled_two_states_two_channels():
    """dim=2, N=2, L=2: checks the [d][n] layout of A and the [b][n][t] layout of B, C."""
    A = np.array([[-1.0, -2.0], [-0.5, -3.0]])
    x = np.array([[1.0, 2.0], [-1.0, 0.5]])          # [d][t]
    dt = np.array([[0.5, 0.25], [1.0, 2.0]])         # [d][t]
    Bm = np.array([[1.0, -1.0], [2.0, 0.5]])         # [n][t]
    Cm = np.array([[0.5, 1.5], [-1.0, 2.0]])         # [n][t]
    want = np.zeros((2, 2))
    for d in range(2):
        h = [0.0, 0.0]
        for t in range(2):
            y = 0.0
            for n in range(2):
                h[n] = math.exp(dt[d, t] * A[d, n]) * h[n] + dt[d, t] * Bm[n, t] * x[d, t]
                y += Cm[n, t] * h[n]
            want[d, t] = y
    out, _ = oracle.fwd(x[None], dt[None], A, Bm[None], Cm[None], delta_softplus=False)
    np.testing.assert_allclose(out[0], want, rtol=1e-15, atol=1e-15)


def test_lti_equals_bruteforce_convolution():
    """Constant Δ, B, C (LTI): recurrence == causal conv with K_k = Σ_n C ā^k Δ B."""
    r = rng(1)
    batch, dim, N, L = 2, 3, 4, 256
    A = -np.exp(r.standard_normal((dim, N)))
    dconst = r.uniform(0.01, 0.5, (batch, dim))
    Bc = r.standard_normal((batch, N))
    Cc = r.standard_normal((batch, N))
    Dv = r.uniform(0.5, 1.5, dim)
    u = r.standard_normal((batch, dim, L))
    delta = np.repeat(dconst[:, :, None], L, axis=2)
    B = np.repeat(Bc[:, :, None], L, axis=2)
    C = np.repeat(Cc[:, :, None], L, axis=2)
    out, _ = oracle.fwd(u, delta, A, B, C, D=Dv, delta_softplus=False)
    k = np.arange(L)
    for b in range(batch):
        for d in range(dim):
            dt = dconst[b, d]
            abar = np.exp(dt * A[d])                                     # [N]
            K = (Cc[b][None, :] * abar[None, :] ** k[:, None] * dt * Bc[b][None, :]).sum(1)
            want = np.array([np.dot(K[:t + 1][::-1], u[b, d, :t + 1]) for t in range(L)])
            want += Dv[d] * u[b, d]
            np.testing.assert_allclose(out[b, d], want, rtol=1e-11, atol=1e-12)


def test_A_zero_is_running_sum():
    """A = 0 makes ā = 1: h_t is a cumulative sum of Δ_s B_s u_s."""
    r = rng(2)
    batch, dim, N, L = 2, 3, 5, 100
    u = r.standard_normal((batch, dim, L))
    delta = r.uniform(0.0, 2.0, (batch, dim, L))
    B = r.standard_normal((batch, N, L))
    C = r.standard_normal((batch, N, L))
    out, last = oracle.fwd(u, delta, np.zeros((dim, N)), B, C, delta_softplus=False)
    inc = delta[:, :, None, :] * B[:, None, :, :] * u[:, :, None, :]    # [b,d,n,t]
    h = np.cumsum(inc, axis=3)
    want = (C[:, None, :, :] * h).sum(2)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(last, h[..., -1], rtol=1e-12, atol=1e-12)


def test_delta_zero_keeps_state_zero():
    """Δ = 0: nothing enters the state, so out = D u (no gate) and h stays 0."""
    c = rand_case(3, z=False)
    zeros = np.zeros_like(c["u"])
    out, last = oracle.fwd(c["u"], zeros, c["A"], c["B"], c["C"], D=c["D"],
                           delta_softplus=False)
    np.testing.assert_array_equal(last, 0.0)
    np.testing.assert_allclose(out, c["D"][None, :, None] * c["u"], rtol=0, atol=0)


def test_gate_identity():
    """silu(z) - silu(-z) = z, so out(z) - out(-z) = y * z with y the ungated output."""
    c = rand_case(4)
    args = (c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"])
    y, _ = oracle.fwd(*args, z=None, delta_bias=c["delta_bias"])
    op, _ = oracle.fwd(*args, z=c["z"], delta_bias=c["delta_bias"])
    om, _ = oracle.fwd(*args, z=-c["z"], delta_bias=c["delta_bias"])
    np.testing.assert_allclose(op - om, y * c["z"], rtol=1e-12, atol=1e-12)
    # z = 0 closes the gate completely
    o0, _ = oracle.fwd(*args, z=np.zeros_like(c["z"]), delta_bias=c["delta_bias"])
    np.testing.assert_array_equal(o0, 0.0)


def test_softplus_identities():
    """With A=0, B=C=u=1, N=1, y_t = Σ_{s<=t} Δ_s; checks softplus(0)=ln2 and
    softplus(r) - softplus(-r) = r, plus both tails."""
    L = 1
    one = np.ones((1, 1, L))

    def dt_of(r, bias=None):
        out, _ = oracle.fwd(one, np.full((1, 1, L), r), np.zeros((1, 1)), one, one,
                            delta_bias=bias, delta_softplus=True)
        return out[0, 0, 0]

    assert abs(dt_of(0.0) - math.log(2.0)) < 1e-16
    for r in (0.3, 1.7, 5.0, 19.0):
        assert abs(dt_of(r) - dt_of(-r) - r) < 1e-13 * max(1.0, r)
    assert abs(dt_of(50.0) - 50.0) < 1e-13
    assert 0.0 < dt_of(-50.0) < 2e-22
    # bias is added before the softplus
    assert abs(dt_of(0.25, np.array([-0.25])) - math.log(2.0)) < 1e-16


def test_large_delta_erases_memory():
    """Large Δ with A <= -1 drives ā to ~0, so h_t ≈ Δ B_t u_t (the state is reset)."""
    r = rng(5)
    batch, dim, N, L = 1, 2, 3, 20
    u = r.standard_normal((batch, dim, L))
    B = r.standard_normal((batch, N, L))
    C = r.standard_normal((batch, N, L))
    A = -1.0 - r.uniform(0, 1, (dim, N))
    dt = 60.0
    out, _ = oracle.fwd(u, np.full_like(u, dt), A, B, C, delta_softplus=False)
    want = dt * (C * B).sum(1)[:, None, :] * u
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)


def test_state_permutation_invariance():
    """A is diagonal: permuting the state index in A, B, C leaves y unchanged."""
    c = rand_case(6, N=8)
    perm = rng(7).permutation(8)
    out, last = oracle.fwd(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                           c["delta_bias"])
    outp, lastp = oracle.fwd(c["u"], c["delta"], c["A"][:, perm], c["B"][:, perm],
                             c["C"][:, perm], c["D"], c["z"], c["delta_bias"])
    np.testing.assert_allclose(outp, out, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lastp, last[:, :, perm], rtol=1e-13, atol=1e-13)


def test_split_sequence_carries_state():
    """O(N) state: running the second half from the first half's final state
    equals one pass over the whole sequence."""
    c = rand_case(8, L=64)
    full, lastf = oracle.fwd(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                             c["delta_bias"])
    h = 29

    def part(sl, h0=None):
        return oracle.fwd(c["u"][..., sl], c["delta"][..., sl], c["A"], c["B"][..., sl],
                          c["C"][..., sl], c["D"], c["z"][..., sl], c["delta_bias"], h0=h0)
    o1, l1 = part(slice(0, h))
    o2, l2 = part(slice(h, 64), l1)
    np.testing.assert_allclose(np.concatenate([o1, o2], -1), full, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(l2, lastf, rtol=1e-13, atol=1e-13)


def _combine(later, earlier):
    """(A_j, b_j) • (A_i, b_i) = (A_j A_i, A_j b_i + b_j) -- page-4 §2.2."""
    Aj, bj = later
    Ai, bi = earlier
    return Aj * Ai, Aj * bi + bj


def test_step_hand_computed_two_states():
    """One decoding step from a nonzero state, written out by hand: N=2,
    softplus on, gate on (h' = exp(Δa) h + Δ B u, y = C·h' + D u, y z σ(z))."""
    h = np.array([[[0.3, -1.2]]])
    a = np.array([[-0.7, -2.0]])
    Bv, Cv = np.array([[1.5, -0.25]]), np.array([[-1.0, 2.0]])
    x, r, zz, Dd, bias = 0.8, -0.4, 1.3, 0.6, 0.1
    dt = math.log1p(math.exp(r + bias))
    h_new = [math.exp(dt * a[0, n]) * h[0, 0, n] + dt * Bv[0, n] * x for n in range(2)]
    y = Cv[0, 0] * h_new[0] + Cv[0, 1] * h_new[1] + Dd * x
    want = y * zz / (1.0 + math.exp(-zz))
    out, st = oracle.step(h, np.array([[x]]), np.array([[r]]), a, Bv, Cv, D=np.array([Dd]),
                          z=np.array([[zz]]), delta_bias=np.array([bias]))
    assert abs(out[0, 0] - want) < 1e-14
    np.testing.assert_allclose(st[0, 0], h_new, rtol=1e-14, atol=1e-15)


def test_steps_reproduce_the_scan():
    """L single steps started from zero give the scan's outputs and final state."""
    c = rand_case(21, batch=2, dim=3, L=9, N=4)
    out, last = oracle.fwd(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                           c["delta_bias"], True)
    st = np.zeros((2, 3, 4))
    for t in range(9):
        y, st = oracle.step(st, c["u"][..., t], c["delta"][..., t], c["A"], c["B"][..., t],
                            c["C"][..., t], c["D"], c["z"][..., t], c["delta_bias"], True)
        np.testing.assert_allclose(y, out[..., t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st, last, rtol=1e-12, atol=1e-13)


def test_combine_operator_is_associative():
    r = rng(9)
    for _ in range(100):
        a, b, c = [(r.uniform(0, 1), r.standard_normal()) for _ in range(3)]
        x = _combine(c, _combine(b, a))
        y = _combine(_combine(c, b), a)
        assert abs(x[0] - y[0]) <= 1e-15 * abs(x[0]) + 1e-300
        assert abs(x[1] - y[1]) <= 1e-14 * (abs(x[1]) + 1)


@pytest.mark.parametrize("chunk", [1, 3, 64, 200])
def test_chunked_two_level_scan_matches_oracle(chunk):
    """A two-level scan (per-chunk (∏ā, local state) pairs, an exclusive scan
    of the pairs across chunks with the associative operator, then a fix-up of
    every step from its chunk's carry-in) reproduces the sequential oracle."""
    r = rng(10)
    batch, dim, N, L = 1, 2, 3, 200
    u = r.standard_normal((batch, dim, L))
    dt = r.uniform(0.0, 0.3, (batch, dim, L))
    A = -np.exp(r.standard_normal((dim, N)))
    B = r.standard_normal((batch, N, L))
    C = r.standard_normal((batch, N, L))
    want, wlast = oracle.fwd(u, dt, A, B, C, delta_softplus=False)
    abar = np.exp(dt[:, :, None, :] * A[None, :, :, None])          # [b,d,n,t]
    beta = dt[:, :, None, :] * B[:, None, :, :] * u[:, :, None, :]
    nchunk = -(-L // chunk)
    pairs = []
    for k in range(nchunk):          # level 1: reduce each chunk to one pair
        acc = (np.ones_like(abar[..., 0]), np.zeros_like(beta[..., 0]))
        for t in range(k * chunk, min(L, (k + 1) * chunk)):
            acc = _combine((abar[..., t], beta[..., t]), acc)
        pairs.append(acc)
    carry = [np.zeros_like(beta[..., 0])]
    for k in range(1, nchunk):       # level 2: scan of chunk pairs
        carry.append(_combine(pairs[k - 1], (1.0, carry[-1]))[1])
    y = np.zeros((batch, dim, L))
    for k in range(nchunk):          # fix-up: rerun each chunk from its carry-in
        h = carry[k]
        for t in range(k * chunk, min(L, (k + 1) * chunk)):
            h = abar[..., t] * h + beta[..., t]
            y[..., t] = (C[:, None, :, t] * h).sum(2)
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h, wlast, rtol=1e-12, atol=1e-12)


def test_zoh_matches_ode_solution():
    """The ZOH discretisation (page-4 §2.1) is the exact solution of
    h' = A h + B u over a step of length Δ with u held constant; compare with
    a fine RK4 integration of that ODE."""
    r = rng(11)
    L, N = 6, 2
    u = r.standard_normal((1, 1, L))
    dt = r.uniform(0.05, 0.8, (1, 1, L))
    A = np.array([[-0.7, -2.5]])
    B = r.standard_normal((1, N, L))
    C = r.standard_normal((1, N, L))
    out, last = oracle.fwd(u, dt, A, B, C, delta_softplus=False, zoh=True)
    h = np.zeros(N)
    ys = []
    for t in range(L):
        f = lambda hh: A[0] * hh + B[0, :, t] * u[0, 0, t]
        steps = 2000
        s = dt[0, 0, t] / steps
        for _ in range(steps):
            k1 = f(h); k2 = f(h + 0.5 * s * k1); k3 = f(h + 0.5 * s * k2); k4 = f(h + s * k3)
            h = h + s / 6 * (k1 + 2 * k2 + 2 * k3 + k4)
        ys.append((C[0, :, t] * h).sum())
    np.testing.assert_allclose(out[0, 0], ys, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(last[0, 0], h, rtol=1e-10, atol=1e-12)
    # as A -> 0 the ZOH B̄ tends to Δ B
    o1, _ = oracle.fwd(u, dt, np.full((1, N), -1e-9), B, C, delta_softplus=False, zoh=True)
    o2, _ = oracle.fwd(u, dt, np.full((1, N), -1e-9), B, C, delta_softplus=False, zoh=False)
    np.testing.assert_allclose(o1, o2, rtol=1e-7, atol=1e-9)


def test_threads_do_not_change_results():
    c = rand_case(12, batch=3, dim=5, L=40)
    o1, l1 = oracle.fwd(**c, nthreads=1)
    o4, l4 = oracle.fwd(**c, nthreads=4)
    np.testing.assert_array_equal(o1, o4)
    np.testing.assert_array_equal(l1, l4)


# ----------------------------------------------------------------- adjoint pins

def _loss(c, dout, softplus, zoh=False):
    out, _ = oracle.fwd(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                        c["delta_bias"], delta_softplus=softplus, zoh=zoh, nthreads=1)
    return float((out * dout).sum())


GRAD_OF = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
           "z": "dz", "delta_bias": "ddelta_bias"}


@pytest.mark.parametrize("softplus,gate,skip", [(True, True, True), (False, False, False),
                                                (True, False, True)])
def test_adjoint_matches_central_differences(softplus, gate, skip):
    """Every gradient of the adjoint against central finite differences of the
    (independently pinned) forward, element by element."""
    c = rand_case(13, batch=1, dim=3, L=12, N=4, z=gate, D=skip, bias=softplus)
    dout = rng(14).standard_normal(c["u"].shape)
    g = oracle.bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                   c["delta_bias"], softplus, dout, nthreads=1)
    for name, gname in GRAD_OF.items():
        if c[name] is None:
            assert gname not in g
            continue
        theta = c[name]
        fd = np.zeros_like(theta)
        for idx in np.ndindex(theta.shape):
            old = theta[idx]
            h = 1e-6 * max(1.0, abs(old))
            theta[idx] = old + h
            fp = _loss(c, dout, softplus)
            theta[idx] = old - h
            fm = _loss(c, dout, softplus)
            theta[idx] = old
            fd[idx] = (fp - fm) / (2 * h)
        scale = max(1.0, np.abs(fd).max())
        np.testing.assert_allclose(g[gname], fd, rtol=0, atol=1e-6 * scale,
                                   err_msg=f"gradient {gname}")


@pytest.mark.parametrize("a_scale", [1.0, 1e-5, 0.0])
def test_zoh_adjoint_matches_central_differences(a_scale):
    """The zero-order-hold adjoint against central differences of the ZOH
    forward (itself pinned to an RK4 solution), for ordinary A, for |Δ A|
    small enough to take the series branch of dk/dA, and for A = 0 entries."""
    c = rand_case(31, batch=1, dim=3, L=10, N=4)
    c["A"] = c["A"] * a_scale
    if a_scale == 0.0:
        c["A"][0, 1] = -0.5            # mixed: zero and nonzero A in one channel
    dout = rng(32).standard_normal(c["u"].shape)
    g = oracle.bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                   c["delta_bias"], True, dout, zoh=True, nthreads=1)
    for name, gname in GRAD_OF.items():
        theta = c[name]
        fd = np.zeros_like(theta)
        for idx in np.ndindex(theta.shape):
            old = theta[idx]
            h = 1e-6 * max(1.0, abs(old))
            theta[idx] = old + h
            fp = _loss(c, dout, True, zoh=True)
            theta[idx] = old - h
            fm = _loss(c, dout, True, zoh=True)
            theta[idx] = old
            fd[idx] = (fp - fm) / (2 * h)
        scale = max(1.0, np.abs(fd).max())
        np.testing.assert_allclose(g[gname], fd, rtol=0, atol=1e-6 * scale,
                                   err_msg=f"zoh gradient {gname}")


def test_zoh_adjoint_differs_from_euler_b():
    """A dropped ZOH term would leave the gradients equal to the B̄ = ΔB ones;
    at |ΔA| ~ 1 they must differ."""
    c = rand_case(33, batch=1, dim=2, L=6, N=4)
    dout = rng(34).standard_normal(c["u"].shape)
    g0 = oracle.bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                    c["delta_bias"], True, dout, zoh=False)
    g1 = oracle.bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                    c["delta_bias"], True, dout, zoh=True)
    for k in ("du", "ddelta", "dA", "dB"):
        assert np.abs(g0[k] - g1[k]).max() > 1e-3 * np.abs(g0[k]).max(), k


def test_adjoint_directional_derivative_larger_case():
    """<grad, v> equals the directional derivative along a random v (checks the
    reductions over batch and channel at a larger shape)."""
    c = rand_case(15, batch=2, dim=6, L=64, N=16)
    dout = rng(16).standard_normal(c["u"].shape)
    g = oracle.bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                   c["delta_bias"], True, dout)
    r = rng(17)
    v = {k: r.standard_normal(c[k].shape) for k in GRAD_OF}
    eps = 1e-6

    def at(s):
        cc = {k: (c[k] + s * eps * v[k]) for k in GRAD_OF}
        return _loss(cc, dout, True)
    fd = (at(1) - at(-1)) / (2 * eps)
    an = sum(float((g[GRAD_OF[k]] * v[k]).sum()) for k in GRAD_OF)
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an))


@pytest.mark.parametrize("cuts", [(0, 200), (0, 64, 200), (0, 1, 97, 150, 200)])
def test_segments_reassembled_by_carries_equal_the_whole_scan(cuts):
    """Split-sequence invariant behind sequence sharding: each segment run from
    a zero state gives (Σ Δ, end state); combine_carries turns those into the
    state entering every segment, and re-running each segment from it equals
    the forward over the whole sequence (out and final state)."""
    r = rng(12)
    batch, dim, N, L = 2, 3, 4, 200
    u = r.standard_normal((batch, dim, L))
    delta = r.standard_normal((batch, dim, L))
    A = -np.exp(r.standard_normal((dim, N)))
    B = r.standard_normal((batch, N, L))
    C = r.standard_normal((batch, N, L))
    D = r.uniform(0.5, 1.5, dim)
    z = r.standard_normal((batch, dim, L))
    bias = r.uniform(-1, 1, dim)
    h0 = r.standard_normal((batch, dim, N))
    want, wlast = oracle.fwd(u, delta, A, B, C, D, z, bias, True, h0=h0)
    segs = list(zip(cuts[:-1], cuts[1:]))
    ds, ends = [], []
    for a, b in segs:
        _, e = oracle.fwd(u[..., a:b], delta[..., a:b], A, B[..., a:b], C[..., a:b], D,
                          z[..., a:b], bias, True)
        ds.append(oracle.delta_sums(delta[..., a:b], bias, True))
        ends.append(e)
    hin = oracle.combine_carries(A, np.stack(ds), np.stack(ends), h0)
    got = np.empty_like(want)
    for s, (a, b) in enumerate(segs):
        got[..., a:b], last = oracle.fwd(u[..., a:b], delta[..., a:b], A, B[..., a:b], C[..., a:b],
                                         D, z[..., a:b], bias, True, h0=hin[s])
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(last, wlast, rtol=1e-11, atol=1e-12)


def test_delta_sums_softplus_and_raw():
    d = np.array([[[0.0, 1.0, -30.0]]])
    np.testing.assert_allclose(oracle.delta_sums(d, None, False), [[-29.0]])
    np.testing.assert_allclose(oracle.delta_sums(d, np.array([1.0]), True),
                               [[np.log1p(np.e) + np.log1p(np.e ** 2) + np.log1p(np.exp(-29.0))]],
                               rtol=1e-14)
