"""Pins for the fp64 oracle: facts the pages and the mathematics fix.

None of these re-type the oracle's loop.  Each checks it against something
else: a closed form, a limit, an identity, a brute-force evaluation in a
different order, or a correctly rounded sum.  Together they are chosen so that
a plausible slip in the oracle (a dropped term, a wrong sign or index, B and C
swapped, the bias outside the softplus, the readout before the update, the
gate missing the skip term) fails at least one of them.
"""
import math
import random

import numpy as np
import pytest

import oracle
from selective_state_space_ss_b200 import inputs as I


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ---------------------------------------------------------------- scalars --

def test_softplus_identities():
    # softplus(0) = ln 2; softplus(x) - softplus(-x) = x for every x;
    # softplus(x) -> x for large x and -> e^x for very negative x.
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-16, abs=0)
    for x in (-35.0, -7.25, -1e-3, 0.3, 2.0, 19.5, 29.9, 30.1, 55.0):
        assert oracle.softplus(x) - oracle.softplus(-x) == pytest.approx(x, rel=1e-15, abs=1e-15)
    assert oracle.softplus(60.0) == 60.0
    assert oracle.softplus(-40.0) == pytest.approx(math.exp(-40.0), rel=1e-15, abs=0)
    # monotone and positive
    xs = np.linspace(-50, 50, 1001)
    v = np.array([oracle.softplus(x) for x in xs])
    assert np.all(v > 0) and np.all(np.diff(v) > 0)


def test_silu_identities():
    # SiLU(z) = z * sigmoid(z): SiLU(0) = 0, SiLU(z) - SiLU(-z) = z,
    # SiLU(z) -> z for large z and -> 0 for very negative z.
    assert oracle.silu(0.0) == 0.0
    for z in (-20.0, -3.0, -0.5, 0.25, 1.0, 4.0, 30.0):
        assert oracle.silu(z) - oracle.silu(-z) == pytest.approx(z, rel=1e-15, abs=1e-15)
    assert oracle.silu(50.0) == pytest.approx(50.0, rel=1e-20, abs=0)
    assert abs(oracle.silu(-50.0)) < 1e-19
    assert oracle.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15, abs=0)


# ------------------------------------------------------ LTI closed form ----

@pytest.mark.parametrize("softplus_on", [False, True])
def test_lti_closed_form(softplus_on):
    """Constant Delta, B, C: y = u * K_bar with K_k = sum_n C_n e^{k Delta A_n} Delta B_n.

    The recurrence-equals-convolution identity of a time-invariant SSM
    ("从Transformer的痛点 ... Mamba", sec. 2.3; "Mamba 深度解读报告", sec. 2.2).
    With the softplus on, delta = -bias exactly, so Delta = softplus(0) = ln 2.
    """
    rng = np.random.default_rng(7)
    batch, dim, L, N = 2, 3, 200, 5
    A = -rng.uniform(0.05, 3.0, size=(dim, N))
    Bc = rng.normal(size=(batch, N))
    Cc = rng.normal(size=(batch, N))
    u = rng.normal(size=(batch, dim, L))
    if softplus_on:
        bias = rng.uniform(-3, 3, size=dim).astype(np.float32)
        delta = np.broadcast_to(-bias[None, :, None], (batch, dim, L))
        dvals = np.full(dim, math.log(2.0))
    else:
        bias = None
        dvals = rng.uniform(0.01, 0.2, size=dim).astype(np.float32).astype(np.float64)
        delta = np.broadcast_to(dvals[None, :, None], (batch, dim, L))
    Bt = np.broadcast_to(Bc[:, :, None], (batch, N, L))
    Ct = np.broadcast_to(Cc[:, :, None], (batch, N, L))
    y, h = oracle.scan_fwd(_f32(u), _f32(delta), _f32(A), _f32(Bt), _f32(Ct),
                           delta_bias=bias, softplus=softplus_on)
    # closed form from the fp32-rounded parameters, direct causal convolution
    A32 = _f32(A).astype(np.float64)
    B32, C32, u32 = (_f32(v).astype(np.float64) for v in (Bc, Cc, u))
    k = np.arange(L, dtype=np.float64)
    for b in range(batch):
        for d in range(dim):
            dl = dvals[d]
            K = np.zeros(L)
            for n in range(N):
                K += C32[b, n] * np.exp(k * dl * A32[d, n]) * dl * B32[b, n]
            ref = np.convolve(u32[b, d], K)[:L]
            assert _rel(y[b, d], ref) < 1e-12
            # final state: h_L[n] = sum_s e^{(L-1-s) Delta A_n} Delta B_n u_s
            for n in range(N):
                hs = np.sum(np.exp((L - 1 - k) * dl * A32[d, n]) * dl * B32[b, n] * u32[b, d])
                assert h[b, d, n] == pytest.approx(hs, rel=1e-12, abs=1e-14)


# ------------------------------------------- the associative operator ------

def _combine(earlier, later):
    """(a1,b1) then (a2,b2): the pages' (a,b)∘(c,d) = (ac, ad+b), later on the left."""
    a1, b1 = earlier
    a2, b2 = later
    return (a2 * a1, a2 * b1 + b2)


def test_operator_associative():
    rng = np.random.default_rng(11)
    n = 1_000_000
    x = (rng.uniform(0.0, 1.0, n), rng.normal(size=n))
    y = (rng.uniform(0.0, 1.0, n), rng.normal(size=n))
    z = (rng.uniform(0.0, 1.0, n), rng.normal(size=n))
    left = _combine(_combine(x, y), z)
    right = _combine(x, _combine(y, z))
    scale = np.abs(x[1]) + np.abs(y[1]) + np.abs(z[1])
    assert np.max(np.abs(left[0] - right[0])) <= 1e-15
    assert np.max(np.abs(left[1] - right[1]) / scale) <= 1e-14


def _tree_prefix(pairs):
    """Inclusive prefix of a list of (a, b) pairs by a Blelloch up/down sweep."""
    n = len(pairs)
    size = 1
    while size < n:
        size *= 2
    ident = (np.ones_like(pairs[0][0]), np.zeros_like(pairs[0][1]))
    t = list(pairs) + [ident] * (size - n)
    step = 1
    while step < size:  # up-sweep
        for i in range(2 * step - 1, size, 2 * step):
            t[i] = _combine(t[i - step], t[i])
        step *= 2
    t[size - 1] = ident
    step = size // 2
    while step >= 1:  # down-sweep (exclusive)
        for i in range(2 * step - 1, size, 2 * step):
            left = t[i - step]
            t[i - step] = t[i]
            t[i] = _combine(t[i], left)
        step //= 2
    return [_combine(t[i], pairs[i]) for i in range(n)]


def test_tree_fold_equals_serial_oracle():
    """A work-efficient tree scan over (A_bar_t, Delta_t B_t u_t) gives the oracle's states."""
    rng = np.random.default_rng(5)
    batch, dim, L, N = 1, 2, 37, 4
    u = _f32(rng.normal(size=(batch, dim, L)))
    delta = _f32(rng.uniform(0.01, 0.5, size=(batch, dim, L)))
    A = _f32(-rng.uniform(0.1, 4.0, size=(dim, N)))
    B = _f32(rng.normal(size=(batch, N, L)))
    C = _f32(rng.normal(size=(batch, N, L)))
    y, h = oracle.scan_fwd(u, delta, A, B, C, softplus=False)
    for d in range(dim):
        pairs = []
        for t in range(L):
            dl = float(delta[0, d, t])
            a = np.exp(dl * A[d].astype(np.float64))
            bb = dl * B[0, :, t].astype(np.float64) * float(u[0, d, t])
            pairs.append((a, bb))
        pref = _tree_prefix(pairs)
        for t in range(L):
            ht = pref[t][1]
            yt = float(np.dot(C[0, :, t].astype(np.float64), ht))
            assert yt == pytest.approx(y[0, d, t], rel=1e-12, abs=1e-13)
        assert np.allclose(pref[-1][1], h[0, d], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------- the Delta limits -----

def _rand_case(rng, batch, dim, L, N):
    return dict(u=_f32(rng.normal(size=(batch, dim, L))),
                B=_f32(rng.normal(size=(batch, N, L))),
                C=_f32(rng.normal(size=(batch, N, L))),
                z=_f32(rng.normal(size=(batch, dim, L))),
                D=_f32(rng.normal(size=dim)),
                A=_f32(-rng.uniform(1.0, 8.0, size=(dim, N))))


def test_hold_limit_exact_zero_delta():
    """Delta = 0 exactly: A_bar = 1 and B_bar u = 0, so the state is held bitwise
    ("Mamba 选择性机制", sec. 2.1: small Delta keeps the state)."""
    rng = np.random.default_rng(3)
    batch, dim, L, N, P = 2, 3, 50, 6, 20
    c = _rand_case(rng, batch, dim, L, N)
    delta = np.zeros((batch, dim, L), np.float32)
    delta[:, :, :P] = rng.uniform(0.05, 0.5, size=(batch, dim, P))
    y, h = oracle.scan_fwd(c["u"], delta, c["A"], c["B"], c["C"], D=c["D"], softplus=False)
    yp, hp = oracle.scan_fwd(c["u"][:, :, :P].copy(), delta[:, :, :P].copy(), c["A"],
                             c["B"][:, :, :P].copy(), c["C"][:, :, :P].copy(), D=c["D"], softplus=False)
    assert np.array_equal(h, hp)  # held bitwise from the end of the prefix
    assert np.array_equal(y[:, :, :P], yp)
    Cw, uw = c["C"].astype(np.float64), c["u"].astype(np.float64)
    for t in range(P, L):
        ref = np.einsum("bn,bdn->bd", Cw[:, :, t], hp) + c["D"].astype(np.float64)[None] * uw[:, :, t]
        assert _rel(y[:, :, t], ref) < 1e-14


def test_hold_limit_softplus_with_bias():
    """delta + bias = -60 under the softplus: Delta ~ 9e-27, the state is held.

    The bias is nonzero, so a bias added outside the softplus would give
    Delta ~ 3 and fail here."""
    rng = np.random.default_rng(4)
    batch, dim, L, N, P = 1, 4, 40, 5, 15
    c = _rand_case(rng, batch, dim, L, N)
    bias = np.full(dim, 3.0, np.float32)
    delta = np.full((batch, dim, L), -63.0, np.float32)
    delta[:, :, :P] = _f32(rng.normal(scale=0.5, size=(batch, dim, P)))
    y, h = oracle.scan_fwd(c["u"], delta, c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                           delta_bias=bias, softplus=True)
    _, hp = oracle.scan_fwd(*(np.ascontiguousarray(v[:, :, :P]) for v in (c["u"], delta)), c["A"],
                            *(np.ascontiguousarray(v[:, :, :P]) for v in (c["B"], c["C"])),
                            D=c["D"], z=np.ascontiguousarray(c["z"][:, :, :P]),
                            delta_bias=bias, softplus=True)
    assert _rel(h, hp) < 1e-22
    gate = np.vectorize(oracle.silu)(c["z"].astype(np.float64))
    for t in range(P, L):
        ref = (np.einsum("bn,bdn->bd", c["C"][:, :, t].astype(np.float64), hp)
               + c["D"].astype(np.float64)[None] * c["u"][:, :, t]) * gate[:, :, t]
        assert _rel(y[:, :, t], ref) < 1e-14


def test_reset_limit():
    """delta + bias = 60 under the softplus and A <= -1: A_bar <= e^-60, the state
    resets every step to Delta B_t u_t, with Delta = 60
    ("Mamba 选择性机制", sec. 2.1: large Delta forgets the past)."""
    rng = np.random.default_rng(6)
    batch, dim, L, N = 2, 3, 30, 7
    c = _rand_case(rng, batch, dim, L, N)
    bias = _f32(rng.uniform(-2, 2, size=dim))
    delta = np.broadcast_to((60.0 - bias.astype(np.float64))[None, :, None], (batch, dim, L))
    delta = _f32(delta)
    x = delta.astype(np.float64) + bias.astype(np.float64)[None, :, None]  # ~60
    y, h = oracle.scan_fwd(c["u"], delta, c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                           delta_bias=bias, softplus=True)
    gate = np.vectorize(oracle.silu)(c["z"].astype(np.float64))
    for t in range(L):
        dl = x[:, :, t]  # softplus(x) = x to double precision at x ~ 60
        cb = np.sum(c["C"][:, :, t].astype(np.float64) * c["B"][:, :, t].astype(np.float64), axis=1)
        ut = c["u"][:, :, t].astype(np.float64)
        ref = (dl * ut * cb[:, None] + c["D"].astype(np.float64)[None] * ut) * gate[:, :, t]
        assert _rel(y[:, :, t], ref) < 1e-14
    href = x[:, :, -1][:, :, None] * c["B"][:, None, :, -1].astype(np.float64) * c["u"][:, :, -1:].astype(np.float64)
    assert _rel(h, href) < 1e-14


# --------------------------------------------- brute-force unrolled sums ---

@pytest.mark.parametrize("L", [1, 2, 5, 8])
def test_bruteforce_unrolled(L):
    """h_t = sum_{s<=t} (prod_{s<k<=t} A_bar_k) Delta_s B_s u_s with explicit products
    ("从Transformer的痛点 ... Mamba", sec. 4.3), then y_t = (C_t.h_t + D u_t) SiLU(z_t)."""
    rng = np.random.default_rng(100 + L)
    batch, dim, N = 2, 3, 4
    c = _rand_case(rng, batch, dim, L, N)
    c["A"] = _f32(-rng.uniform(0.1, 3.0, size=(dim, N)))
    delta = _f32(rng.normal(scale=0.5, size=(batch, dim, L)))
    bias = _f32(rng.uniform(-4, 0, size=dim))
    y, h = oracle.scan_fwd(c["u"], delta, c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                           delta_bias=bias, softplus=True)
    for b in range(batch):
        for d in range(dim):
            dl = [oracle.softplus(float(delta[b, d, t]) + float(bias[d])) for t in range(L)]
            for t in range(L):
                acc = 0.0
                hts = []
                for n in range(N):
                    a = float(c["A"][d, n])
                    hn = 0.0
                    for s in range(t + 1):
                        prod = 1.0
                        for k in range(s + 1, t + 1):
                            prod *= math.exp(dl[k] * a)
                        hn += prod * dl[s] * float(c["B"][b, n, s]) * float(c["u"][b, d, s])
                    hts.append(hn)
                    acc += float(c["C"][b, n, t]) * hn
                ref = (acc + float(c["D"][d]) * float(c["u"][b, d, t])) * oracle.silu(float(c["z"][b, d, t]))
                assert y[b, d, t] == pytest.approx(ref, rel=1e-13, abs=1e-15)
            assert np.allclose(h[b, d], hts, rtol=1e-13, atol=1e-15)


def test_prefix_sum_special_case():
    """N = 1, A = 0, no softplus, C = 1, D = 0, no gate: h_t is the running sum of
    Delta_s B_s u_s; compared with a correctly rounded sum (math.fsum)."""
    rng = np.random.default_rng(9)
    L = 3000
    u = _f32(rng.normal(size=(1, 1, L)))
    delta = _f32(rng.uniform(0.0, 1.0, size=(1, 1, L)))
    B = _f32(rng.normal(size=(1, 1, L)))
    C = np.ones((1, 1, L), np.float32)
    A = np.zeros((1, 1), np.float32)
    y, h = oracle.scan_fwd(u, delta, A, B, C, softplus=False)
    terms = [float(delta[0, 0, s]) * float(B[0, 0, s]) * float(u[0, 0, s]) for s in range(L)]
    running = [math.fsum(terms[: t + 1]) for t in range(0, L, 97)] + [math.fsum(terms)]
    idx = list(range(0, L, 97)) + [L - 1]
    bound = L * 2.0 ** -52 * math.fsum(abs(v) for v in terms)
    for i, t in enumerate(idx):
        assert abs(y[0, 0, t] - running[i]) <= bound
    assert abs(h[0, 0, 0] - running[-1]) <= bound


# ------------------------------------------------------ index plumbing -----

def test_index_plumbing_single_impulse():
    """One input at t = 0, then u = 0: h_L[b,d,n] = e^{(L-1) Delta A[d,n]} Delta B[b,n,0] u[b,d,0].

    A[d,n], B[b,n,0], u[b,d,0], D[d] and the bias are distinct per index, so a
    transposed or shifted index lands on a wrong value."""
    batch, dim, L, N = 3, 5, 9, 4
    d_idx = np.arange(dim)[:, None]
    n_idx = np.arange(N)[None, :]
    A = _f32(-(1 + d_idx + 100 * n_idx) * 1e-3)
    u = np.zeros((batch, dim, L), np.float32)
    u[:, :, 0] = _f32(1.0 + np.arange(batch)[:, None] * 0.5 + np.arange(dim)[None, :] * 0.125)
    B = np.zeros((batch, N, L), np.float32)
    B[:, :, 0] = _f32(1.0 + np.arange(batch)[:, None] * 0.25 + np.arange(N)[None, :] * 2.0)
    C = np.zeros((batch, N, L), np.float32)
    C[:, :, L - 1] = _f32(0.5 + np.arange(batch)[:, None] + 0.1 * np.arange(N)[None, :])
    bias = _f32(0.1 + 0.01 * np.arange(dim))
    Dv = _f32(10.0 + np.arange(dim))
    delta = np.zeros((batch, dim, L), np.float32)
    y, h = oracle.scan_fwd(u, delta, A, B, C, D=Dv, delta_bias=bias, softplus=False)
    for b in range(batch):
        for d in range(dim):
            dl = float(bias[d])
            for n in range(N):
                ref = math.exp((L - 1) * dl * float(A[d, n])) * dl * float(B[b, n, 0]) * float(u[b, d, 0])
                assert h[b, d, n] == pytest.approx(ref, rel=1e-14, abs=0)
            # y_0 = D u_0 + C_0.h_0 (C_0 = 0); y_{L-1} = C_{L-1}.h_{L-1}
            assert y[b, d, 0] == pytest.approx(float(Dv[d]) * float(u[b, d, 0]), rel=1e-15, abs=0)
            assert y[b, d, L - 1] == pytest.approx(float(np.dot(C[b, :, L - 1].astype(np.float64), h[b, d])),
                                                   rel=1e-14, abs=0)
            assert np.all(y[b, d, 1:L - 1] == 0.0)


# ------------------------------------------------------- initial state -----
# A carried state h0 stands for the recurrent mode of the pages: inference
# keeps h and feeds one token at a time ("从Transformer的痛点说起 ... Mamba",
# sec. 5.1 table and sec. 6.3).

def _distinct_h0(batch, dim, N):
    b = np.arange(batch)[:, None, None]
    d = np.arange(dim)[None, :, None]
    n = np.arange(N)[None, None, :]
    return (1.0 + 0.5 * b + 0.125 * d + 2.0 * n) * np.where((b + d + n) % 2 == 0, 1.0, -1.0)


def test_initial_state_free_decay_closed_form():
    """u = 0 and a constant Delta: the state only decays, h_t[n] =
    e^{(t+1) Delta A[d,n]} h0[b,d,n], evaluated directly (no products), and
    y_t = (C_t . h_t) SiLU(z_t).  h0, A and C are distinct per index, so a
    transposed or shifted initial-state index lands on a wrong value."""
    rng = np.random.default_rng(21)
    batch, dim, L, N = 2, 3, 40, 5
    A = _f32(-(0.05 + 0.1 * np.arange(dim)[:, None] + 0.37 * np.arange(N)[None, :]))
    dl = _f32(0.02 + 0.03 * np.arange(dim)).astype(np.float64)
    delta = _f32(np.broadcast_to(dl[None, :, None], (batch, dim, L)))
    u = np.zeros((batch, dim, L), np.float32)
    B = _f32(rng.normal(size=(batch, N, L)))
    C = _f32(rng.normal(size=(batch, N, L)))
    z = _f32(rng.normal(size=(batch, dim, L)))
    Dv = _f32(rng.normal(size=dim))
    h0 = _distinct_h0(batch, dim, N)
    y, h = oracle.scan_fwd(u, delta, A, B, C, D=Dv, z=z, softplus=False, h0=h0)
    A64 = A.astype(np.float64)
    for t in range(L):
        ht = np.exp((t + 1) * dl[None, :, None] * A64[None]) * h0
        ref = np.einsum("bn,bdn->bd", C[:, :, t].astype(np.float64), ht)
        ref = ref * np.vectorize(oracle.silu)(z[:, :, t].astype(np.float64))
        assert _rel(y[:, :, t], ref) < 1e-14
    assert _rel(h, np.exp(L * dl[None, :, None] * A64[None]) * h0) < 1e-14


@pytest.mark.parametrize("L", [1, 3, 5])
def test_initial_state_bruteforce(L):
    """h_t = (prod_{k<=t} A_bar_k) h0 + sum_{s<=t} (prod_{s<k<=t} A_bar_k) Delta_s B_s u_s
    with explicit products, softplus and bias on, gate and skip on."""
    rng = np.random.default_rng(200 + L)
    batch, dim, N = 2, 3, 4
    c = _rand_case(rng, batch, dim, L, N)
    c["A"] = _f32(-rng.uniform(0.1, 3.0, size=(dim, N)))
    delta = _f32(rng.normal(scale=0.5, size=(batch, dim, L)))
    bias = _f32(rng.uniform(-4, 0, size=dim))
    h0 = rng.normal(size=(batch, dim, N))
    y, h = oracle.scan_fwd(c["u"], delta, c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                           delta_bias=bias, softplus=True, h0=h0)
    for b in range(batch):
        for d in range(dim):
            dl = [oracle.softplus(float(delta[b, d, t]) + float(bias[d])) for t in range(L)]
            for t in range(L):
                acc = 0.0
                hts = []
                for n in range(N):
                    a = float(c["A"][d, n])
                    lead = 1.0
                    for k in range(t + 1):
                        lead *= math.exp(dl[k] * a)
                    hn = lead * h0[b, d, n]
                    for s in range(t + 1):
                        prod = 1.0
                        for k in range(s + 1, t + 1):
                            prod *= math.exp(dl[k] * a)
                        hn += prod * dl[s] * float(c["B"][b, n, s]) * float(c["u"][b, d, s])
                    hts.append(hn)
                    acc += float(c["C"][b, n, t]) * hn
                ref = (acc + float(c["D"][d]) * float(c["u"][b, d, t])) * oracle.silu(float(c["z"][b, d, t]))
                assert y[b, d, t] == pytest.approx(ref, rel=1e-13, abs=1e-15)
            assert np.allclose(h[b, d], hts, rtol=1e-13, atol=1e-15)


def test_split_sequence_equals_whole():
    """Scanning [0, P) and then [P, L) from the first part's final state gives
    the whole scan's outputs on [P, L) and its final state (the carried state is
    all the past the recurrence keeps)."""
    w = I.Workload("t", 2, 5, 77, 16, "bf16")
    x = I.make_inputs(w, seed=12)
    P = 30
    cut = lambda k, a, b: np.ascontiguousarray(x[k][:, :, a:b])
    y, h = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    y1, h1 = oracle.scan_fwd(cut("u", 0, P), cut("delta", 0, P), x["A"], cut("B", 0, P), cut("C", 0, P),
                             x["D"], cut("z", 0, P), x["delta_bias"])
    y2, h2 = oracle.scan_fwd(cut("u", P, 77), cut("delta", P, 77), x["A"], cut("B", P, 77),
                             cut("C", P, 77), x["D"], cut("z", P, 77), x["delta_bias"], h0=h1)
    assert np.array_equal(y1, y[:, :, :P])
    assert _rel(y2, y[:, :, P:]) < 1e-13
    assert _rel(h2, h) < 1e-13


def test_step_chain_equals_scan():
    """L single-token steps from h0 = 0 reproduce the scan over the L tokens."""
    w = I.Workload("t", 2, 4, 9, 8, "f32")
    x = I.make_inputs(w, seed=5)
    y, h = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    state = np.zeros((2, 4, 8))
    for t in range(9):
        yt, state = oracle.scan_step(state, x["u"][:, :, t], x["delta"][:, :, t], x["A"], x["B"][:, :, t],
                                     x["C"][:, :, t], x["D"], x["z"][:, :, t], x["delta_bias"])
        assert np.array_equal(yt, y[:, :, t])
    assert np.array_equal(state, h)


# ------------------------------------------------ short convolution -------
# The block's depthwise Conv1d of width W, padding W-1, cut to L outputs, then
# SiLU ("从Transformer的痛点说起 ... Mamba", sec. 3.3 diagram and sec. 4.2 code).
# With B = 0 the state stays zero and y = D u, so y exposes u itself.

def _conv_case(rng, batch, dim, L, N, W):
    c = _rand_case(rng, batch, dim, L, N)
    c["B"] = np.zeros_like(c["B"])
    c["D"] = np.ones(dim, np.float32)
    c["w"] = _f32(rng.normal(size=(dim, W)))
    c["b"] = _f32(rng.normal(size=dim))
    return c


@pytest.mark.parametrize("W", [1, 2, 4, 7])
def test_conv_prologue_matches_numpy_convolution(W):
    """u = SiLU(causal conv + bias), the conv from numpy's full convolution with
    the taps reversed (Conv1d is a cross-correlation), cut to the first L."""
    rng = np.random.default_rng(300 + W)
    batch, dim, L, N = 2, 5, 40, 4
    c = _conv_case(rng, batch, dim, L, N, W)
    delta = _f32(rng.normal(size=(batch, dim, L)))
    y, h = oracle.scan_fwd(c["u"], delta, c["A"], c["B"], c["C"], D=c["D"], softplus=True,
                           conv_weight=c["w"], conv_bias=c["b"])
    assert np.all(h == 0.0)
    x64 = c["u"].astype(np.float64)
    for b in range(batch):
        for d in range(dim):
            pre = np.convolve(x64[b, d], c["w"][d, ::-1].astype(np.float64))[:L] + float(c["b"][d])
            ref = pre / (1.0 + np.exp(-pre))
            assert _rel(y[b, d], ref) < 1e-14


def test_conv_prologue_impulse_taps():
    """x = one impulse per (b, d) at step s: u_t = SiLU(w[d, W-1-(t-s)] x_s + bias)
    for t in [s, s+W-1] and SiLU(bias) elsewhere; taps, bias and impulse size
    differ per index, so a reversed, shifted or transposed tap lands wrong."""
    batch, dim, L, N, W = 2, 3, 16, 4, 4
    rng = np.random.default_rng(12)
    c = _conv_case(rng, batch, dim, L, N, W)
    c["w"] = _f32(0.5 + np.arange(dim)[:, None] * 0.25 + np.arange(W)[None, :] * 1.5)
    c["b"] = _f32(-0.3 + 0.1 * np.arange(dim))
    x = np.zeros((batch, dim, L), np.float32)
    starts = np.array([[3, 7, 12], [0, 5, 9]])
    for b in range(batch):
        for d in range(dim):
            x[b, d, starts[b, d]] = 1.0 + b + 0.5 * d
    delta = np.zeros((batch, dim, L), np.float32)
    y, _ = oracle.scan_fwd(x, delta, c["A"], c["B"], c["C"], D=c["D"], softplus=False,
                           conv_weight=c["w"], conv_bias=c["b"])
    for b in range(batch):
        for d in range(dim):
            s0, xs, bias = starts[b, d], float(x[b, d, starts[b, d]]), float(c["b"][d])
            for t in range(L):
                k = W - 1 - (t - s0)
                pre = bias + (float(c["w"][d, k]) * xs if 0 <= k < W else 0.0)
                assert y[b, d, t] == pytest.approx(oracle.silu(pre), rel=1e-15, abs=1e-300)


def test_conv_prologue_feeds_the_scan():
    """With the convolution on, the scan sees u = SiLU(conv): brute-force
    products over that u (width 3, full B, C, gate and skip)."""
    rng = np.random.default_rng(44)
    batch, dim, L, N, W = 1, 2, 5, 3, 3
    c = _rand_case(rng, batch, dim, L, N)
    c["A"] = _f32(-rng.uniform(0.1, 2.0, size=(dim, N)))
    w = _f32(rng.normal(size=(dim, W)))
    cb = _f32(rng.normal(size=dim))
    delta = _f32(rng.normal(scale=0.5, size=(batch, dim, L)))
    y, h = oracle.scan_fwd(c["u"], delta, c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                           softplus=True, conv_weight=w, conv_bias=cb)
    for d in range(dim):
        xs = [float(v) for v in c["u"][0, d]]
        us = []
        for t in range(L):
            pre = float(cb[d]) + sum(float(w[d, k]) * xs[t - (W - 1) + k]
                                     for k in range(W) if t - (W - 1) + k >= 0)
            us.append(oracle.silu(pre))
        dl = [oracle.softplus(float(delta[0, d, t])) for t in range(L)]
        for t in range(L):
            acc = 0.0
            for n in range(N):
                a = float(c["A"][d, n])
                hn = 0.0
                for s_ in range(t + 1):
                    prod = 1.0
                    for k in range(s_ + 1, t + 1):
                        prod *= math.exp(dl[k] * a)
                    hn += prod * dl[s_] * float(c["B"][0, n, s_]) * us[s_]
                acc += float(c["C"][0, n, t]) * hn
            ref = (acc + float(c["D"][d]) * us[t]) * oracle.silu(float(c["z"][0, d, t]))
            assert y[0, d, t] == pytest.approx(ref, rel=1e-13, abs=1e-15)


# ------------------------------------------------- exact zero-order hold ---
# ZOH: the continuous system h' = A h + B x with the input held constant over
# each step of length Delta ("从Transformer的痛点说起 ... Mamba", sec. 2.2).

def _rk4_hold(a, b, x, dl, h, m=512):
    """Integrate h' = a h + b x over [0, dl] with m classical RK4 steps (no exp)."""
    k = dl / m
    f = lambda v: a * v + b * x
    for _ in range(m):
        k1 = f(h)
        k2 = f(h + 0.5 * k * k1)
        k3 = f(h + 0.5 * k * k2)
        k4 = f(h + k * k3)
        h = h + k / 6.0 * (k1 + 2 * k2 + 2 * k3 + k4)
    return h


def test_zoh_matches_ode_integration():
    """The exact-ZOH recurrence equals a fine Runge-Kutta integration of the
    continuous system with each input held over its step (and the same
    readout): B_bar is (Delta A)^-1 (e^{Delta A} - 1) Delta B."""
    rng = np.random.default_rng(71)
    batch, dim, L, N = 1, 2, 12, 3
    c = _rand_case(rng, batch, dim, L, N)
    c["A"] = _f32(-rng.uniform(0.2, 3.0, size=(dim, N)))
    delta = _f32(rng.uniform(0.05, 0.6, size=(batch, dim, L)))
    y, h = oracle.scan_fwd(c["u"], delta, c["A"], c["B"], c["C"], D=c["D"], softplus=False, zoh=True)
    for d in range(dim):
        hs = np.zeros(N)
        for t in range(L):
            dl = float(delta[0, d, t])
            for n in range(N):
                hs[n] = _rk4_hold(float(c["A"][d, n]), float(c["B"][0, n, t]), float(c["u"][0, d, t]),
                                  dl, hs[n])
            ref = float(np.dot(c["C"][0, :, t].astype(np.float64), hs)) + float(c["D"][d]) * float(c["u"][0, d, t])
            assert y[0, d, t] == pytest.approx(ref, rel=1e-9, abs=1e-12)
        assert np.allclose(h[0, d], hs, rtol=1e-9, atol=1e-12)


def test_zoh_small_delta_series():
    """Delta A ~ 1e-9: B_bar = Delta B (1 + x/2 + x^2/6) to 1e-16, x = Delta A; an
    e^x - 1 evaluation would lose half the digits here."""
    rng = np.random.default_rng(72)
    batch, dim, N = 1, 3, 4
    A = _f32(-rng.uniform(0.5, 2.0, size=(dim, N)))
    u = _f32(rng.normal(size=(batch, dim, 1)))
    B = _f32(rng.normal(size=(batch, N, 1)))
    C = np.zeros((batch, N, 1), np.float32)
    delta = np.full((batch, dim, 1), 1e-9, np.float32)
    _, h = oracle.scan_fwd(u, delta, A, B, C, softplus=False, zoh=True)
    for d in range(dim):
        dl = float(delta[0, d, 0])
        for n in range(N):
            x = dl * float(A[d, n])
            ref = dl * (1.0 + x / 2 + x * x / 6) * float(B[0, n, 0]) * float(u[0, d, 0])
            assert h[0, d, n] == pytest.approx(ref, rel=1e-15, abs=0)


def test_zoh_limit_a_zero_and_simplified_form():
    """A = 0: B_bar = Delta B exactly (the limit), so ZOH and the simplified form
    agree bitwise on those states; with A != 0 they differ."""
    rng = np.random.default_rng(73)
    batch, dim, L, N = 2, 3, 20, 4
    c = _rand_case(rng, batch, dim, L, N)
    delta = _f32(rng.normal(scale=0.5, size=(batch, dim, L)))
    A0 = np.zeros((dim, N), np.float32)
    y1, h1 = oracle.scan_fwd(c["u"], delta, A0, c["B"], c["C"], D=c["D"], z=c["z"], zoh=True)
    y2, h2 = oracle.scan_fwd(c["u"], delta, A0, c["B"], c["C"], D=c["D"], z=c["z"], zoh=False)
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)
    y3, _ = oracle.scan_fwd(c["u"], delta, c["A"], c["B"], c["C"], D=c["D"], z=c["z"], zoh=True)
    y4, _ = oracle.scan_fwd(c["u"], delta, c["A"], c["B"], c["C"], D=c["D"], z=c["z"], zoh=False)
    assert _rel(y3, y4) > 1e-3


# ------------------------------------------------------------- backward ----
# The oracle's reverse-mode gradients against central finite differences of
# the forward oracle itself (fp64 throughout; a perturbed float32 input is
# stepped by exactly representable amounts).

def _loss(x, dy, dlast, softplus):
    y, h = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                           x["delta_bias"], softplus=softplus, nthreads=1)
    v = float(np.sum(y * dy))
    if dlast is not None:
        v += float(np.sum(h * dlast))
    return v


def _fd_check(x, dy, dlast, softplus, rng, per_tensor=12):
    g = oracle.scan_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"],
                        softplus=softplus, dy=dy, dlast=dlast, nthreads=1)
    names = {"u": "du", "delta": "ddelta", "z": "dz", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
             "delta_bias": "ddelta_bias"}
    for key, gname in names.items():
        if x[key] is None:
            continue
        arr = x[key]
        flat = arr.reshape(-1)
        idx = rng.choice(flat.size, min(per_tensor, flat.size), replace=False)
        scale = float(np.max(np.abs(g[gname]))) + 1e-30
        for i in idx:
            orig = flat[i]
            step = np.float32(1e-3 * max(1.0, abs(float(orig))))
            hi, lo = np.float32(orig + step), np.float32(orig - step)
            flat[i] = hi
            f_hi = _loss(x, dy, dlast, softplus)
            flat[i] = lo
            f_lo = _loss(x, dy, dlast, softplus)
            flat[i] = orig
            fd = (f_hi - f_lo) / (float(hi) - float(lo))
            got = float(g[gname].reshape(-1)[i])
            assert abs(fd - got) <= 2e-5 * scale, f"{gname}[{i}]: fd {fd} vs {got}"


@pytest.mark.parametrize("softplus,with_z,with_dlast", [(True, True, False), (True, True, True),
                                                        (False, False, False)])
def test_backward_matches_finite_differences(softplus, with_z, with_dlast):
    rng = np.random.default_rng(90 + 2 * softplus + with_z + 4 * with_dlast)
    batch, dim, L, N = 2, 3, 9, 4
    c = _rand_case(rng, batch, dim, L, N)
    c["A"] = _f32(-rng.uniform(0.2, 2.0, size=(dim, N)))
    x = dict(u=c["u"], B=c["B"], C=c["C"], A=c["A"], D=c["D"], z=c["z"] if with_z else None,
             delta_bias=_f32(rng.uniform(-1.5, -0.5, size=dim)))
    if softplus:
        x["delta"] = _f32(rng.normal(scale=0.5, size=(batch, dim, L)))
    else:  # Delta = delta + bias must stay positive
        x["delta"] = _f32(rng.uniform(1.6, 2.0, size=(batch, dim, L)))
    dy = rng.normal(size=(batch, dim, L))
    dlast = rng.normal(size=(batch, dim, N)) if with_dlast else None
    _fd_check(x, dy, dlast, softplus, rng)


def test_backward_linear_in_dy():
    """The gradients are linear in the upstream gradient: grad(2 dy1 - dy2) =
    2 grad(dy1) - grad(dy2), and zero for dy = 0 (without dlast)."""
    w = I.Workload("t", 2, 4, 11, 8, "bf16")
    x = I.make_inputs(w, seed=21)
    rng = np.random.default_rng(3)
    dy1, dy2 = rng.normal(size=(2, 4, 11)), rng.normal(size=(2, 4, 11))
    args = (x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    g1 = oracle.scan_bwd(*args, dy=dy1)
    g2 = oracle.scan_bwd(*args, dy=dy2)
    g3 = oracle.scan_bwd(*args, dy=2 * dy1 - dy2)
    g0 = oracle.scan_bwd(*args, dy=np.zeros_like(dy1))
    for k in g1:  # dz = dy q SiLU'(z) is linear in dy as well
        assert _rel(g3[k], 2 * g1[k] - g2[k]) < 1e-12, k
        assert np.all(g0[k] == 0.0), k


# ------------------------------------------------------- host plumbing -----

def test_channel_subset_matches_full():
    w = I.Workload("t", 2, 6, 33, 8, "bf16")
    x = I.make_inputs(w, seed=3)
    y, h = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    ch = np.array([11, 0, 7, 5])
    ys, hs = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"],
                             channels=ch)
    assert np.array_equal(ys, y.reshape(-1, 33)[ch])
    assert np.array_equal(hs, h.reshape(-1, 8)[ch])


def test_bf16_widening_is_exact():
    w = I.Workload("t", 1, 4, 17, 4, "bf16")
    x = I.make_inputs(w, seed=8)
    y1, h1 = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    wd = {k: I.bf16_to_f32(x[k]) for k in ("u", "delta", "B", "C", "z")}
    y2, h2 = oracle.scan_fwd(wd["u"], wd["delta"], x["A"], wd["B"], wd["C"], x["D"], wd["z"], x["delta_bias"])
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)


def test_oracle_rejects_bad_arguments():
    u = np.zeros((1, 2, 3), np.float32)
    with pytest.raises(ValueError):
        oracle.scan_fwd(u, u, np.zeros((2, 4), np.float32), np.zeros((1, 4, 3), np.float32),
                        np.zeros((1, 4, 2), np.float32))
    with pytest.raises(TypeError):
        oracle.scan_fwd(u, u.astype(np.float64), np.zeros((2, 4), np.float32),
                        np.zeros((1, 4, 3), np.float32), np.zeros((1, 4, 3), np.float32))
