"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: a
brute-force unrolled sum written independently here, a textbook closed
form, a hand-worked example, or an invariant the pages state.  Chosen so
that a plausible slip in the oracle (a dropped term, a wrong sign, a
B/C swap, an off-by-one time index, bias after instead of before the
softplus) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _softplus_ref(x):
    # textbook definition, evaluated independently of the oracle
    return math.log(1.0 + math.exp(x)) if x < 30 else x + math.exp(-x)


def _silu_ref(v):
    return v / (1.0 + math.exp(-v))


def _brute_force(u, delta, bias, A, B, C, D, z, h0, softplus):
    """y_t = sum_{s<=t} sum_n C_t[n] (prod_{r=s+1..t} exp(d_r A[n])) d_s B_s[n] u_s
             + sum_n C_t[n] (prod_{r=0..t} exp(d_r A[n])) h0[n] + D u_t,
    times silu(z_t); evaluated term by term with explicit products."""
    batch, dim, L = u.shape
    N = A.shape[1]
    y = np.zeros((batch, dim, L))
    hs = np.zeros((batch, dim, N))
    for b in range(batch):
        for d in range(dim):
            dl = [float(delta[b, d, t]) + (float(bias[d]) if bias is not None else 0.0)
                  for t in range(L)]
            if softplus:
                dl = [_softplus_ref(v) for v in dl]

            def prod(n, lo, hi):  # prod_{r=lo..hi} exp(dl_r A[n])
                p = 1.0
                for r in range(lo, hi + 1):
                    p *= math.exp(dl[r] * float(A[d, n]))
                return p

            def state(n, t):
                acc = 0.0
                for s in range(t + 1):
                    acc += prod(n, s + 1, t) * dl[s] * float(B[b, n, s]) * float(u[b, d, s])
                if h0 is not None:
                    acc += prod(n, 0, t) * float(h0[b, d, n])
                return acc

            for t in range(L):
                out = sum(float(C[b, n, t]) * state(n, t) for n in range(N))
                if D is not None:
                    out += float(D[d]) * float(u[b, d, t])
                if z is not None:
                    out *= _silu_ref(float(z[b, d, t]))
                y[b, d, t] = out
            for n in range(N):
                hs[b, d, n] = state(n, L - 1)
    return y, hs


def _rand_tiny(seed, batch=1, dim=2, N=3, L=12, gate=True, with_h0=True):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((batch, dim, L))
    delta = 0.5 * rng.standard_normal((batch, dim, L))
    bias = rng.uniform(-3, 0, dim)
    A = -rng.uniform(0.2, 2.0, (dim, N))
    B = rng.standard_normal((batch, N, L))
    C = rng.standard_normal((batch, N, L))
    D = rng.standard_normal(dim)
    z = rng.standard_normal((batch, dim, L)) if gate else None
    h0 = rng.standard_normal((batch, dim, N)) if with_h0 else None
    return u, delta, bias, A, B, C, D, z, h0


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("softplus", [True, False])
def test_oracle_matches_bruteforce(seed, softplus):
    u, delta, bias, A, B, C, D, z, h0 = _rand_tiny(seed, batch=2)
    if not softplus:
        delta = np.abs(delta)  # keep the step positive without softplus
    y_ref, h_ref = _brute_force(u, delta, bias, A, B, C, D, z, h0, softplus)
    y, h = oracle.selscan(u, delta, A, B, C, D=D, z=z, delta_bias=bias,
                          delta_softplus=softplus, h0=h0)
    np.testing.assert_allclose(y, y_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(h, h_ref, rtol=1e-11, atol=1e-12)


def test_oracle_handworked_golden():
    """Hand-worked N=2, L=3 example (exact fractions, see the fixture)."""
    vals = {}
    with open(os.path.join(GOLDEN, "handworked_n2_l3.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            vals[k] = np.array([float(x) for x in v])
    u = vals["u"].reshape(1, 1, 3)
    B = np.stack([vals["B0"], vals["B1"]]).reshape(1, 2, 3)
    C = np.stack([vals["C0"], vals["C1"]]).reshape(1, 2, 3)
    A = vals["A"].reshape(1, 2)
    delta = np.ones((1, 1, 3))
    y, h = oracle.selscan(u, delta, A, B, C, D=vals["D"], delta_softplus=False)
    np.testing.assert_allclose(y.ravel(), vals["y"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(h.ravel(), vals["last_state"], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("N", [1, 4])
def test_oracle_lti_is_causal_convolution(N):
    """Constant delta, B, C: the scan equals a causal convolution of u with
    K_k = sum_n C_n exp(k delta A_n) delta B_n ("P20 -- Mamba", section 5:
    a time-invariant SSM is a convolution with a long kernel)."""
    rng = np.random.default_rng(7)
    L, dim = 40, 3
    u = rng.standard_normal((1, dim, L))
    dval = rng.uniform(0.05, 0.5, dim)
    delta = np.repeat(dval[None, :, None], L, axis=2)
    A = -rng.uniform(0.1, 1.0, (dim, N))
    bvec = rng.standard_normal(N)
    cvec = rng.standard_normal(N)
    B = np.repeat(bvec[None, :, None], L, axis=2)
    C = np.repeat(cvec[None, :, None], L, axis=2)
    D = rng.standard_normal(dim)
    y, _ = oracle.selscan(u, delta, A, B, C, D=D, delta_softplus=False)
    for d in range(dim):
        k = np.arange(L)
        K = sum(cvec[n] * np.exp(k * dval[d] * A[d, n]) * dval[d] * bvec[n]
                for n in range(N))
        conv = np.array([sum(K[j] * u[0, d, t - j] for j in range(t + 1))
                         for t in range(L)])
        np.testing.assert_allclose(y[0, d], conv + D[d] * u[0, d], rtol=1e-11,
                                   atol=1e-12)


def test_oracle_geometric_closed_form():
    """One state, constant input: h_t = delta b x (1 - a^(t+1)) / (1 - a)."""
    L = 64
    dval, Aval, bval, cval, xval = 0.1, -2.0, 1.5, -0.75, 2.0
    a = math.exp(dval * Aval)
    u = np.full((1, 1, L), xval)
    y, h = oracle.selscan(u, np.full((1, 1, L), dval), np.array([[Aval]]),
                          np.full((1, 1, L), bval), np.full((1, 1, L), cval),
                          delta_softplus=False)
    t = np.arange(L)
    h_ref = dval * bval * xval * (1 - a ** (t + 1)) / (1 - a)
    np.testing.assert_allclose(y[0, 0], cval * h_ref, rtol=1e-12)
    assert abs(h[0, 0, 0] - h_ref[-1]) < 1e-12 * abs(h_ref[-1])


def test_oracle_softplus_known_values():
    """With A = 0, B = C = u = 1 and no skip, y_0 = delta_0: the step size the
    oracle uses must be softplus(Delta + bias), bias added first."""
    cases = [(0.0, 0.0, math.log(2.0)),
             (0.25, math.log(math.e - 1.0) - 0.25, 1.0),
             (-30.0, 0.0, math.exp(-30.0)),
             (30.0, 0.0, 30.0 + math.exp(-30.0)),
             (2.0, -1.0, math.log1p(math.e))]
    for raw, bias, want in cases:
        one = np.ones((1, 1, 1))
        y, _ = oracle.selscan(np.full((1, 1, 1), 1.0), np.full((1, 1, 1), raw),
                              np.zeros((1, 1)), one, one,
                              delta_bias=np.array([bias]), delta_softplus=True)
        assert abs(y[0, 0, 0] - want) <= 1e-14 * max(1.0, want), (raw, bias)


def test_oracle_delta_zero_freezes_state():
    """delta = 0 on a run of tokens leaves h bit-identical across the run and
    y = C_t . h + D u_t there ("03 -- Modelos de espacio de estados", the
    selective mechanism: a closed gate keeps the state)."""
    u, delta, _, A, B, C, D, _, _ = _rand_tiny(3, dim=2, N=4, L=30, gate=False,
                                               with_h0=False)
    delta = np.abs(delta)
    delta[:, :, 10:20] = 0.0
    _, h10 = oracle.selscan(u[..., :10], delta[..., :10], A, B[..., :10],
                            C[..., :10], D=D, delta_softplus=False)
    _, h20 = oracle.selscan(u[..., :20], delta[..., :20], A, B[..., :20],
                            C[..., :20], D=D, delta_softplus=False)
    assert np.array_equal(h10, h20)
    y, _ = oracle.selscan(u, delta, A, B, C, D=D, delta_softplus=False)
    for t in range(10, 20):
        want = np.einsum("n,dn->d", C[0, :, t], h10[0]) + D * u[0, :, t]
        np.testing.assert_allclose(y[0, :, t], want, rtol=1e-13, atol=1e-13)


def test_oracle_large_delta_resets_state():
    """delta |A| >= 50 forgets the past: h_t = delta B_t u_t up to exp(-50)."""
    u, delta, _, A, B, C, D, _, _ = _rand_tiny(4, dim=2, N=3, L=16, gate=False,
                                               with_h0=False)
    A = -np.abs(A) - 1.0
    delta = np.abs(delta)
    delta[:, :, -1] = 60.0
    _, h = oracle.selscan(u, delta, A, B, C, delta_softplus=False)
    want = 60.0 * B[0, :, -1][None, :] * u[0, :, -1][:, None]
    np.testing.assert_allclose(h[0], want, rtol=1e-12)


def test_oracle_linear_in_u():
    """Without the gate the scan is linear in u (delta is an input)."""
    u1, delta, bias, A, B, C, D, _, _ = _rand_tiny(5, dim=3, N=4, L=25,
                                                   gate=False, with_h0=False)
    u2 = np.random.default_rng(9).standard_normal(u1.shape)
    al, be = 1.7, -0.6
    y1, h1 = oracle.selscan(u1, delta, A, B, C, D=D, delta_bias=bias)
    y2, h2 = oracle.selscan(u2, delta, A, B, C, D=D, delta_bias=bias)
    y3, h3 = oracle.selscan(al * u1 + be * u2, delta, A, B, C, D=D,
                            delta_bias=bias)
    np.testing.assert_allclose(y3, al * y1 + be * y2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(h3, al * h1 + be * h2, rtol=1e-10, atol=1e-12)


def test_oracle_step_equals_scan():
    """L single decode steps that carry h reproduce the full scan
    ("03 -- Modelos de espacio de estados", section "Coste de inferencia")."""
    u, delta, bias, A, B, C, D, z, h0 = _rand_tiny(6, batch=2, dim=3, N=5, L=20)
    y_scan, h_scan = oracle.selscan(u, delta, A, B, C, D=D, z=z,
                                    delta_bias=bias, h0=h0)
    st = h0.copy()
    ys = []
    for t in range(u.shape[2]):
        yt, st = oracle.selscan_step(st, u[:, :, t], delta[:, :, t], A,
                                     B[:, :, t], C[:, :, t], D=D, z=z[:, :, t],
                                     delta_bias=bias)
        ys.append(yt)
    np.testing.assert_allclose(np.stack(ys, axis=2), y_scan, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st, h_scan, rtol=1e-12, atol=1e-13)


def test_oracle_channel_subset_matches_full():
    inp = synthetic.make_diag(2, 12, 16, 50, dtype="bf16", seed=11)
    args = (inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"])
    kw = dict(D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"])
    y, h = oracle.selscan(*args, **kw)
    ys, hs = oracle.selscan(*args, **kw, channels=(5, 9))
    assert np.array_equal(ys, y[:, 5:9]) and np.array_equal(hs, h[:, 5:9])


def _scalar_tiny(seed, batch=2, H=4, P=3, N=5, L=29, G=2, gate=True, h0=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((batch, H * P, L))
    dt = rng.uniform(-2.0, 0.5, (batch, H, L))
    dt_bias = rng.uniform(-1.0, 0.0, H)
    A = -np.exp(rng.uniform(0.0, math.log(16.0), H))
    B = rng.standard_normal((batch, G, N, L))
    C = rng.standard_normal((batch, G, N, L))
    D = rng.standard_normal(H)
    z = rng.standard_normal((batch, H * P, L)) if gate else None
    hh = rng.standard_normal((batch, H, P, N)) if h0 else None
    return x, dt, dt_bias, A, B, C, D, z, hh


def test_oracle_scalarA_equals_broadcast_diagonal():
    """Mamba-2's transition is a scalar per head times the identity ("Mamba-3"
    blog, first section): the scalar-A scan equals the diagonal scan with
    A[d, n] = A[head(d)], the head's step size and the group's B, C."""
    x, dt, dt_bias, A, B, C, D, z, h0 = _scalar_tiny(1)
    batch, H, L = dt.shape
    P = x.shape[1] // H
    N = B.shape[2]
    G = B.shape[1]
    y, hs = oracle.selscan_scalarA(x, dt, A, B, C, P, D=D, z=z, dt_bias=dt_bias,
                                   dt_softplus=True, h0=h0)
    Ad = np.repeat(A, P)[:, None] * np.ones((1, N))
    delta_d = np.repeat(dt, P, axis=1)
    bias_d = np.repeat(dt_bias, P)
    D_d = np.repeat(D, P)
    y2, hs2 = oracle.selscan(x, delta_d, Ad, B, C, D=D_d, z=z, delta_bias=bias_d,
                             delta_softplus=True, h0=h0.reshape(batch, H * P, N))
    assert G == 2
    np.testing.assert_allclose(y, y2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(hs.reshape(batch, H * P, N), hs2, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("chunk", [1, 4, 7, 29, 64])
def test_oracle_ssd_chunked_equals_recurrence(chunk):
    """The chunked SSD matrix form ("Mamba-2 y state-space models", 4.2)
    equals the recurrence for any chunk length, ragged last chunk included."""
    x, dt, dt_bias, A, B, C, D, z, h0 = _scalar_tiny(2)
    P = x.shape[1] // A.shape[0]
    y_rec, h_rec = oracle.selscan_scalarA(x, dt, A, B, C, P, D=D, z=z,
                                          dt_bias=dt_bias, dt_softplus=True, h0=h0)
    y_ssd, h_ssd = oracle.ssd_chunked(x, dt, A, B, C, P, chunk, D=D, z=z,
                                      dt_bias=dt_bias, dt_softplus=True, h0=h0)
    np.testing.assert_allclose(y_ssd, y_rec, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(h_ssd, h_rec, rtol=1e-10, atol=1e-11)


def test_oracle_empty_sequence():
    """L = 0: no output and the state stays at h0 (zero by default)."""
    u = np.zeros((1, 2, 0))
    y, h = oracle.selscan(u, u, np.ones((2, 3)) * -1, np.zeros((1, 3, 0)),
                          np.zeros((1, 3, 0)))
    assert y.shape == (1, 2, 0) and np.all(h == 0)


def test_round_bf16_matches_torch():
    """The synthetic generator's bf16 rounding is round-to-nearest-even."""
    torch = pytest.importorskip("torch")
    a = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 3
    a[:4] = [1.00390625, 1.01171875, -1.00390625, 0.0]  # exact ties and zero
    ours = synthetic.round_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours, ref)


def test_scalarA_groups_split_into_independent_problems():
    """Scalar-A with G groups of B/C: heads of group g see only B[:, g],
    C[:, g], so the result equals G single-group problems over the head
    slices (structure of Mamba-2's grouped B/C; a wrong group index fails)."""
    rng = np.random.default_rng(17)
    batch, H, P, N, L, G = 2, 4, 3, 5, 9, 2
    x = rng.standard_normal((batch, H * P, L))
    dt = rng.uniform(0.01, 0.2, (batch, H, L))
    A = -rng.uniform(0.5, 3.0, H)
    B = rng.standard_normal((batch, G, N, L))
    C = rng.standard_normal((batch, G, N, L))
    D = rng.standard_normal(H)
    y, hs = oracle.selscan_scalarA(x, dt, A, B, C, P, D=D)
    per = H // G
    for g in range(G):
        hsl = slice(g * per, (g + 1) * per)
        csl = slice(g * per * P, (g + 1) * per * P)
        yg, hg = oracle.selscan_scalarA(x[:, csl], dt[:, hsl], A[hsl], B[:, g:g + 1],
                                        C[:, g:g + 1], P, D=D[hsl])
        np.testing.assert_allclose(y[:, csl], yg, rtol=0, atol=0)
        np.testing.assert_allclose(hs[:, hsl], hg, rtol=0, atol=0)
