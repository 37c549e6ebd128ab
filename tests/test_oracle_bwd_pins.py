"""Pins of the oracle's backward pass (oracle.selscan_bwd) against the
forward oracle alone: every gradient entry must equal the central finite
difference of the loss sum(dy * y) + sum(dlast * last_state), which is
computed from oracle.selscan only and shares no code with the backward
walk.  fp64 on tiny shapes, so the difference quotient is accurate to
~1e-9; the check is elementwise, so a dropped term, a wrong sign or index,
or a transposed operand in any gradient fails.

The backward rule itself is the chain rule through the recurrence of
"03 -- Modelos de espacio de estados" (sections "Discretizacion" and
"Parallel scan"): training differentiates the same recurrence that the
forward pass evaluates ("P20 -- Mamba", section 5)."""
import numpy as np
import pytest

import oracle

EPS = 1e-6


def _inputs(rng, batch, dim, N, L, G, gate, D, bias, h0):
    f = lambda *s: rng.standard_normal(s)
    inp = dict(u=f(batch, dim, L), delta=0.5 * f(batch, dim, L),
               A=-np.exp(rng.uniform(-1.0, 1.5, (dim, N))),
               B=f(batch, G, N, L), C=f(batch, G, N, L),
               D=f(dim) if D else None, z=f(batch, dim, L) if gate else None,
               delta_bias=0.3 * f(dim) if bias else None,
               h0=f(batch, dim, N) if h0 else None)
    return inp


def _loss(inp, dy, dlast, softplus):
    y, hs = oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                           z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=softplus,
                           h0=inp["h0"])
    val = float(np.sum(dy * y))
    if dlast is not None:
        val += float(np.sum(dlast * hs))
    return val


@pytest.mark.parametrize("gate,softplus,D,bias,h0,G", [
    (True, True, True, True, True, 1),
    (False, True, True, True, False, 1),
    (True, False, False, False, True, 1),
    (False, False, True, True, True, 3),
])
def test_gradients_equal_finite_differences(gate, softplus, D, bias, h0, G):
    rng = np.random.default_rng(11 + G + 2 * gate + 4 * softplus)
    batch, dim, N, L = 2, 3, 3, 5
    inp = _inputs(rng, batch, dim, N, L, G, gate, D, bias, h0)
    dy = rng.standard_normal((batch, dim, L))
    dlast = rng.standard_normal((batch, dim, N)) if h0 else None
    grads = oracle.selscan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                               D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                               delta_softplus=softplus, h0=inp["h0"], dlast=dlast)
    names = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
             "z": "dz", "delta_bias": "ddelta_bias", "h0": "dh0"}
    checked = 0
    for key, gname in names.items():
        if inp[key] is None:
            assert grads[gname] is None
            continue
        x = inp[key]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + EPS
            lp = _loss(inp, dy, dlast, softplus)
            x[idx] = keep - EPS
            lm = _loss(inp, dy, dlast, softplus)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * EPS)
        got = np.asarray(grads[gname]).reshape(x.shape)
        np.testing.assert_allclose(got, fd, rtol=1e-6, atol=1e-7, err_msg=gname)
        checked += x.size
    assert checked > 100


def test_zero_upstream_gradient_gives_zero():
    rng = np.random.default_rng(5)
    inp = _inputs(rng, 1, 2, 3, 4, 1, True, True, True, True)
    zero = np.zeros((1, 2, 4))
    g = oracle.selscan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], zero,
                           D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"])
    for k, v in g.items():
        if v is not None:
            assert np.all(v == 0.0), k


# ---------------------------------------------------------------- scalar A

def _sa_inputs(rng, batch, H, P, N, L, G, gate, D, bias, h0):
    f = lambda *s: rng.standard_normal(s)
    return dict(x=f(batch, H * P, L), dt=np.exp(rng.uniform(-3.0, -0.5, (batch, H, L))),
                A=-np.exp(rng.uniform(-1.0, 1.0, H)),
                B=f(batch, G, N, L), C=f(batch, G, N, L),
                D=f(H) if D else None, z=f(batch, H * P, L) if gate else None,
                dt_bias=0.3 * f(H) if bias else None,
                h0=f(batch, H, P, N) if h0 else None)


def _sa_loss(inp, P, dy, dlast, softplus):
    y, hs = oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], P,
                                   D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                   dt_softplus=softplus, h0=inp["h0"])
    val = float(np.sum(dy * y))
    if dlast is not None:
        val += float(np.sum(dlast * hs))
    return val


@pytest.mark.parametrize("gate,softplus,D,bias,h0,G", [
    (True, True, True, True, True, 1),
    (False, False, True, False, False, 1),
    (False, True, False, True, True, 2),
])
def test_scalarA_gradients_equal_finite_differences(gate, softplus, D, bias, h0, G):
    """oracle.selscan_scalarA_bwd against central differences of the
    scalar-A forward oracle (its own recurrence over heads, not the diagonal
    code): every entry of every gradient, including the per-head sums that
    the broadcast reading produces (dt, A, D, dt_bias shared by a head's
    channels; B, C shared by a group's heads)."""
    rng = np.random.default_rng(31 + G + 2 * gate + 4 * softplus)
    batch, H, P, N, L = 2, 2, 2, 3, 5
    inp = _sa_inputs(rng, batch, H, P, N, L, G, gate, D, bias, h0)
    dy = rng.standard_normal((batch, H * P, L))
    dlast = rng.standard_normal((batch, H, P, N)) if h0 else None
    grads = oracle.selscan_scalarA_bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], P, dy,
                                       D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                       dt_softplus=softplus, h0=inp["h0"], dlast=dlast)
    names = {"x": "dx", "dt": "ddt", "A": "dA", "B": "dB", "C": "dC", "D": "dD", "z": "dz",
             "dt_bias": "ddt_bias", "h0": "dh0"}
    checked = 0
    for key, gname in names.items():
        if inp[key] is None:
            assert grads[gname] is None
            continue
        v = inp[key]
        fd = np.zeros_like(v)
        for idx in np.ndindex(v.shape):
            keep = v[idx]
            v[idx] = keep + EPS
            lp = _sa_loss(inp, P, dy, dlast, softplus)
            v[idx] = keep - EPS
            lm = _sa_loss(inp, P, dy, dlast, softplus)
            v[idx] = keep
            fd[idx] = (lp - lm) / (2 * EPS)
        got = np.asarray(grads[gname]).reshape(v.shape)
        np.testing.assert_allclose(got, fd, rtol=1e-6, atol=1e-7, err_msg=gname)
        checked += v.size
    assert checked > 100
