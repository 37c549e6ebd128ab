"""Whole-tensor oracle results for the GPU parity tests, computed on several
host threads.

Test infrastructure only.  The oracle itself is unchanged and
single-threaded: each call computes one contiguous range of channels (or
heads) with ``oracle.selscan`` / ``oracle.selscan_scalarA``, and the calls
run side by side because the oracle's C loop is entered through ctypes,
which releases the interpreter lock for the duration of the call.  The
ranges are independent problems (the scan has no coupling between channels),
so concatenating them gives exactly the single-call result.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle


def workers() -> int:
    return max(1, min(os.cpu_count() or 1, 32))


def _ranges(total: int, parts: int):
    edges = np.linspace(0, total, max(1, min(parts, total)) + 1).astype(int)
    return [(int(a), int(b)) for a, b in zip(edges[:-1], edges[1:]) if b > a]


def selscan(inp, h0=None, parts=None):
    """oracle.selscan over every channel of a diagonal-A input dict (as made
    by ``synthetic.make_diag``), split into channel ranges run in parallel.
    Returns (y, last_state) in float64, shapes (batch, dim, L), (batch, dim, N)."""
    dim = np.asarray(inp["u"]).shape[1]
    rs = _ranges(dim, parts or workers())

    def one(r):
        return oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                              D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                              delta_softplus=inp["softplus"], h0=h0, channels=r)

    with ThreadPoolExecutor(len(rs)) as ex:
        res = list(ex.map(one, rs))
    return (np.concatenate([r[0] for r in res], axis=1),
            np.concatenate([r[1] for r in res], axis=1))


def selscan_scalarA(inp, parts=None, dt_softplus=False, dt_bias=None, h0=None):
    """oracle.selscan_scalarA over every head of a scalar-A input dict (as made
    by ``synthetic.make_scalarA``), split into head ranges run in parallel."""
    H = np.asarray(inp["A"]).shape[0]
    rs = _ranges(H, parts or workers())

    def one(r):
        return oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                      inp["headdim"], D=inp["D"], z=inp["z"],
                                      dt_bias=dt_bias, dt_softplus=dt_softplus,
                                      h0=h0, heads=r)

    with ThreadPoolExecutor(len(rs)) as ex:
        res = list(ex.map(one, rs))
    return (np.concatenate([r[0] for r in res], axis=1),
            np.concatenate([r[1] for r in res], axis=1))


def selscan_bwd(inp, dy, parts=None, delta_softplus=True):
    """oracle.selscan_bwd over every channel of a diagonal-A input dict with
    one B/C group, split into channel ranges run in parallel.  The gradients
    of per-channel quantities (du, ddelta, dz, dA, dD, ddelta_bias) are those
    of each range, concatenated; dB and dC, sums over all channels, are the
    sums of the ranges' dB and dC (the loss is a sum over channels)."""
    u = np.asarray(inp["u"])
    batch, dim, _ = u.shape
    B = np.asarray(inp["B"])
    assert B.ndim == 3 or B.shape[1] == 1, "one B/C group (channel ranges keep no group map)"
    rs = _ranges(dim, parts or workers())

    def one(r):
        d0, d1 = r
        seq = lambda a: None if a is None else np.ascontiguousarray(np.asarray(a)[:, d0:d1])
        par = lambda a: None if a is None else np.ascontiguousarray(np.asarray(a)[d0:d1])
        return oracle.selscan_bwd(seq(inp["u"]), seq(inp["delta"]), par(inp["A"]), inp["B"],
                                  inp["C"], seq(dy), D=par(inp["D"]), z=seq(inp["z"]),
                                  delta_bias=par(inp["delta_bias"]),
                                  delta_softplus=delta_softplus)

    with ThreadPoolExecutor(len(rs)) as ex:
        res = list(ex.map(one, rs))
    out = {}
    for k, v in res[0].items():
        if v is None:
            out[k] = None
        elif k in ("dB", "dC"):
            out[k] = np.sum([r[k] for r in res], axis=0)
        elif k in ("du", "ddelta", "dz", "dh0"):
            out[k] = np.concatenate([r[k] for r in res], axis=1)
        else:
            out[k] = np.concatenate([r[k] for r in res], axis=0)
    return out


def selscan_scalarA_bwd(inp, dy, parts=None, dt_softplus=False, dt_bias=None):
    """oracle.selscan_scalarA_bwd over every head of a scalar-A input dict with
    one B/C group, split into head ranges run in parallel: per-head
    gradients concatenated, dB and dC summed over the ranges."""
    H = np.asarray(inp["A"]).shape[0]
    P = inp["headdim"]
    B = np.asarray(inp["B"])
    assert B.ndim == 3 or B.shape[1] == 1, "one B/C group (head ranges keep no group map)"
    rs = _ranges(H, parts or workers())

    def one(r):
        h0, h1 = r
        ch = lambda a: None if a is None else np.ascontiguousarray(np.asarray(a)[:, h0 * P:h1 * P])
        hd = lambda a: None if a is None else np.ascontiguousarray(np.asarray(a)[:, h0:h1])
        par = lambda a: None if a is None else np.ascontiguousarray(np.asarray(a)[h0:h1])
        return oracle.selscan_scalarA_bwd(ch(inp["x"]), hd(inp["dt"]), par(inp["A"]), inp["B"],
                                          inp["C"], P, ch(dy), D=par(inp["D"]), z=ch(inp["z"]),
                                          dt_bias=par(dt_bias), dt_softplus=dt_softplus)

    with ThreadPoolExecutor(len(rs)) as ex:
        res = list(ex.map(one, rs))
    out = {}
    for k, v in res[0].items():
        if v is None:
            out[k] = None
        elif k in ("dB", "dC"):
            out[k] = np.sum([r[k] for r in res], axis=0)
        elif k in ("dx", "dz", "ddt", "dh0"):
            out[k] = np.concatenate([r[k] for r in res], axis=1)
        else:
            out[k] = np.concatenate([r[k] for r in res], axis=0)
    return out
