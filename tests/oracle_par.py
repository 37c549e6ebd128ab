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
