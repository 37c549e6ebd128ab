"""fp64 CPU oracle for the selective scan (S6) and its scalar-A (SSD) form.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``smoke()`` in
``__graft_entry__.py`` and the CPU-baseline / reference leg of ``bench.py``
import this package.  It shares no code with the CUDA path and never imports
it; the product path never imports this package.

The arithmetic lives in ``selscan_oracle.c`` (plain single-threaded loops in
double precision, each routine citing the page passage it follows).  This
module only compiles that file with gcc and marshals numpy arrays into it.

Pinned by ``tests/test_oracle_pins.py`` against: a brute-force unrolled sum,
the time-invariant (LTI) special case as a causal convolution, the closed
form of a one-state geometric series (``tests/golden``), the Delta = 0 and
large-Delta gate invariants, linearity in the input, decode-step == scan,
scalar-A == diagonal scan with broadcast A, and the SSD chunked form ==
recurrence for several chunk lengths.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "selscan_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call([
        "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
        "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        common = [_i64] * 5
        lib.oracle_selscan.argtypes = common + [
            _dp, _dp, _dp, ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp,
            _dp, _dp, _i64, _i64]
        lib.oracle_selscan_step.argtypes = [_i64] * 4 + [
            _dp, _dp, _dp, ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
        scal = [_i64] * 6 + [_dp, _dp, _dp, ctypes.c_int, _dp, _dp, _dp,
                             _dp, _dp, _dp, _dp, _dp]
        lib.oracle_selscan_scalarA.argtypes = scal + [_i64, _i64]
        lib.oracle_ssd_chunked.argtypes = scal + [_i64]
        lib.oracle_selscan_bwd.argtypes = common + [
            _dp, _dp, _dp, ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp,
            _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
        for f in (lib.oracle_selscan, lib.oracle_selscan_step,
                  lib.oracle_selscan_scalarA, lib.oracle_ssd_chunked,
                  lib.oracle_selscan_bwd):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return arr, arr.ctypes.data_as(_dp)


def _check(rc: int) -> None:
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")


def _bc4(B, batch):
    """B/C given as (batch, N, L) are one group: view as (batch, 1, N, L)."""
    B = np.asarray(B)
    if B.ndim == 3:
        B = B.reshape(batch, 1, B.shape[1], B.shape[2])
    return B


def selscan(u, delta, A, B, C, D=None, z=None, delta_bias=None,
            delta_softplus=True, h0=None, channels=None):
    """Diagonal-A selective scan in fp64.

    u, delta, z: (batch, dim, L); A: (dim, N); B, C: (batch, N, L) or
    (batch, G, N, L); D, delta_bias: (dim,); h0: (batch, dim, N).
    ``channels`` = (begin, end) restricts the computation to those channels
    (the returned arrays then hold only those rows).
    Returns (y, last_state) as float64 arrays.
    """
    u = np.asarray(u)
    batch, dim, L = u.shape
    A = np.asarray(A)
    N = A.shape[1]
    B4, C4 = _bc4(B, batch), _bc4(C, batch)
    G = B4.shape[1]
    if channels is not None and tuple(channels) != (0, dim):
        # marshal only the requested channels (and their B/C group)
        d0, d1 = channels
        per = dim // G
        g0, g1 = d0 // per, (d1 - 1) // per
        if G > 1 and g0 != g1:
            raise ValueError("a channel sample must lie within one B/C group")
        sl = (lambda a: None if a is None else np.asarray(a)[:, d0:d1])
        vec = (lambda a: None if a is None else np.asarray(a)[d0:d1])
        return selscan(sl(u), sl(delta), np.asarray(A)[d0:d1], B4[:, g0:g0 + 1],
                       C4[:, g0:g0 + 1], D=vec(D), z=sl(z), delta_bias=vec(delta_bias),
                       delta_softplus=delta_softplus, h0=sl(h0), channels=None)
    d0, d1 = 0, dim
    keep = []
    uu, up = _f64(u); keep.append(uu)
    dd, dp_ = _f64(delta); keep.append(dd)
    bb, bp = _f64(delta_bias); keep.append(bb)
    aa, ap = _f64(A); keep.append(aa)
    BB, Bp = _f64(B4); keep.append(BB)
    CC, Cp = _f64(C4); keep.append(CC)
    DD, Dp = _f64(D); keep.append(DD)
    zz, zp = _f64(z); keep.append(zz)
    hh, hp = _f64(h0); keep.append(hh)
    y = np.zeros((batch, dim, L), dtype=np.float64)
    hs = np.zeros((batch, dim, N), dtype=np.float64)
    rc = _load().oracle_selscan(
        batch, dim, N, L, G, up, dp_, bp, int(bool(delta_softplus)), ap, Bp,
        Cp, Dp, zp, hp, y.ctypes.data_as(_dp), hs.ctypes.data_as(_dp), d0, d1)
    _check(rc)
    return y, hs


def selscan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None,
                delta_softplus=True, h0=None, dlast=None):
    """Gradients of the diagonal-A scan in fp64 for the loss
    sum(dy * y) + sum(dlast * last_state).  Shapes as in selscan; dy like u;
    dlast like h0.  Returns a dict with du, ddelta (like u), dA (like A),
    dB, dC (like B), and dD, dz, ddelta_bias, dh0 (None where the input is
    None)."""
    u = np.asarray(u)
    batch, dim, L = u.shape
    A = np.asarray(A)
    N = A.shape[1]
    B_in = np.asarray(B)
    B4, C4 = _bc4(B, batch), _bc4(C, batch)
    G = B4.shape[1]
    keep = []
    ptr = []
    for a in (u, delta, delta_bias, A, B4, C4, D, z, h0, dy, dlast):
        arr, pp = _f64(a)
        keep.append(arr)
        ptr.append(pp)
    out = {
        "du": np.zeros((batch, dim, L)), "ddelta": np.zeros((batch, dim, L)),
        "dA": np.zeros((dim, N)), "dB": np.zeros(B4.shape), "dC": np.zeros(C4.shape),
        "dD": np.zeros(dim) if D is not None else None,
        "dz": np.zeros((batch, dim, L)) if z is not None else None,
        "ddelta_bias": np.zeros(dim) if delta_bias is not None else None,
        "dh0": np.zeros((batch, dim, N)) if h0 is not None else None,
    }
    optr = lambda k: None if out[k] is None else out[k].ctypes.data_as(_dp)
    rc = _load().oracle_selscan_bwd(
        batch, dim, N, L, G, ptr[0], ptr[1], ptr[2], int(bool(delta_softplus)), ptr[3],
        ptr[4], ptr[5], ptr[6], ptr[7], ptr[8], ptr[9], ptr[10],
        optr("du"), optr("ddelta"), optr("dA"), optr("dB"), optr("dC"), optr("dD"),
        optr("dz"), optr("ddelta_bias"), optr("dh0"))
    _check(rc)
    out["dB"] = out["dB"].reshape(B_in.shape)
    out["dC"] = out["dC"].reshape(np.asarray(C).shape)
    return out


def selscan_step(state, u, delta, A, B, C, D=None, z=None, delta_bias=None,
                 delta_softplus=True):
    """One decode step.  state: (batch, dim, N) (not modified; a new state is
    returned); u, delta, z: (batch, dim); B, C: (batch, N) or (batch, G, N).
    Returns (y, new_state)."""
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    batch, dim, N = st.shape
    B = np.asarray(B)
    C = np.asarray(C)
    if B.ndim == 2:
        B = B.reshape(batch, 1, N)
        C = C.reshape(batch, 1, N)
    G = B.shape[1]
    keep = []
    uu, up = _f64(u); keep.append(uu)
    dd, dp_ = _f64(delta); keep.append(dd)
    bb, bp = _f64(delta_bias); keep.append(bb)
    aa, ap = _f64(A); keep.append(aa)
    BB, Bp = _f64(B); keep.append(BB)
    CC, Cp = _f64(C); keep.append(CC)
    DD, Dp = _f64(D); keep.append(DD)
    zz, zp = _f64(z); keep.append(zz)
    y = np.zeros((batch, dim), dtype=np.float64)
    rc = _load().oracle_selscan_step(
        batch, dim, N, G, up, dp_, bp, int(bool(delta_softplus)), ap, Bp, Cp,
        Dp, zp, st.ctypes.data_as(_dp), y.ctypes.data_as(_dp))
    _check(rc)
    return y, st


def _scalar_args(x, dt, A, B, C, D, z, dt_bias, h0, headdim):
    x = np.asarray(x)
    batch, dim, L = x.shape
    nheads = np.asarray(A).shape[0]
    if dim != nheads * headdim:
        raise ValueError("x.shape[1] must equal nheads * headdim")
    B4, C4 = _bc4(B, batch), _bc4(C, batch)
    G, N = B4.shape[1], B4.shape[2]
    keep = []
    ptrs = []
    for a in (x, dt, dt_bias):
        arr, p = _f64(a); keep.append(arr); ptrs.append(p)
    rest = []
    for a in (A, B4, C4, D, z, h0):
        arr, p = _f64(a); keep.append(arr); rest.append(p)
    return (batch, nheads, headdim, N, L, G), ptrs, rest, keep


def selscan_scalarA(x, dt, A, B, C, headdim, D=None, z=None, dt_bias=None,
                    dt_softplus=False, h0=None, heads=None):
    """Scalar-A scan, recurrent form.  x, z: (batch, H*P, L); dt: (batch, H, L);
    A, D, dt_bias: (H,); B, C: (batch, G, N, L) or (batch, N, L);
    h0: (batch, H, P, N).  ``heads`` = (begin, end) restricts the heads
    computed (returned arrays hold only those heads' channels/states).
    Returns (y, last_state) in float64."""
    nh = np.asarray(A).shape[0]
    if heads is not None and tuple(heads) != (0, nh):
        # marshal only the requested heads (and their B/C group)
        a0, a1 = heads
        Bq = _bc4(B, np.asarray(x).shape[0])
        Cq = _bc4(C, np.asarray(x).shape[0])
        per = nh // Bq.shape[1]
        g0, g1 = a0 // per, (a1 - 1) // per
        if Bq.shape[1] > 1 and g0 != g1:
            raise ValueError("a head sample must lie within one B/C group")
        ch = (lambda a: None if a is None else np.asarray(a)[:, a0 * headdim:a1 * headdim])
        hv = (lambda a: None if a is None else np.asarray(a)[a0:a1])
        return selscan_scalarA(ch(x), np.asarray(dt)[:, a0:a1], hv(A), Bq[:, g0:g0 + 1],
                               Cq[:, g0:g0 + 1], headdim, D=hv(D), z=ch(z),
                               dt_bias=hv(dt_bias), dt_softplus=dt_softplus,
                               h0=None if h0 is None else np.asarray(h0)[:, a0:a1])
    dims, ptrs, rest, keep = _scalar_args(x, dt, A, B, C, D, z, dt_bias, h0,
                                          headdim)
    batch, nheads, P, N, L, G = dims
    h0_, h1_ = 0, nheads
    y = np.zeros((batch, nheads * P, L), dtype=np.float64)
    hs = np.zeros((batch, nheads, P, N), dtype=np.float64)
    rc = _load().oracle_selscan_scalarA(
        *dims, ptrs[0], ptrs[1], ptrs[2], int(bool(dt_softplus)), *rest,
        y.ctypes.data_as(_dp), hs.ctypes.data_as(_dp), h0_, h1_)
    _check(rc)
    return y, hs


def ssd_chunked(x, dt, A, B, C, headdim, chunk, D=None, z=None, dt_bias=None,
                dt_softplus=False, h0=None):
    """Scalar-A scan in the chunked SSD matrix form (same arguments as
    ``selscan_scalarA`` plus the chunk length).  Returns (y, last_state)."""
    dims, ptrs, rest, keep = _scalar_args(x, dt, A, B, C, D, z, dt_bias, h0,
                                          headdim)
    batch, nheads, P, N, L, G = dims
    y = np.zeros((batch, nheads * P, L), dtype=np.float64)
    hs = np.zeros((batch, nheads, P, N), dtype=np.float64)
    rc = _load().oracle_ssd_chunked(
        *dims, ptrs[0], ptrs[1], ptrs[2], int(bool(dt_softplus)), *rest,
        y.ctypes.data_as(_dp), hs.ctypes.data_as(_dp), int(chunk))
    _check(rc)
    return y, hs


def selscan_scalarA_bwd(x, dt, A, B, C, headdim, dy, D=None, z=None, dt_bias=None,
                        dt_softplus=False, h0=None, dlast=None):
    """Gradients of the scalar-A scan (``selscan_scalarA``) in fp64 for the
    loss sum(dy * y) + sum(dlast * last_state).

    "Mamba-3: un modelo de espacio de estados centrado en la inferencia",
    first section: Mamba-2's transition is one scalar per head times the
    identity.  The scalar-A scan is therefore the diagonal scan with
    A[d, n] = A[h] for every channel d = h * P + p of head h and every state,
    the step size dt[b, h, t] (and dt_bias[h], D[h]) repeated over the head's
    P channels, and B / C of the head's group; its gradients are those of
    that diagonal problem (``selscan_bwd``) with every repeated parameter's
    gradient summed over the channels that share it (the chain rule for a
    copy).  Shapes as in ``selscan_scalarA``; dy like x; dlast like h0
    (batch, H, P, N).  Returns a dict with dx (like x), ddt (like dt), dA
    (H,), dB, dC (like B), and dD, dz, ddt_bias, dh0 (None where the input
    is None)."""
    x = np.asarray(x)
    batch, dim, L = x.shape
    A = np.asarray(A, dtype=np.float64)
    H = A.shape[0]
    P = int(headdim)
    if dim != H * P:
        raise ValueError("x.shape[1] must equal nheads * headdim")
    B4 = _bc4(B, batch)
    N = B4.shape[2]
    rep = lambda v: None if v is None else np.repeat(np.asarray(v, np.float64), P, axis=0)
    delta = np.repeat(np.asarray(dt, np.float64), P, axis=1)
    A_full = np.repeat(A, P)[:, None] * np.ones((1, N))
    flat = lambda s: None if s is None else np.asarray(s, np.float64).reshape(batch, dim, N)
    g = selscan_bwd(x, delta, A_full, B, C, dy, D=rep(D), z=z, delta_bias=rep(dt_bias),
                    delta_softplus=dt_softplus, h0=flat(h0), dlast=flat(dlast))
    per_head = lambda v: None if v is None else v.reshape(H, P, *v.shape[1:]).sum(axis=1)
    return {
        "dx": g["du"],
        "ddt": g["ddelta"].reshape(batch, H, P, L).sum(axis=2),
        "dA": g["dA"].reshape(H, P * N).sum(axis=1),
        "dB": g["dB"], "dC": g["dC"],
        "dD": per_head(g["dD"]),
        "dz": g["dz"],
        "ddt_bias": per_head(g["ddelta_bias"]),
        "dh0": None if g["dh0"] is None else g["dh0"].reshape(batch, H, P, N),
    }
