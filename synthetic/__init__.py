"""Seeded synthetic inputs for the selective scan.

This module is shared by the tests, the benchmark and the smoke entry; it
holds only random-number recipes and the bf16 storage rounding, none of the
scan's arithmetic.  Every array is produced on the host with numpy's PCG64
generator in a fixed order, so a (config, seed) pair always yields the same
bytes.  Arrays that a config stores in bf16 are returned as float32 arrays
whose values are exactly representable in bf16 (rounded to nearest even), so
the CUDA side converts them to bf16 without loss and the oracle widens the
very same values to fp64.

Distributions (shared by all diagonal-A configs):
  u, z ~ N(0, 1); B, C ~ N(0, 1) with shape (batch, N, L); D ~ N(0, 1);
  A[d, n] = -(n + 1)  (the S4D-real initialisation);
  Delta_raw = 0.5 * N(0, 1) and a per-channel bias chosen so that
  softplus(bias) is log-uniform on [lo, hi]; the scan applies the softplus.
Scalar-A (Mamba-2-style) config:
  x ~ N(0, 1); per-head A = -exp(U[log 1, log 16]); the step size is drawn
  directly, per head and token, log-uniform on [1e-3, 1e-1] (no softplus);
  B, C ~ N(0, 1) with shape (batch, ngroups, N, L); D ~ N(0, 1) per head.
"""
from __future__ import annotations

import math

import numpy as np

# Named workloads.  Index = position in the benchmark's config list.
CONFIGS = {
    0: dict(name="tiny fp32 scan (B1 D64 N16 L256)", kind="diag", batch=1,
            dim=64, N=16, L=256, dtype="f32", seed=0, dt_range=(1e-3, 1e-1),
            gate=False, D=True),
    1: dict(name="Mamba-130M-like layer scan (B8 D1536 N16 L2048, bf16, gate)",
            kind="diag", batch=8, dim=1536, N=16, L=2048, dtype="bf16",
            seed=1, dt_range=(1e-3, 1e-1), gate=True, D=True),
    2: dict(name="Mamba-2.8B-like layer scan (B4 D5120 N16 L4096, bf16, gate)",
            kind="diag", batch=4, dim=5120, N=16, L=4096, dtype="bf16",
            seed=2, dt_range=(1e-3, 1e-1), gate=True, D=True),
    3: dict(name="long-context scan (B1 D2048 N16 L131072, bf16)",
            kind="diag", batch=1, dim=2048, N=16, L=131072, dtype="bf16",
            seed=3, dt_range=(1e-4, 1e-1), gate=False, D=True),
    4: dict(name="Mamba-2-style scalar-A scan (B4 H32 P64 N128 G1 L4096, bf16)",
            kind="scalarA", batch=4, nheads=32, headdim=64, N=128, ngroups=1,
            L=4096, dtype="bf16", seed=4, dt_range=(1e-3, 1e-1), gate=False,
            D=True, chunk=256),
}


def round_bf16(a) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); the result is
    a float32 array holding bf16-exact values."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    bits = a.view(np.uint32)
    bits = (bits + np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1)))
    bits &= np.uint32(0xFFFF0000)
    return bits.view(np.float32)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    return round_bf16(a) if dtype == "bf16" else np.ascontiguousarray(a, np.float32)


def _log_uniform(rng, lo, hi, size):
    return np.exp(rng.uniform(math.log(lo), math.log(hi), size=size))


def make_diag(batch, dim, N, L, dtype="bf16", seed=0, dt_range=(1e-3, 1e-1),
              gate=True, D=True, bias=True, ngroups=None):
    """Inputs for the diagonal-A scan.  Returns a dict of float32 numpy
    arrays: u, delta, delta_bias, A, B, C, D, z (None where switched off),
    plus 'dtype' and 'softplus' (always True here)."""
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((batch, dim, L), dtype=np.float32)
    delta = 0.5 * rng.standard_normal((batch, dim, L), dtype=np.float32)
    target = _log_uniform(rng, dt_range[0], dt_range[1], dim)
    delta_bias = np.log(np.expm1(target)).astype(np.float32) if bias else None
    A = np.tile(-np.arange(1, N + 1, dtype=np.float32), (dim, 1))
    bshape = (batch, N, L) if ngroups is None else (batch, ngroups, N, L)
    B = rng.standard_normal(bshape, dtype=np.float32)
    C = rng.standard_normal(bshape, dtype=np.float32)
    Dv = rng.standard_normal(dim, dtype=np.float32) if D else None
    z = rng.standard_normal((batch, dim, L), dtype=np.float32) if gate else None
    return dict(
        u=_store(u, dtype), delta=_store(delta, dtype), delta_bias=delta_bias,
        A=A, B=_store(B, dtype), C=_store(C, dtype), D=Dv,
        z=None if z is None else _store(z, dtype), dtype=dtype, softplus=True)


def make_scalarA(batch, nheads, headdim, N, L, ngroups=1, dtype="bf16",
                 seed=0, dt_range=(1e-3, 1e-1), gate=False, D=True):
    """Inputs for the scalar-A scan: x, dt (fp32, already positive), A (H,),
    B, C (batch, G, N, L), D (H,), z (None unless gate)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((batch, nheads * headdim, L), dtype=np.float32)
    dt = _log_uniform(rng, dt_range[0], dt_range[1],
                      (batch, nheads, L)).astype(np.float32)
    A = (-np.exp(rng.uniform(0.0, math.log(16.0), size=nheads))).astype(np.float32)
    B = rng.standard_normal((batch, ngroups, N, L), dtype=np.float32)
    C = rng.standard_normal((batch, ngroups, N, L), dtype=np.float32)
    Dv = rng.standard_normal(nheads, dtype=np.float32) if D else None
    z = (rng.standard_normal((batch, nheads * headdim, L), dtype=np.float32)
         if gate else None)
    return dict(
        x=_store(x, dtype), dt=dt, dt_bias=None, A=A, B=_store(B, dtype),
        C=_store(C, dtype), D=Dv, z=None if z is None else _store(z, dtype),
        headdim=headdim, dtype=dtype, softplus=False)


def make_config(idx: int, **overrides):
    """Inputs of named config ``idx`` (see CONFIGS); keyword overrides
    replace any field (e.g. a smaller L for a fast test)."""
    cfg = dict(CONFIGS[idx])
    cfg.update(overrides)
    if cfg["kind"] == "diag":
        return make_diag(cfg["batch"], cfg["dim"], cfg["N"], cfg["L"],
                         dtype=cfg["dtype"], seed=cfg["seed"],
                         dt_range=cfg["dt_range"], gate=cfg["gate"],
                         D=cfg["D"])
    return make_scalarA(cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["N"],
                        cfg["L"], ngroups=cfg["ngroups"], dtype=cfg["dtype"],
                        seed=cfg["seed"], dt_range=cfg["dt_range"],
                        gate=cfg["gate"], D=cfg["D"])


def elements(idx: int) -> int:
    """batch * d_inner * L of config ``idx`` (the unit of the throughput)."""
    c = CONFIGS[idx]
    dim = c["dim"] if c["kind"] == "diag" else c["nheads"] * c["headdim"]
    return c["batch"] * dim * c["L"]
