"""GPU parity of both backward passes on the method's own edge cases, against
the fp64 oracles' gradients on the same inputs ("03 -- Modelos de espacio de
estados", section "El mecanismo selectivo de Mamba": the step size decides
whether the state is kept or reset; "P20 -- Mamba", section 5: training runs
the chain rule through that recurrence, so the same stretches must hold in
the gradients).

Diagonal form (selscan_bwd): 2 x 256 channels x 4096 tokens, bf16 with the
library's own time-segment count and with 3 forced segments, and fp32; the
special stretches cross 8-token checkpoint chunks and segment boundaries.
Scalar-A form (selscan_bwd_scalarA): 4 heads x 1024 tokens (32 chunks of 32).

Tolerances as for the other backward tests: relative L2 per gradient, bf16
5e-3 for the bf16-stored gradients (du / dx, ddelta, dz) and 2e-3 for the
fp32 ones; fp32 inputs 1e-4."""
import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu

DIAG_FORMS = [("bf16", 0), ("bf16", 3), ("f32", 0)]
DIAG_IDS = ["bf16-auto-segments", "bf16-3-segments", "f32"]


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _dev(a, dtype):
    import torch
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t.float()


def _f32(a):
    import torch
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda().float()


def store(a, dtype):
    return synthetic.round_bf16(a) if dtype == "bf16" else np.ascontiguousarray(a, np.float32)


# ------------------------------------------------------------ diagonal form
def diag_base(dtype, seed, **kw):
    return synthetic.make_diag(2, 256, 16, 4096, dtype=dtype, seed=seed, **kw)


def diag_check(inp, segs, what, softplus=True):
    import selective_state_space_selscan_b200 as ss
    dtype = inp["dtype"]
    dy = store(np.random.default_rng(77).standard_normal(inp["u"].shape).astype(np.float32),
               dtype)
    ss.debug_bwd_segments(segs)
    try:
        g = ss.selscan_bwd(_dev(inp["u"], dtype), _dev(inp["delta"], dtype), _f32(inp["A"]),
                           _dev(inp["B"], dtype), _dev(inp["C"], dtype), _dev(dy, dtype),
                           D=_f32(inp["D"]), z=_dev(inp["z"], dtype),
                           delta_bias=_f32(inp["delta_bias"]), delta_softplus=softplus)
        ss.check()
    finally:
        ss.debug_bwd_segments(0)
    got = {k: (None if v is None else v.float().cpu().numpy()) for k, v in g.items()}
    want = oracle.selscan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                              D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                              delta_softplus=softplus)
    lo = 5e-3 if dtype == "bf16" else 1e-4
    hi = 2e-3 if dtype == "bf16" else 1e-4
    for k, w in want.items():
        if w is None:
            assert got[k] is None, (what, k)
            continue
        assert np.isfinite(got[k]).all(), (what, k)
        tol = lo if k in ("du", "ddelta", "dz") else hi
        e = rel(got[k].reshape(w.shape), w)
        assert e <= tol, f"{what} {k}: rel L2 {e:.3e} > {tol}"
    return got, want


@pytest.mark.parametrize("dtype,segs", DIAG_FORMS, ids=DIAG_IDS)
def test_diag_zero_input_runs(dtype, segs):
    """u = 0 over tokens 1000..1599 of every channel, over the first 130
    tokens of some channels, and over whole channels."""
    inp = diag_base(dtype, 61)
    u = inp["u"].copy()
    u[:, :, 1000:1600] = 0.0
    u[1, 100:108, :130] = 0.0
    u[0, :8, :] = 0.0
    inp["u"] = u
    diag_check(inp, segs, f"zero runs {dtype} segs {segs}")


@pytest.mark.parametrize("dtype,segs", DIAG_FORMS, ids=DIAG_IDS)
def test_diag_zero_step_run(dtype, segs):
    """Softplus off, no bias, Delta = 0 over the last 704 tokens: the state
    is frozen there, and the gradient flows back through that stretch
    unchanged (abar = 1)."""
    inp = diag_base(dtype, 62, bias=False)
    rng = np.random.default_rng(17)
    delta = np.abs(rng.standard_normal(inp["u"].shape).astype(np.float32)) * 0.05
    delta[:, :, 3392:] = 0.0
    inp["delta"] = store(delta, dtype)
    diag_check(inp, segs, f"zero step {dtype} segs {segs}", softplus=False)


@pytest.mark.parametrize("dtype,segs", DIAG_FORMS, ids=DIAG_IDS)
def test_diag_large_step_reset(dtype, segs):
    """Delta |A| >= 50 on tokens 1500..1503 (softplus off): the state is reset
    there, so no gradient reaches the tokens before it through the state."""
    inp = diag_base(dtype, 63, bias=False)
    rng = np.random.default_rng(18)
    delta = np.abs(rng.standard_normal(inp["u"].shape).astype(np.float32)) * 0.05
    delta[:, :, 1500:1504] = 50.0
    inp["delta"] = store(delta, dtype)
    diag_check(inp, segs, f"reset {dtype} segs {segs}", softplus=False)


@pytest.mark.parametrize("dtype,segs", DIAG_FORMS, ids=DIAG_IDS)
def test_diag_alternating_sign(dtype, segs):
    """u changes sign at every token."""
    inp = diag_base(dtype, 64)
    sgn = np.where(np.arange(4096) % 2 == 0, 1.0, -1.0).astype(np.float32)
    inp["u"] = store(np.abs(inp["u"]) * sgn, dtype)
    diag_check(inp, segs, f"alternating sign {dtype} segs {segs}")


@pytest.mark.parametrize("dtype,segs", DIAG_FORMS, ids=DIAG_IDS)
def test_diag_input_dynamic_range(dtype, segs):
    """|u| log-uniform over [1e-30, 1e3] token by token (random sign) on half
    of the channels."""
    inp = diag_base(dtype, 65)
    rng = np.random.default_rng(19)
    u = inp["u"].copy()
    mag = 10.0 ** rng.uniform(-30.0, 3.0, size=u[:, ::2].shape)
    sgn = np.where(rng.random(size=mag.shape) < 0.5, -1.0, 1.0)
    u[:, ::2] = (mag * sgn).astype(np.float32)
    inp["u"] = store(u, dtype)
    diag_check(inp, segs, f"dynamic range {dtype} segs {segs}")


# ------------------------------------------------------------ scalar-A form
P, N = 64, 128


def sa_base(seed, gate=False):
    inp = synthetic.make_scalarA(1, 4, P, N, 1024, ngroups=1, seed=seed, gate=gate, D=True)
    inp["dy"] = synthetic.round_bf16(
        np.random.default_rng(seed + 1000).standard_normal(inp["x"].shape).astype(np.float32))
    return inp


def sa_check(inp, what, softplus=False):
    import selective_state_space_selscan_b200 as ss
    bf = lambda a: _dev(a, "bf16")
    g = ss.selscan_bwd_scalarA(bf(inp["x"]), _f32(inp["dt"]), _f32(inp["A"]), bf(inp["B"]),
                               bf(inp["C"]), P, bf(inp["dy"]), D=_f32(inp["D"]),
                               z=bf(inp["z"]), dt_softplus=softplus)
    ss.check()
    got = {k: (None if v is None else v.float().cpu().numpy()) for k, v in g.items()}
    want = oracle.selscan_scalarA_bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], P,
                                      inp["dy"], D=inp["D"], z=inp["z"], dt_softplus=softplus)
    for k, w in want.items():
        if w is None:
            assert got[k] is None, (what, k)
            continue
        assert np.isfinite(got[k]).all(), (what, k)
        tol = 5e-3 if k in ("dx", "dz") else 2e-3
        e = rel(got[k].reshape(w.shape), w)
        assert e <= tol, f"{what} {k}: rel L2 {e:.3e} > {tol}"
    return got, want


def test_scalarA_zero_input_runs():
    """x = 0 over tokens 200..455 (eight whole chunks) of every head and over
    the whole of head 3, with the gate on."""
    inp = sa_base(81, gate=True)
    x = inp["x"].copy()
    x[:, :, 200:456] = 0.0
    x[:, 3 * P:4 * P, :] = 0.0
    inp["x"] = x
    sa_check(inp, "zero input runs")


def test_scalarA_zero_step_run():
    """Softplus off, dt = 0 over tokens 512..1023: the state is frozen there
    (every decay is 1, nothing enters), and the gradient passes through."""
    inp = sa_base(82)
    dt = inp["dt"].copy()
    dt[:, :, 512:] = 0.0
    inp["dt"] = dt
    sa_check(inp, "zero step run")


def test_scalarA_large_step_reset():
    """dt |A| = 100 on tokens 300..302 (inside a chunk) and on token 640 (the
    first of a chunk): the decays underflow to zero in fp32, which resets the
    state, and the masks of those chunks cut every path across the step."""
    inp = sa_base(83)
    dt = inp["dt"].copy()
    big = (100.0 / np.abs(inp["A"])).astype(np.float32)
    for t in (300, 301, 302, 640):
        dt[:, :, t] = big[None, :]
    inp["dt"] = dt
    sa_check(inp, "large step")


def test_scalarA_alternating_sign():
    """x changes sign at every token."""
    inp = sa_base(84)
    sgn = np.where(np.arange(1024) % 2 == 0, 1.0, -1.0).astype(np.float32)
    inp["x"] = synthetic.round_bf16(np.abs(inp["x"]) * sgn)
    sa_check(inp, "alternating sign")
