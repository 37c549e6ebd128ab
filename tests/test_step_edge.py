"""GPU parity of the decode step (selscan_step, selscan_step_scalarA) on the
method's own edge cases ("03 -- Modelos de espacio de estados", section "El
mecanismo selectivo de Mamba": the step size decides whether the state is
kept or reset):

- a zero step with softplus off and no bias keeps the state bit for bit
  (the decay is exp(0) = 1 and nothing enters: h <- 1 * h + 0);
- a step with delta |A| >= 50 resets it: the new state is delta B u to the
  step's own rounding, and y and the state match the oracle's step;
- a zero input only decays the state (h <- abar h), against the oracle;
- inputs spanning 1e-30 .. 1e3 across channels, against the oracle.

Tolerances as in the other step tests: state relative L2 <= 1e-5 (fp32
arithmetic), y <= 1e-5 in fp32 and <= 5e-3 in bf16."""
import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def dev(a, dtype):
    import torch
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t.float()


def f32(a):
    import torch
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda().float()


def store(a, dtype):
    return synthetic.round_bf16(a) if dtype == "bf16" else np.ascontiguousarray(a, np.float32)


def diag_tok(dtype, seed):
    inp = synthetic.make_diag(4, 256, 16, 1, dtype=dtype, seed=seed, gate=True, bias=False)
    sq = lambda a: None if a is None else a[..., 0]
    return dict(u=sq(inp["u"]), delta=sq(inp["delta"]), z=sq(inp["z"]), B=sq(inp["B"]),
                C=sq(inp["C"]), A=inp["A"], D=inp["D"])


def diag_step(t, state0, dtype, softplus):
    import selective_state_space_selscan_b200 as ss
    state = f32(state0)
    y = ss.selscan_step(state, dev(t["u"], dtype), dev(t["delta"], dtype), f32(t["A"]),
                        dev(t["B"], dtype), dev(t["C"], dtype), D=f32(t["D"]),
                        z=dev(t["z"], dtype), delta_softplus=softplus)
    ss.check()
    y_ref, st_ref = oracle.selscan_step(state0, t["u"], t["delta"], t["A"], t["B"], t["C"],
                                        D=t["D"], z=t["z"], delta_softplus=softplus)
    return y.float().cpu().numpy(), state.cpu().numpy(), y_ref, st_ref


def state0_for(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_diag_zero_step_keeps_state_exactly(dtype):
    t = diag_tok(dtype, 91)
    t["delta"] = np.zeros_like(t["delta"])
    s0 = state0_for((4, 256, 16), 1)
    y, st, y_ref, st_ref = diag_step(t, s0, dtype, softplus=False)
    assert np.array_equal(st, s0), "state moved under a zero step"
    assert rel(y, y_ref) <= (1e-5 if dtype == "f32" else 5e-3)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_diag_large_step_resets_state(dtype):
    t = diag_tok(dtype, 92)
    t["delta"] = store(np.full_like(t["delta"], 60.0), dtype)
    s0 = state0_for((4, 256, 16), 2)
    y, st, y_ref, st_ref = diag_step(t, s0, dtype, softplus=False)
    assert rel(st, st_ref) <= 1e-5 and rel(y, y_ref) <= (1e-5 if dtype == "f32" else 5e-3)
    want = 60.0 * t["B"][:, None, :].astype(np.float64) * t["u"][:, :, None]
    assert rel(st, want) <= 1e-5, "the state did not forget its past"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_diag_zero_input_decays_state(dtype):
    t = diag_tok(dtype, 93)
    t["u"] = np.zeros_like(t["u"])
    s0 = state0_for((4, 256, 16), 3)
    y, st, y_ref, st_ref = diag_step(t, s0, dtype, softplus=True)
    assert rel(st, st_ref) <= 1e-5 and rel(y, y_ref) <= (1e-5 if dtype == "f32" else 5e-3)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_diag_input_dynamic_range(dtype):
    t = diag_tok(dtype, 94)
    rng = np.random.default_rng(4)
    mag = 10.0 ** rng.uniform(-30.0, 3.0, size=t["u"].shape)
    t["u"] = store((mag * np.where(rng.random(mag.shape) < 0.5, -1.0, 1.0)).astype(np.float32),
                   dtype)
    s0 = state0_for((4, 256, 16), 4)
    y, st, y_ref, st_ref = diag_step(t, s0, dtype, softplus=True)
    assert rel(st, st_ref) <= 1e-5 and rel(y, y_ref) <= (1e-5 if dtype == "f32" else 5e-3)


# ------------------------------------------------------------ scalar A
H, P, N = 4, 64, 128


def sa_tok(dtype, seed):
    return synthetic.make_scalarA(3, H, P, N, 1, dtype=dtype, seed=seed, gate=True)


def sa_step(inp, state0, dtype):
    import selective_state_space_selscan_b200 as ss
    sq = lambda a: None if a is None else a[..., 0]
    state = f32(state0)
    y = ss.selscan_step_scalarA(state, dev(sq(inp["x"]), dtype), f32(sq(inp["dt"])),
                                f32(inp["A"]), dev(sq(inp["B"]), dtype),
                                dev(sq(inp["C"]), dtype), P, D=f32(inp["D"]),
                                z=dev(sq(inp["z"]), dtype))
    ss.check()
    y_ref, st_ref = oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], P,
                                           D=inp["D"], z=inp["z"], h0=state0)
    return y.float().cpu().numpy(), state.cpu().numpy(), y_ref[..., 0], st_ref


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_scalarA_zero_step_keeps_state_exactly(dtype):
    inp = sa_tok(dtype, 95)
    inp["dt"] = np.zeros_like(inp["dt"])
    s0 = state0_for((3, H, P, N), 5)
    y, st, y_ref, st_ref = sa_step(inp, s0, dtype)
    assert np.array_equal(st, s0), "state moved under a zero step"
    assert rel(y, y_ref) <= (1e-5 if dtype == "f32" else 5e-3)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_scalarA_large_step_resets_state(dtype):
    inp = sa_tok(dtype, 96)
    inp["dt"] = np.broadcast_to((100.0 / np.abs(inp["A"]))[None, :, None],
                                inp["dt"].shape).astype(np.float32)
    s0 = state0_for((3, H, P, N), 6)
    y, st, y_ref, st_ref = sa_step(inp, s0, dtype)
    assert rel(st, st_ref) <= 1e-5 and rel(y, y_ref) <= (1e-5 if dtype == "f32" else 5e-3)
