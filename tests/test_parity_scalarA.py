"""GPU parity of the scalar-A (Mamba-2 / SSD) scan, selscan_fwd_scalarA through
the C ABI, against the fp64 oracle (recurrent form) on the same seeded,
bf16-rounded inputs.  Tolerance: relative L2 <= 5e-3 for y and last_state
(bf16 inputs, fp32 state)."""
import math

import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu

TOL = 5e-3


def rel_l2(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))


def run_gpu(inp, dt_softplus=False, dt_bias=None):
    import torch
    import selective_state_space_selscan_b200 as ss
    bf = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch.bfloat16)
    f32 = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda().float()
    y, hs = ss.selscan_fwd_scalarA(bf(inp["x"]), f32(inp["dt"]), f32(inp["A"]), bf(inp["B"]),
                                   bf(inp["C"]), inp["headdim"], D=f32(inp["D"]), z=bf(inp["z"]),
                                   dt_bias=f32(dt_bias), dt_softplus=dt_softplus)
    ss.check()
    return y.float().cpu().numpy(), hs.cpu().numpy()


def run_oracle(inp, heads=None, dt_softplus=False, dt_bias=None):
    return oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                  inp["headdim"], D=inp["D"], z=inp["z"], dt_bias=dt_bias,
                                  dt_softplus=dt_softplus, heads=heads)


def check(y, hs, y_ref, hs_ref, what):
    assert np.isfinite(y).all() and np.isfinite(hs).all(), what
    ey, eh = rel_l2(y, y_ref), rel_l2(hs, hs_ref)
    assert ey <= TOL and eh <= TOL, f"{what}: rel L2 y={ey:.3e} state={eh:.3e}"


@pytest.mark.parametrize("L", [128, 296, 640])
def test_small_ragged(L):
    """Several chunks of 128 tokens and a ragged last chunk."""
    inp = synthetic.make_scalarA(2, 4, 64, 128, L, seed=41)
    y, hs = run_gpu(inp)
    y_ref, hs_ref = run_oracle(inp)
    check(y, hs, y_ref, hs_ref, f"L={L}")


def test_gate_bias_softplus():
    inp = synthetic.make_scalarA(1, 3, 64, 128, 384, seed=42, gate=True)
    rng = np.random.default_rng(3)
    raw = synthetic.round_bf16(rng.standard_normal(inp["dt"].shape).astype(np.float32)) * 0.5
    inp["dt"] = raw.astype(np.float32)
    bias = np.log(np.expm1(np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), 3)))).astype(np.float32)
    y, hs = run_gpu(inp, dt_softplus=True, dt_bias=bias)
    y_ref, hs_ref = run_oracle(inp, dt_softplus=True, dt_bias=bias)
    check(y, hs, y_ref, hs_ref, "gate+bias+softplus")


def test_strong_decay_no_overflow():
    """Large |A| and large steps: the mask factors must stay finite."""
    inp = synthetic.make_scalarA(1, 2, 64, 128, 256, seed=43)
    inp["A"] = np.array([-16.0, -40.0], np.float32)
    inp["dt"] = np.full_like(inp["dt"], 0.5)
    y, hs = run_gpu(inp)
    y_ref, hs_ref = run_oracle(inp)
    check(y, hs, y_ref, hs_ref, "strong decay")


def test_empty_sequence():
    import torch
    import selective_state_space_selscan_b200 as ss
    x = torch.empty(2, 128, 0, dtype=torch.bfloat16, device="cuda")
    dt = torch.empty(2, 2, 0, device="cuda")
    Bc = torch.empty(2, 1, 128, 0, dtype=torch.bfloat16, device="cuda")
    A = -torch.ones(2, device="cuda")
    st = torch.full((2, 2, 64, 128), 5.0, device="cuda")
    y, hs = ss.selscan_fwd_scalarA(x, dt, A, Bc, Bc, 64, last_state=st)
    ss.check()
    assert y.shape == (2, 128, 0) and torch.all(hs == 0)


def test_full_size_config4_whole():
    """Full config (B4 H32 P64 N128 L4096) in the benchmark's launch
    configuration, compared with the oracle on every head, channel, token and
    batch row (the oracle runs over head ranges on several host threads).
    The measured errors are printed (pytest -s) so that the cost of keeping
    the carried-in state in bf16 for the C h term is visible."""
    import oracle_par
    inp = synthetic.make_config(4)
    y, hs = run_gpu(inp)
    y_ref, hs_ref = oracle_par.selscan_scalarA(inp)
    check(y, hs, y_ref, hs_ref, "config 4")
    print(f"config 4: rel L2 y={rel_l2(y, y_ref):.3e} state={rel_l2(hs, hs_ref):.3e}")


@pytest.mark.parametrize("G", [2, 4])
def test_grouped_BC(G):
    """Several B/C groups (Mamba-2 with ngroups > 1): head h reads group
    h / (H / G)."""
    inp = synthetic.make_scalarA(2, 4, 64, 128, 384, ngroups=G, seed=44 + G)
    y, hs = run_gpu(inp)
    y_ref, hs_ref = run_oracle(inp)
    check(y, hs, y_ref, hs_ref, f"G={G}")
