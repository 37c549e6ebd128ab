"""GPU parity of the decode step (selscan_step, selscan_step_scalarA) with the
fp64 oracle: one step against the oracle's step (diagonal) or its scan over
one token from the given state (scalar A), and a chain of steps, carrying the
state in place, against the oracle's scan of the whole sequence ("03 --
Modelos de espacio de estados: RWKV, S4, Mamba y el selective scan",
sections "Parallel scan" and "Coste de inferencia": the recurrent and the
scanned form compute the same h_t).

Tolerances: y relative L2 <= 1e-5 in fp32 and <= 5e-3 in bf16 (the bf16
rounding of y alone is about 1e-3); the fp32 state <= 1e-5 per step (fp32
arithmetic on bf16-rounded inputs), 5e-3 after a chain of bf16 steps (each
y is rounded, the state is not, but the comparison is with the oracle's
single fp64 scan)."""
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


def tok(batch, dim, N, dtype, seed, groups=None, gate=True):
    """One token of diagonal-scan inputs (bf16-rounded where bf16)."""
    inp = synthetic.make_diag(batch, dim, N, 1, dtype=dtype, seed=seed, gate=gate,
                              ngroups=groups)
    sq = lambda a: None if a is None else a[..., 0]
    return dict(u=sq(inp["u"]), delta=sq(inp["delta"]), z=sq(inp["z"]), B=sq(inp["B"]),
                C=sq(inp["C"]), A=inp["A"], D=inp["D"], delta_bias=inp["delta_bias"])


@pytest.mark.parametrize("dtype,N,groups", [("f32", 16, None), ("bf16", 16, None),
                                            ("bf16", 16, 4), ("f32", 64, None),
                                            ("bf16", 128, 2)])
def test_diag_step_matches_oracle(dtype, N, groups):
    import selective_state_space_selscan_b200 as ss
    batch, dim = 3, 200
    t = tok(batch, dim, N, dtype, seed=61 + N, groups=groups)
    state0 = np.random.default_rng(7).standard_normal((batch, dim, N)).astype(np.float32)
    state = f32(state0)
    y = ss.selscan_step(state, dev(t["u"], dtype), dev(t["delta"], dtype), f32(t["A"]),
                        dev(t["B"], dtype), dev(t["C"], dtype), D=f32(t["D"]),
                        z=dev(t["z"], dtype), delta_bias=f32(t["delta_bias"]))
    ss.check()
    y_ref, st_ref = oracle.selscan_step(state0, t["u"], t["delta"], t["A"], t["B"], t["C"],
                                        D=t["D"], z=t["z"], delta_bias=t["delta_bias"])
    assert rel(state.cpu().numpy(), st_ref) <= 1e-5
    assert rel(y.float().cpu().numpy(), y_ref) <= (1e-5 if dtype == "f32" else 5e-3)


def test_diag_step_strided_views():
    """u and z as halves of one (batch, 2D) projection, B and C as slices of
    one (batch, R + 2N) projection: strided operands read in place."""
    import torch
    import selective_state_space_selscan_b200 as ss
    batch, dim, N, R = 4, 96, 16, 6
    rng = np.random.default_rng(8)
    xz = synthetic.round_bf16(rng.standard_normal((batch, 2 * dim)).astype(np.float32))
    xdbl = synthetic.round_bf16(rng.standard_normal((batch, R + 2 * N)).astype(np.float32))
    delta = synthetic.round_bf16(0.5 * rng.standard_normal((batch, dim)).astype(np.float32))
    A = np.tile(-np.arange(1, N + 1, dtype=np.float32), (dim, 1))
    Dv = rng.standard_normal(dim).astype(np.float32)
    state0 = rng.standard_normal((batch, dim, N)).astype(np.float32)
    xz_d, xdbl_d = dev(xz, "bf16"), dev(xdbl, "bf16")
    state = f32(state0)
    y = torch.zeros(batch, 2 * dim, dtype=torch.bfloat16, device="cuda")[:, ::2]
    ss.selscan_step(state, xz_d[:, :dim], dev(delta, "bf16"), f32(A), xdbl_d[:, R:R + N],
                    xdbl_d[:, R + N:], D=f32(Dv), z=xz_d[:, dim:], out=y)
    ss.check()
    y_ref, st_ref = oracle.selscan_step(state0, xz[:, :dim], delta, A, xdbl[:, R:R + N],
                                        xdbl[:, R + N:], D=Dv, z=xz[:, dim:])
    assert rel(state.cpu().numpy(), st_ref) <= 1e-5
    assert rel(y.float().cpu().numpy(), y_ref) <= 5e-3


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_diag_steps_equal_scan(dtype):
    """64 steps carrying the state in place reproduce the oracle's scan."""
    import torch
    import selective_state_space_selscan_b200 as ss
    batch, dim, N, L = 2, 128, 16, 64
    inp = synthetic.make_diag(batch, dim, N, L, dtype=dtype, seed=63)
    y_ref, st_ref = oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                   D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"])
    u, d, z = dev(inp["u"], dtype), dev(inp["delta"], dtype), dev(inp["z"], dtype)
    B, C = dev(inp["B"], dtype), dev(inp["C"], dtype)
    A, Dv, bias = f32(inp["A"]), f32(inp["D"]), f32(inp["delta_bias"])
    state = torch.zeros(batch, dim, N, device="cuda")
    ys = [ss.selscan_step(state, u[..., t], d[..., t], A, B[..., t], C[..., t], D=Dv,
                          z=z[..., t], delta_bias=bias) for t in range(L)]
    ss.check()
    y = torch.stack(ys, dim=-1).float().cpu().numpy()
    tol = 1e-5 if dtype == "f32" else 5e-3
    assert rel(y, y_ref) <= tol
    assert rel(state.cpu().numpy(), st_ref) <= tol


def scalar_tok(batch, H, P, N, G, dtype, seed, gate):
    inp = synthetic.make_scalarA(batch, H, P, N, 1, ngroups=G, dtype=dtype, seed=seed,
                                 gate=gate)
    return inp


@pytest.mark.parametrize("dtype,H,P,N,G,gate", [("bf16", 4, 64, 128, 1, False),
                                                ("bf16", 4, 64, 128, 2, True),
                                                ("f32", 3, 48, 16, 1, True),
                                                ("f32", 2, 64, 64, 2, False)])
def test_scalarA_step_matches_oracle(dtype, H, P, N, G, gate):
    import selective_state_space_selscan_b200 as ss
    batch = 3
    inp = scalar_tok(batch, H, P, N, G, dtype, seed=70 + N, gate=gate)
    rng = np.random.default_rng(9)
    bias = (0.3 * rng.standard_normal(H)).astype(np.float32)
    state0 = (0.5 * rng.standard_normal((batch, H, P, N))).astype(np.float32)
    state = f32(state0)
    sq = lambda a: None if a is None else a[..., 0]
    y = ss.selscan_step_scalarA(state, dev(sq(inp["x"]), dtype), f32(sq(inp["dt"])),
                                f32(inp["A"]), dev(sq(inp["B"]), dtype),
                                dev(sq(inp["C"]), dtype), P, D=f32(inp["D"]),
                                z=dev(sq(inp["z"]), dtype), dt_bias=f32(bias),
                                dt_softplus=True)
    ss.check()
    y_ref, st_ref = oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                           P, D=inp["D"], z=inp["z"], dt_bias=bias,
                                           dt_softplus=True, h0=state0)
    assert rel(state.cpu().numpy(), st_ref) <= 1e-5
    assert rel(y.float().cpu().numpy(), y_ref[..., 0]) <= (1e-5 if dtype == "f32" else 5e-3)


def test_scalarA_steps_equal_scan():
    """32 Mamba-2 decode steps in place against the oracle's scan."""
    import torch
    import selective_state_space_selscan_b200 as ss
    batch, H, P, N, L = 2, 3, 64, 128, 32
    inp = synthetic.make_scalarA(batch, H, P, N, L, seed=72, gate=True)
    y_ref, st_ref = oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                           P, D=inp["D"], z=inp["z"])
    x, z = dev(inp["x"], "bf16"), dev(inp["z"], "bf16")
    B, C = dev(inp["B"], "bf16"), dev(inp["C"], "bf16")
    dt, A, Dv = f32(inp["dt"]), f32(inp["A"]), f32(inp["D"])
    state = torch.zeros(batch, H, P, N, device="cuda")
    ys = [ss.selscan_step_scalarA(state, x[..., t], dt[..., t], A, B[..., t], C[..., t], P,
                                  D=Dv, z=z[..., t]) for t in range(L)]
    ss.check()
    y = torch.stack(ys, dim=-1).float().cpu().numpy()
    assert rel(y, y_ref) <= 5e-3
    assert rel(state.cpu().numpy(), st_ref) <= 5e-3


def test_step_empty_batch():
    import torch
    import selective_state_space_selscan_b200 as ss
    A = -torch.ones(32, 16, device="cuda")
    st = torch.empty(0, 32, 16, device="cuda")
    e = torch.empty(0, 32, dtype=torch.bfloat16, device="cuda")
    bc = torch.empty(0, 16, dtype=torch.bfloat16, device="cuda")
    y = ss.selscan_step(st, e, e, A, bc, bc)
    ss.check()
    assert y.shape == (0, 32)
