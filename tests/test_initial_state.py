"""Initial state (selscan_fwd_h0 / selscan_fwd_scalarA_h0) against the fp64
oracle with h0, and chunked prefill: scanning [0, L1) and continuing from its
final state over [L1, L) must reproduce the single full scan ("Mamba-2 y
state-space models", 4.3: the layer carries a fixed-size state)."""
import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _dev(inp, dt):
    import torch
    cv = (lambda a: None if a is None else (
        torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch.bfloat16) if dt == "bf16"
        else torch.from_numpy(np.ascontiguousarray(a)).cuda().float()))
    f32 = (lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda().float())
    return cv, f32


@pytest.mark.parametrize("dtype,tol", [("bf16", 5e-3), ("f32", 1e-5)])
def test_diag_h0_matches_oracle(dtype, tol):
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(2, 192, 16, 1536, dtype=dtype, seed=51)
    h0 = np.random.default_rng(5).standard_normal((2, 192, 16)).astype(np.float32)
    cv, f32 = _dev(inp, dtype)
    y, hs = ss.selscan_fwd(cv(inp["u"]), cv(inp["delta"]), f32(inp["A"]), cv(inp["B"]),
                           cv(inp["C"]), D=f32(inp["D"]), z=cv(inp["z"]),
                           delta_bias=f32(inp["delta_bias"]), h0=f32(h0))
    ss.check()
    y_ref, hs_ref = oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                   D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"], h0=h0)
    assert rel(y.float().cpu().numpy(), y_ref) <= tol
    assert rel(hs.cpu().numpy(), hs_ref) <= tol


def test_diag_chunked_prefill_in_place():
    """Two calls with the state carried in place (h0 is last_state)."""
    import torch
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(4, 256, 16, 2048, dtype="bf16", seed=52)
    cv, f32 = _dev(inp, "bf16")
    u, d, z = cv(inp["u"]), cv(inp["delta"]), cv(inp["z"])
    B, C = cv(inp["B"]), cv(inp["C"])
    kw = dict(D=f32(inp["D"]), delta_bias=f32(inp["delta_bias"]))
    A = f32(inp["A"])
    L1 = 768
    state = torch.zeros(4, 256, 16, device="cuda")
    y1, _ = ss.selscan_fwd(u[..., :L1], d[..., :L1], A, B[..., :L1].contiguous(),
                           C[..., :L1].contiguous(), z=z[..., :L1], last_state=state, h0=state,
                           **kw)
    y2, _ = ss.selscan_fwd(u[..., L1:], d[..., L1:], A, B[..., L1:].contiguous(),
                           C[..., L1:].contiguous(), z=z[..., L1:], last_state=state, h0=state,
                           **kw)
    ss.check()
    y_ref, hs_ref = oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                   D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"])
    y = torch.cat([y1, y2], dim=2).float().cpu().numpy()
    assert rel(y, y_ref) <= 5e-3
    assert rel(state.cpu().numpy(), hs_ref) <= 5e-3


def test_scalarA_h0_matches_oracle():
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_scalarA(2, 3, 64, 128, 384, seed=53)
    h0 = (0.5 * np.random.default_rng(6).standard_normal((2, 3, 64, 128))).astype(np.float32)
    cv, f32 = _dev(inp, "bf16")
    y, hs = ss.selscan_fwd_scalarA(cv(inp["x"]), f32(inp["dt"]), f32(inp["A"]), cv(inp["B"]),
                                   cv(inp["C"]), 64, D=f32(inp["D"]), h0=f32(h0))
    ss.check()
    y_ref, hs_ref = oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                           64, D=inp["D"], h0=h0)
    assert rel(y.float().cpu().numpy(), y_ref) <= 5e-3
    assert rel(hs.cpu().numpy(), hs_ref) <= 5e-3


def test_empty_sequence_returns_h0():
    import torch
    import selective_state_space_selscan_b200 as ss
    A = -torch.arange(1, 17, dtype=torch.float32, device="cuda").repeat(64, 1)
    e = torch.empty(2, 64, 0, dtype=torch.bfloat16, device="cuda")
    Bc = torch.empty(2, 16, 0, dtype=torch.bfloat16, device="cuda")
    h0 = torch.randn(2, 64, 16, device="cuda")
    y, hs = ss.selscan_fwd(e, e, A, Bc, Bc, h0=h0)
    ss.check()
    assert torch.equal(hs, h0)
