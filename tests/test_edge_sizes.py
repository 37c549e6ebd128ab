"""Smallest shapes of every entry point against the fp64 oracle: a single
(partial) chunk, a single channel, channel counts that are not a multiple
of the tile, batch 1."""
import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("batch,dim,L,dtype", [(1, 1, 8, "bf16"), (1, 3, 40, "bf16"),
                                               (2, 129, 16, "bf16"), (1, 1, 4, "f32"),
                                               (3, 70, 12, "f32")])
def test_scan_tiny(batch, dim, L, dtype):
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(batch, dim, 16, L, dtype=dtype, seed=101 + dim + L)
    y, hs = ss.selscan_fwd(_dev(inp["u"], dtype), _dev(inp["delta"], dtype), _f32(inp["A"]),
                           _dev(inp["B"], dtype), _dev(inp["C"], dtype), D=_f32(inp["D"]),
                           z=_dev(inp["z"], dtype), delta_bias=_f32(inp["delta_bias"]))
    ss.check()
    y_ref, hs_ref = oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                   D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"])
    tol = 5e-3 if dtype == "bf16" else 1e-5
    assert rel(y.float().cpu().numpy(), y_ref) <= tol
    assert rel(hs.cpu().numpy(), hs_ref) <= tol


@pytest.mark.parametrize("L", [8, 64])
def test_ssd_tiny(L):
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_scalarA(1, 2, 64, 128, L, seed=110 + L)
    y, hs = ss.selscan_fwd_scalarA(_dev(inp["x"], "bf16"), _f32(inp["dt"]), _f32(inp["A"]),
                                   _dev(inp["B"], "bf16"), _dev(inp["C"], "bf16"), 64,
                                   D=_f32(inp["D"]))
    ss.check()
    y_ref, hs_ref = oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                           64, D=inp["D"])
    assert rel(y.float().cpu().numpy(), y_ref) <= 5e-3
    assert rel(hs.cpu().numpy(), hs_ref) <= 5e-3


def test_step_single_channel():
    import selective_state_space_selscan_b200 as ss
    t = synthetic.make_diag(1, 1, 16, 1, dtype="f32", seed=120)
    st0 = np.random.default_rng(121).standard_normal((1, 1, 16)).astype(np.float32)
    state = _f32(st0)
    y = ss.selscan_step(state, _f32(t["u"][..., 0]), _f32(t["delta"][..., 0]), _f32(t["A"]),
                        _f32(t["B"][..., 0]), _f32(t["C"][..., 0]), D=_f32(t["D"]),
                        z=_f32(t["z"][..., 0]), delta_bias=_f32(t["delta_bias"]))
    ss.check()
    y_ref, st_ref = oracle.selscan_step(st0, t["u"][..., 0], t["delta"][..., 0], t["A"],
                                        t["B"][..., 0], t["C"][..., 0], D=t["D"],
                                        z=t["z"][..., 0], delta_bias=t["delta_bias"])
    assert rel(y.cpu().numpy(), y_ref) <= 1e-5 and rel(state.cpu().numpy(), st_ref) <= 1e-5


@pytest.mark.parametrize("dim,L", [(1, 8), (33, 24)])
def test_bwd_tiny(dim, L):
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(1, dim, 16, L, dtype="f32", seed=130 + dim)
    dy = np.random.default_rng(131).standard_normal(inp["u"].shape).astype(np.float32)
    g = ss.selscan_bwd(_f32(inp["u"]), _f32(inp["delta"]), _f32(inp["A"]), _f32(inp["B"]),
                       _f32(inp["C"]), _f32(dy), D=_f32(inp["D"]), z=_f32(inp["z"]),
                       delta_bias=_f32(inp["delta_bias"]))
    ss.check()
    want = oracle.selscan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                              D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"])
    for k in ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias"):
        assert rel(g[k].cpu().numpy().reshape(want[k].shape), want[k]) <= 1e-4, k
