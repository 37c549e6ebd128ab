"""Out-of-bounds write checks without a sanitizer: every output is a view
into a larger buffer whose guard regions (extra rows, extra columns before
and after each row, extra elements around contiguous outputs) are filled
with a canary; after the call the guards must be untouched.  Ragged shapes
so that bulk stores are clipped and tail chunks are partial."""
import numpy as np
import pytest

import synthetic

pytestmark = pytest.mark.gpu

CANARY = -8192.0  # exact in bf16 and fp32


def _dev(a, dtype):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t.float()


def _f32(a):
    import torch
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda().float()


def guarded_seq(shape, dtype):
    """(outer0, outer1, L) view inside a buffer with a guard row before and
    after and 8 guard columns on each side of every row."""
    import torch
    b, d, L = shape
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    buf = torch.full((b, d + 2, L + 16), CANARY, dtype=tdt, device="cuda")
    view = buf[:, 1:d + 1, 8:8 + L]
    mask = torch.ones_like(buf, dtype=torch.bool)
    mask[:, 1:d + 1, 8:8 + L] = False
    return buf, view, mask


def guarded_flat(shape):
    """Contiguous fp32 view with 4 guard elements before and after."""
    import torch
    n = int(np.prod(shape))
    buf = torch.full((n + 8,), CANARY, dtype=torch.float32, device="cuda")
    view = buf[4:4 + n].view(*shape)
    mask = torch.ones_like(buf, dtype=torch.bool)
    mask[4:4 + n] = False
    return buf, view, mask


def intact(buf, mask):
    return bool((buf.float()[mask] == CANARY).all())


@pytest.mark.parametrize("dtype,L,dim", [("bf16", 200, 136), ("f32", 100, 70)])
def test_scan_outputs_stay_in_bounds(dtype, L, dim):
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(2, dim, 16, L, dtype=dtype, seed=140)
    yb, y, ym = guarded_seq((2, dim, L), dtype)
    sb, st, sm = guarded_flat((2, dim, 16))
    ss.selscan_fwd(_dev(inp["u"], dtype), _dev(inp["delta"], dtype), _f32(inp["A"]),
                   _dev(inp["B"], dtype), _dev(inp["C"], dtype), D=_f32(inp["D"]),
                   z=_dev(inp["z"], dtype), delta_bias=_f32(inp["delta_bias"]), out=y,
                   last_state=st)
    ss.check()
    assert intact(yb, ym) and intact(sb, sm)
    assert bool((y.float() != CANARY).all())


def test_two_pass_outputs_stay_in_bounds():
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(1, 136, 16, 4104, dtype="bf16", seed=141)
    yb, y, ym = guarded_seq((1, 136, 4104), "bf16")
    sb, st, sm = guarded_flat((1, 136, 16))
    ss.debug_diag_mode(1)
    try:
        ss.selscan_fwd(_dev(inp["u"], "bf16"), _dev(inp["delta"], "bf16"), _f32(inp["A"]),
                       _dev(inp["B"], "bf16"), _dev(inp["C"], "bf16"), D=_f32(inp["D"]),
                       z=_dev(inp["z"], "bf16"), delta_bias=_f32(inp["delta_bias"]), out=y,
                       last_state=st)
        ss.check()
    finally:
        ss.debug_diag_mode(-1)
    assert intact(yb, ym) and intact(sb, sm)


def test_ssd_outputs_stay_in_bounds():
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_scalarA(2, 3, 64, 128, 200, seed=142)
    yb, y, ym = guarded_seq((2, 192, 200), "bf16")
    sb, st, sm = guarded_flat((2, 3, 64, 128))
    ss.selscan_fwd_scalarA(_dev(inp["x"], "bf16"), _f32(inp["dt"]), _f32(inp["A"]),
                           _dev(inp["B"], "bf16"), _dev(inp["C"], "bf16"), 64, D=_f32(inp["D"]),
                           out=y, last_state=st)
    ss.check()
    assert intact(yb, ym) and intact(sb, sm)


def test_step_outputs_stay_in_bounds():
    import torch
    import selective_state_space_selscan_b200 as ss
    t = synthetic.make_diag(3, 40, 16, 1, dtype="bf16", seed=143)
    sb, st, sm = guarded_flat((3, 40, 16))
    st.copy_(torch.randn(3, 40, 16, device="cuda"))
    yb = torch.full((3, 48), CANARY, dtype=torch.bfloat16, device="cuda")
    y = yb[:, 4:44]
    ym = torch.ones_like(yb, dtype=torch.bool)
    ym[:, 4:44] = False
    ss.selscan_step(st, _dev(t["u"][..., 0], "bf16"), _dev(t["delta"][..., 0], "bf16"),
                    _f32(t["A"]), _dev(t["B"][..., 0], "bf16"), _dev(t["C"][..., 0], "bf16"),
                    D=_f32(t["D"]), z=_dev(t["z"][..., 0], "bf16"),
                    delta_bias=_f32(t["delta_bias"]), out=y)
    ss.check()
    assert intact(sb, sm) and intact(yb, ym)


def test_bwd_outputs_stay_in_bounds():
    import torch
    import selective_state_space_selscan_b200 as ss
    from selective_state_space_selscan_b200 import describe, _ref, lib, _stream_handle
    L, dim = 100, 70
    inp = synthetic.make_diag(2, dim, 16, L, dtype="f32", seed=144)
    dy = np.random.default_rng(145).standard_normal(inp["u"].shape).astype(np.float32)
    bufs = {k: guarded_seq((2, dim, L), "f32") for k in ("du", "ddelta", "dz")}
    flats = {"dA": guarded_flat((dim, 16)), "dB": guarded_flat((2, 16, L)),
             "dC": guarded_flat((2, 16, L)), "dD": guarded_flat((dim,)),
             "dbias": guarded_flat((dim,)), "dh0": guarded_flat((2, dim, 16))}
    ins = [describe(_f32(inp[k])) for k in ("u", "delta", "delta_bias")]
    keep = [_f32(inp[k]) for k in ("A", "B", "C", "D", "z")] + [_f32(dy)]
    rest = [describe(keep[0]), describe(keep[1]), describe(keep[2]), describe(keep[3]),
            describe(keep[4]), None, describe(keep[5]), None]
    outs = [describe(bufs["du"][1]), describe(bufs["ddelta"][1]), describe(flats["dA"][1]),
            describe(flats["dB"][1]), describe(flats["dC"][1]), describe(flats["dD"][1]),
            describe(bufs["dz"][1]), describe(flats["dbias"][1]), describe(flats["dh0"][1])]
    rc = lib().selscan_bwd(_ref(ins[0]), _ref(ins[1]), _ref(ins[2]), 1,
                           *[_ref(x) for x in rest], *[_ref(x) for x in outs],
                           _stream_handle(None))
    assert rc == 0
    ss.check()
    for k, (b, _, m) in list(bufs.items()) + list(flats.items()):
        assert intact(b, m), k
