"""selscan_fwd_noalloc: the scan for callers that cannot allocate device
memory during a call (servers or real-time loops with a fixed memory
footprint, or systems without the stream-ordered allocator).  Its scratch
lives in a static device array shared by all calls, so this checks two calls
in a row -- the second must not see the first one's flags or carries --
against the allocating entry point, selscan_fwd, through the C ABI.

Kept in a file that pytest collects last; it also passes alone in a fresh
process (it builds its own inputs).
"""
import numpy as np
import pytest

import synthetic

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 5e-3}


def _rel(a, b):
    a = a.double()
    b = b.double()
    return float((a - b).norm() / b.norm().clamp_min(1e-30))


@pytest.mark.parametrize("shape,dtype", [
    ((8, 1536, 2048), "bf16"),   # several segments per tile: flags and carries in use
    ((2, 192, 1000), "bf16"),    # ragged tiles and tail
    ((1, 64, 256), "f32"),
])
def test_noalloc_matches_allocating_entry_twice(shape, dtype):
    import torch
    import selective_state_space_selscan_b200 as ss
    b, d, L = shape
    inp = synthetic.make_diag(b, d, 16, L, dtype=dtype, seed=77, gate=(dtype == "bf16"))
    cv = (lambda a: None if a is None else (
        torch.from_numpy(a).cuda().to(torch.bfloat16) if dtype == "bf16"
        else torch.from_numpy(a).cuda().float()))
    f32 = (lambda a: None if a is None else torch.from_numpy(a).cuda().float())
    args = (cv(inp["u"]), cv(inp["delta"]), f32(inp["A"]), cv(inp["B"]), cv(inp["C"]))
    kw = dict(D=f32(inp["D"]), z=cv(inp["z"]), delta_bias=f32(inp["delta_bias"]))
    y_ref, h_ref = ss.selscan_fwd(*args, **kw)
    ss.check()
    for call in range(2):
        y = torch.full_like(y_ref, float("nan"))
        h = torch.full_like(h_ref, float("nan"))
        ss.selscan_fwd_noalloc(*args, out=y, last_state=h, **kw)
        ss.check()
        assert torch.isfinite(y.float()).all() and torch.isfinite(h).all(), call
        ey, eh = _rel(y.float(), y_ref.float()), _rel(h, h_ref)
        assert ey <= TOL[dtype] and eh <= TOL[dtype], (call, ey, eh)
