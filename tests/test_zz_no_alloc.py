"""selscan_fwd_noalloc: the scan for callers that cannot allocate device
memory during a call (servers or real-time loops with a fixed memory
footprint, or systems without the stream-ordered allocator).  Its scratch
lives in a static device array shared by all calls, so every case makes two
calls in a row -- the second must not see the first one's tickets, flags,
carries or aggregates -- and checks both against the fp64 oracle (whole
tensor, tolerance as in the other parity tests) and bit for bit against the
allocating entry point selscan_fwd, which runs the same kernels with the same
work decomposition.

Shapes: more tiles than SMs, so several segments per tile (chained carries
in the array); ragged tiles and tail; fp32; few tiles over a long sequence
(the two-pass form, its aggregates in the array); and the two largest
scratch needs the scheduler produces on a 148-SM GPU (about 9.3 MiB
chained; 9.5 MiB two-pass among shapes the oracle checks in seconds, 9.6
MiB at most; of the 16 MiB array).

Kept in a file that pytest collects last; it also passes alone in a fresh
process (it builds its own inputs).
"""
import numpy as np
import pytest

import oracle_par
import synthetic

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 5e-3}


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


@pytest.mark.parametrize("shape,dtype", [
    ((2, 9600, 1024), "bf16"),     # 150 tiles x 4 segments: flags and carries in use
    ((2, 192, 1000), "bf16"),      # ragged tiles and tail
    ((1, 64, 256), "f32"),
    ((1, 256, 65536), "bf16"),     # two tiles, long sequence: the two-pass form
    ((1, 21632, 2048), "bf16"),    # 169 tiles x 8 segments: largest chained scratch
    ((1, 128, 303104), "bf16"),    # one tile, long: one wave of 148 segments, two-pass
    ((1, 4864, 9920), "bf16"),     # 38 tiles x 31 segments: largest two-pass scratch (oracle-sized)
])
def test_noalloc_matches_oracle_twice(shape, dtype):
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
    y_fwd, h_fwd = ss.selscan_fwd(*args, **kw)
    ss.check()
    y_ref, h_ref = oracle_par.selscan(inp)
    for call in range(2):
        y = torch.full_like(y_fwd, float("nan"))
        h = torch.full_like(h_fwd, float("nan"))
        ss.selscan_fwd_noalloc(*args, out=y, last_state=h, **kw)
        ss.check()
        yn, hn = y.float().cpu().numpy(), h.cpu().numpy()
        assert np.isfinite(yn).all() and np.isfinite(hn).all(), call
        ey, eh = _rel(yn, y_ref), _rel(hn, h_ref)
        assert ey <= TOL[dtype] and eh <= TOL[dtype], (call, ey, eh)
        assert torch.equal(y, y_fwd) and torch.equal(h, h_fwd), f"call {call} differs from selscan_fwd"
