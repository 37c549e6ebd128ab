"""CPU tests of the C ABI boundary: the library loads, exports every entry
point the headers declare, and rejects malformed arguments synchronously
(before any CUDA call) with the documented status codes.

Every call here uses placeholder pointers and is INVALID in at least one
way, so validation stops it before anything reaches a device.
"""
import ctypes
import glob
import os
import re

import pytest

import selective_state_space_selscan_b200 as ss

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names.update(re.findall(r"SELSCAN_API\s+[\w\s\*]+?\b(selscan_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    names = _declared_symbols()
    assert {"selscan_fwd", "selscan_fwd_scalarA", "selscan_check",
            "selscan_strerror", "selscan_version"} <= names
    lib = ctypes.CDLL(ss.LIB_PATH)
    for n in sorted(names):
        assert hasattr(lib, n), f"{n} declared but not exported"


def test_release_scratch_without_pools():
    """Before any call has allocated scratch there is nothing to trim, and
    the call makes no CUDA request (so it also runs without a GPU)."""
    ss.release_scratch()


def test_version_and_strerror():
    assert ss.version() == 10000
    for code in range(9):
        assert ss._strerror(code)
    assert "unknown" in ss._strerror(99)


FAKE = 0x7f0000000000  # 16-byte aligned placeholder, never dereferenced


def _t(shape, dtype=ss.SELSCAN_BF16, strides=None, data=FAKE):
    d = ss.SelscanTensor()
    d.data = data
    d.dtype = dtype
    d.ndim = len(shape)
    if strides is None:
        strides, acc = [], 1
        for s in reversed(shape):
            strides.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, strides)):
        d.shape[i] = s
        d.stride[i] = st
    return d


def _fwd(**over):
    b, D, N, L = 2, 64, 16, 128
    args = dict(u=_t((b, D, L)), delta=_t((b, D, L)), bias=_t((D,), ss.SELSCAN_F32),
                A=_t((D, N), ss.SELSCAN_F32), B=_t((b, N, L)), C=_t((b, N, L)),
                Dv=_t((D,), ss.SELSCAN_F32), z=_t((b, D, L)), y=_t((b, D, L)),
                hs=_t((b, D, N), ss.SELSCAN_F32))
    args.update(over)
    r = lambda x: None if x is None else ctypes.byref(x)
    return ss.lib().selscan_fwd(r(args["u"]), r(args["delta"]), r(args["bias"]), 1,
                                r(args["A"]), r(args["B"]), r(args["C"]), r(args["Dv"]),
                                r(args["z"]), r(args["y"]), r(args["hs"]), None)


C = ss.STATUS_CODE


@pytest.mark.parametrize("over,expect", [
    (dict(u=None), "SELSCAN_ERR_NULL"),
    (dict(y=None), "SELSCAN_ERR_NULL"),
    (dict(B=_t((2, 16, 128), data=0)), "SELSCAN_ERR_NULL"),
    (dict(delta=_t((2, 64, 127))), "SELSCAN_ERR_SHAPE"),
    (dict(A=_t((63, 16), ss.SELSCAN_F32)), "SELSCAN_ERR_SHAPE"),
    (dict(hs=_t((2, 64, 8), ss.SELSCAN_F32)), "SELSCAN_ERR_SHAPE"),
    (dict(z=_t((2, 64, 128), ss.SELSCAN_F32)), "SELSCAN_ERR_DTYPE"),
    (dict(bias=_t((64,), ss.SELSCAN_BF16)), "SELSCAN_ERR_DTYPE"),
    (dict(u=_t((2, 64, 128), dtype=7)), "SELSCAN_ERR_DTYPE"),
    (dict(u=_t((2, 64, 128), strides=(8192, 128, 2))), "SELSCAN_ERR_STRIDE"),
    (dict(A=_t((64, 16), ss.SELSCAN_F32, strides=(1, 64))), "SELSCAN_ERR_STRIDE"),
    (dict(u=_t((2, 64, 128), data=FAKE + 8)), "SELSCAN_ERR_ALIGN"),
    (dict(y=_t((2, 64, 128), strides=(8192, 124, 1))), "SELSCAN_ERR_ALIGN"),
    (dict(B=_t((2, 2, 16, 128))), "SELSCAN_ERR_UNSUPPORTED"),
])
def test_fwd_rejects(over, expect):
    assert _fwd(**over) == C[expect]


def test_fwd_rejects_state_size_other_than_16():
    b, D, N, L = 1, 32, 8, 64
    rc = _fwd(A=_t((D, N), ss.SELSCAN_F32), u=_t((b, D, L)), delta=_t((b, D, L)),
              B=_t((b, N, L)), C=_t((b, N, L)), y=_t((b, D, L)), z=None,
              bias=_t((D,), ss.SELSCAN_F32), Dv=_t((D,), ss.SELSCAN_F32),
              hs=_t((b, D, N), ss.SELSCAN_F32), )
    assert rc == C["SELSCAN_ERR_UNSUPPORTED"]


def _scal(**over):
    b, H, P, N, L, G = 2, 4, 64, 128, 256, 1
    args = dict(x=_t((b, H * P, L)), dt=_t((b, H, L), ss.SELSCAN_F32), bias=None,
                A=_t((H,), ss.SELSCAN_F32), B=_t((b, G, N, L)), C=_t((b, G, N, L)),
                Dv=_t((H,), ss.SELSCAN_F32), z=None, P=P, y=_t((b, H * P, L)),
                hs=_t((b, H, P, N), ss.SELSCAN_F32))
    args.update(over)
    r = lambda x: None if x is None else ctypes.byref(x)
    return ss.lib().selscan_fwd_scalarA(r(args["x"]), r(args["dt"]), r(args["bias"]), 0,
                                        r(args["A"]), r(args["B"]), r(args["C"]),
                                        r(args["Dv"]), r(args["z"]), args["P"], r(args["y"]),
                                        r(args["hs"]), None)


@pytest.mark.parametrize("over,expect", [
    (dict(x=None), "SELSCAN_ERR_NULL"),
    (dict(P=32), "SELSCAN_ERR_SHAPE"),
    (dict(x=_t((2, 256, 256), ss.SELSCAN_F32)), "SELSCAN_ERR_DTYPE"),
    (dict(dt=_t((2, 4, 256))), "SELSCAN_ERR_DTYPE"),
    (dict(B=_t((2, 1, 128, 255))), "SELSCAN_ERR_SHAPE"),
    (dict(hs=_t((2, 4, 64, 64), ss.SELSCAN_F32)), "SELSCAN_ERR_SHAPE"),
    (dict(x=_t((2, 256, 256), data=FAKE + 4)), "SELSCAN_ERR_ALIGN"),
    (dict(B=_t((2, 2, 64, 256)), C=_t((2, 2, 64, 256)),
          hs=_t((2, 4, 64, 64), ss.SELSCAN_F32)), "SELSCAN_ERR_UNSUPPORTED"),
])
def test_scalarA_rejects(over, expect):
    assert _scal(**over) == C[expect]


def _step(scalar=False, **over):
    b, D, N = 2, 64, 16
    if scalar:
        H, P, N = 2, 32, 128
        args = dict(state=_t((b, H, P, N), ss.SELSCAN_F32), u=_t((b, H * P)),
                    delta=_t((b, H), ss.SELSCAN_F32), bias=None, A=_t((H,), ss.SELSCAN_F32),
                    B=_t((b, N)), C=_t((b, N)), Dv=_t((H,), ss.SELSCAN_F32), z=None,
                    y=_t((b, H * P)), P=P)
    else:
        args = dict(state=_t((b, D, N), ss.SELSCAN_F32), u=_t((b, D)), delta=_t((b, D)),
                    bias=_t((D,), ss.SELSCAN_F32), A=_t((D, N), ss.SELSCAN_F32),
                    B=_t((b, N)), C=_t((b, N)), Dv=_t((D,), ss.SELSCAN_F32), z=_t((b, D)),
                    y=_t((b, D)))
    args.update(over)
    r = lambda x: None if x is None else ctypes.byref(x)
    common = (r(args["state"]), r(args["u"]), r(args["delta"]), r(args["bias"]), 1,
              r(args["A"]), r(args["B"]), r(args["C"]), r(args["Dv"]), r(args["z"]))
    if scalar:
        return ss.lib().selscan_step_scalarA(*common, args["P"], r(args["y"]), None)
    return ss.lib().selscan_step(*common, r(args["y"]), None)


@pytest.mark.parametrize("over,expect", [
    (dict(state=None), "SELSCAN_ERR_NULL"),
    (dict(y=None), "SELSCAN_ERR_NULL"),
    (dict(u=_t((2, 64, 1))), "SELSCAN_ERR_SHAPE"),
    (dict(delta=_t((2, 64), ss.SELSCAN_F32)), "SELSCAN_ERR_DTYPE"),
    (dict(state=_t((2, 64, 16), ss.SELSCAN_F32, data=FAKE + 4)), "SELSCAN_ERR_ALIGN"),
    (dict(state=_t((2, 64, 16), ss.SELSCAN_F32, strides=(2048, 32, 1))), "SELSCAN_ERR_STRIDE"),
    (dict(B=_t((2, 3, 16)), C=_t((2, 3, 16))), "SELSCAN_ERR_SHAPE"),
    (dict(B=_t((2, 2, 16)), C=_t((2, 4, 16))), "SELSCAN_ERR_SHAPE"),
    (dict(y=_t((2, 64), strides=(-64, 1))), "SELSCAN_ERR_STRIDE"),
    (dict(A=_t((64, 8), ss.SELSCAN_F32), state=_t((2, 64, 8), ss.SELSCAN_F32),
          B=_t((2, 8)), C=_t((2, 8))), "SELSCAN_ERR_UNSUPPORTED"),
])
def test_step_rejects(over, expect):
    assert _step(**over) == C[expect]


@pytest.mark.parametrize("over,expect", [
    (dict(P=48), "SELSCAN_ERR_SHAPE"),
    (dict(delta=_t((2, 2))), "SELSCAN_ERR_DTYPE"),
    (dict(state=_t((2, 2, 32, 64), ss.SELSCAN_F32)), "SELSCAN_ERR_SHAPE"),
    (dict(A=_t((2, 1), ss.SELSCAN_F32)), "SELSCAN_ERR_SHAPE"),
])
def test_step_scalarA_rejects(over, expect):
    assert _step(scalar=True, **over) == C[expect]


def _bwd(**over):
    b, D, N, L = 2, 64, 16, 48
    f32 = ss.SELSCAN_F32
    args = dict(u=_t((b, D, L)), delta=_t((b, D, L)), bias=None, A=_t((D, N), f32),
                B=_t((b, N, L)), C=_t((b, N, L)), Dv=None, z=None, h0=None, dy=_t((b, D, L)),
                dlast=None, du=_t((b, D, L)), dd=_t((b, D, L)), dA=_t((D, N), f32),
                dB=_t((b, N, L), f32), dC=_t((b, N, L), f32), dD=None, dz=None, dbias=None,
                dh0=None)
    args.update(over)
    r = lambda x: None if x is None else ctypes.byref(x)
    order = ("u", "delta", "bias")
    rest = ("A", "B", "C", "Dv", "z", "h0", "dy", "dlast", "du", "dd", "dA", "dB", "dC",
            "dD", "dz", "dbias", "dh0")
    return ss.lib().selscan_bwd(r(args["u"]), r(args["delta"]), r(args["bias"]), 1,
                                *[r(args[k]) for k in rest], None)


@pytest.mark.parametrize("over,expect", [
    (dict(u=None), "SELSCAN_ERR_NULL"),
    (dict(dy=None), "SELSCAN_ERR_NULL"),
    (dict(dA=None), "SELSCAN_ERR_NULL"),
    (dict(dy=_t((2, 64, 47))), "SELSCAN_ERR_SHAPE"),
    (dict(du=_t((2, 64, 48), ss.SELSCAN_F32)), "SELSCAN_ERR_DTYPE"),
    (dict(dB=_t((2, 16, 48))), "SELSCAN_ERR_DTYPE"),
    (dict(z=_t((2, 64, 48))), "SELSCAN_ERR_NULL"),          # gate given, dz missing
    (dict(dh0=_t((2, 64, 8), ss.SELSCAN_F32)), "SELSCAN_ERR_SHAPE"),
    (dict(delta=_t((2, 64, 48), strides=(64 * 96, 96, 2))), "SELSCAN_ERR_STRIDE"),
    (dict(A=_t((64, 8), ss.SELSCAN_F32), dA=_t((64, 8), ss.SELSCAN_F32),
          B=_t((2, 8, 48)), C=_t((2, 8, 48)), dB=_t((2, 8, 48), ss.SELSCAN_F32),
          dC=_t((2, 8, 48), ss.SELSCAN_F32)), "SELSCAN_ERR_UNSUPPORTED"),
    (dict(u=_t((2, 64, 48), dtype=7)), "SELSCAN_ERR_DTYPE"),
    (dict(dy=_t((2, 64, 48), data=FAKE + 8)), "SELSCAN_ERR_ALIGN"),
    (dict(du=_t((2, 64, 48), strides=(64 * 48, 44, 1))), "SELSCAN_ERR_ALIGN"),
    (dict(dB=_t((2, 16, 48), ss.SELSCAN_F32, strides=(16 * 48, 1, 16))), "SELSCAN_ERR_STRIDE"),
    (dict(dC=None), "SELSCAN_ERR_NULL"),
    (dict(h0=_t((2, 64, 16))), "SELSCAN_ERR_DTYPE"),          # bf16 initial state
    (dict(dlast=_t((2, 63, 16), ss.SELSCAN_F32)), "SELSCAN_ERR_SHAPE"),
    (dict(B=_t((2, 2, 16, 48))), "SELSCAN_ERR_UNSUPPORTED"),  # groups of B / C
])
def test_bwd_rejects(over, expect):
    assert _bwd(**over) == C[expect]


def _bwd_sa(**over):
    b, H, P, N, L, G = 2, 4, 64, 128, 64, 1
    f32 = ss.SELSCAN_F32
    args = dict(x=_t((b, H * P, L)), dt=_t((b, H, L), f32), bias=None, A=_t((H,), f32),
                B=_t((b, G, N, L)), C=_t((b, G, N, L)), Dv=None, z=None, P=P, h0=None,
                dy=_t((b, H * P, L)), dlast=None, dx=_t((b, H * P, L)), ddt=_t((b, H, L), f32),
                dA=_t((H,), f32), dB=_t((b, G, N, L), f32), dC=_t((b, G, N, L), f32),
                dD=None, dz=None, dbias=None, dh0=None)
    args.update(over)
    r = lambda x: None if x is None else ctypes.byref(x)
    mid = ("A", "B", "C", "Dv", "z")
    tail = ("h0", "dy", "dlast", "dx", "ddt", "dA", "dB", "dC", "dD", "dz", "dbias", "dh0")
    return ss.lib().selscan_bwd_scalarA(r(args["x"]), r(args["dt"]), r(args["bias"]), 0,
                                        *[r(args[k]) for k in mid], args["P"],
                                        *[r(args[k]) for k in tail], None)


@pytest.mark.parametrize("over,expect", [
    (dict(x=None), "SELSCAN_ERR_NULL"),
    (dict(dy=None), "SELSCAN_ERR_NULL"),
    (dict(ddt=None), "SELSCAN_ERR_NULL"),
    (dict(dB=None), "SELSCAN_ERR_NULL"),
    (dict(z=_t((2, 256, 64))), "SELSCAN_ERR_NULL"),           # gate given, dz missing
    (dict(P=48), "SELSCAN_ERR_SHAPE"),
    (dict(x=_t((2, 256, 64), ss.SELSCAN_F32)), "SELSCAN_ERR_DTYPE"),
    (dict(dt=_t((2, 4, 64))), "SELSCAN_ERR_DTYPE"),             # bf16 step sizes
    (dict(ddt=_t((2, 4, 63), ss.SELSCAN_F32)), "SELSCAN_ERR_SHAPE"),
    (dict(dB=_t((2, 1, 128, 64))), "SELSCAN_ERR_DTYPE"),        # bf16 gradient of B
    (dict(dC=_t((2, 2, 128, 64), ss.SELSCAN_F32)), "SELSCAN_ERR_SHAPE"),
    (dict(dh0=_t((2, 4, 64, 64), ss.SELSCAN_F32)), "SELSCAN_ERR_SHAPE"),
    (dict(B=_t((2, 3, 128, 64)), C=_t((2, 3, 128, 64))), "SELSCAN_ERR_SHAPE"),  # 3 does not divide 4
    (dict(B=_t((2, 1, 128, 64), strides=(128 * 128, 128 * 128, 128, 2))), "SELSCAN_ERR_STRIDE"),
    (dict(dx=_t((2, 256, 64), data=FAKE + 8)), "SELSCAN_ERR_ALIGN"),
    (dict(B=_t((2, 1, 64, 64)), C=_t((2, 1, 64, 64)), dB=_t((2, 1, 64, 64), ss.SELSCAN_F32),
          dC=_t((2, 1, 64, 64), ss.SELSCAN_F32)), "SELSCAN_ERR_UNSUPPORTED"),
])
def test_bwd_scalarA_rejects(over, expect):
    assert _bwd_sa(**over) == C[expect]


def test_forward_segment_plan():
    """The forward's choice of time segments and form (host arithmetic, no
    GPU): few tiles (2 tiles <= CTAs) with a spread of more than one
    segment take the two-pass form, with the count (at most the spread)
    that minimises whole waves of units per pass plus the folds of earlier
    segments; otherwise the chained form takes one segment when the tiles
    fit on the CTAs (a tile's segments run one after another, so more
    segments only lengthen that chain) and the spread rule (about 8 units
    per CTA, segments of at least 4 chunks) when they do not.  Negative
    values denote the two-pass form."""
    plan = ss.debug_fwd_plan
    assert plan(160, 64, 148) == 8         # B4 D5120 L4096: 8 segments
    assert plan(96, 32, 148) == 1          # B8 D1536 L2048: one segment per tile
    assert plan(128, 64, 148) == 1         # B4 D4096 L4096
    assert plan(75, 64, 148) == 1          # 2 x 75 > 148: still chained
    assert plan(74, 64, 148) == -2         # 2 x 74 <= 148: two-pass, one wave of units
    assert plan(16, 2048, 148) == -37      # B1 D2048 L131072: 4 waves of 56 chunks
    assert plan(1, 4736, 148) == -148      # one tile, long: one wave (the spread: 1184)
    assert plan(2, 1024, 148) == -74       # B1 D256 L65536: one wave
    assert plan(32, 512, 148) == -9        # B2 D2048 L32768
    assert plan(320, 16, 148) == 4         # B16 D2560 L1024: spread, capped at 16 / 4
    assert plan(169, 32, 148) == 8         # the largest chained scratch
    assert plan(1, 4, 148) == 1            # one chunk group: nothing to split
    assert plan(0, 10, 10) == 1 and plan(10, 0, 10) == 1 and plan(10, 10, 0) == 1
    for tiles in (1, 7, 74, 75, 148, 149, 640, 3000):
        for chunks in (1, 3, 4, 64, 2048):
            s = plan(tiles, chunks, 148)
            assert 1 <= abs(s) <= max(1, (chunks + 3) // 4)
            if s < 0:
                assert 2 * tiles <= 148 and s < -1
                spread = min(-(-8 * 148 // tiles), (chunks + 3) // 4)
                assert -s <= spread
            elif tiles <= 148:
                assert s == 1 or 2 * tiles <= 148


def test_backward_segment_plan():
    """The backward's choice of time segments (host arithmetic, no GPU):
    ceil(units / slots) / S is minimised over at most four waves, with at
    least 32 checkpoint chunks per segment, and among near-ties the
    smallest S that gives 1.5 waves or more is taken.  1184 slots = 8
    resident warps on each of 148 SMs."""
    plan = ss.debug_bwd_plan
    assert plan(640, 512, 1184) == 7       # B4 D5120 L4096: 4480 units, 3.8 waves
    assert plan(384, 256, 1184) == 6       # B8 D1536 L2048: 2304 units, 1.95 waves
    assert plan(64, 16384, 1184) == 37     # B1 D2048 L131072: 2368 units, 2 waves
    assert plan(640, 128, 1184) == 3       # L = 1024: at most 4 segments of 32 chunks
    assert plan(2, 31, 1184) == 1          # fewer than 32 chunks: one segment
    assert plan(5000, 512, 1184) == 1      # more than four waves of tiles already
    assert plan(0, 10, 10) == 1 and plan(10, 0, 10) == 1 and plan(10, 10, 0) == 1
    for tiles in (1, 7, 100, 640, 3000):
        for nchunks in (1, 40, 512, 16384):
            s = plan(tiles, nchunks, 1184)
            assert 1 <= s <= max(1, nchunks // 32)
            assert s == 1 or tiles * s <= 4 * 1184
