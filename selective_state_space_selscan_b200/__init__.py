"""libselscan: selective-scan (S6) forward for NVIDIA B200 (sm_100a).

This package is a thin ctypes binding over the C ABI in ``include/selscan.h``
(built in-tree as ``libselscan.so`` by ``build.py``).  It only marshals
arguments: every step of the scan runs in the library's CUDA kernels.  There
is no CPU fallback; if the shared library is missing the functions raise.

PyTorch is used for device memory and streams only: tensors are passed by
pointer, shape and strides.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libselscan.so")

SELSCAN_F32 = 0
SELSCAN_BF16 = 1

STATUS = {
    0: "SELSCAN_OK", 1: "SELSCAN_ERR_NULL", 2: "SELSCAN_ERR_SHAPE",
    3: "SELSCAN_ERR_STRIDE", 4: "SELSCAN_ERR_DTYPE", 5: "SELSCAN_ERR_ALIGN",
    6: "SELSCAN_ERR_UNSUPPORTED", 7: "SELSCAN_ERR_CUDA", 8: "SELSCAN_ERR_TIMEOUT",
}
STATUS_CODE = {v: k for k, v in STATUS.items()}

# entry points declared in include/selscan.h
EXPORTS = ("selscan_fwd", "selscan_fwd_h0", "selscan_fwd_scalarA", "selscan_fwd_scalarA_h0",
           "selscan_fwd_noalloc", "selscan_step", "selscan_step_scalarA", "selscan_check",
           "selscan_strerror", "selscan_version", "selscan_launch_count", "selscan_bwd",
           "selscan_release_scratch")


class SelscanError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS.get(status, f"status {status}")
        super().__init__(f"{where}: {self.name} ({_strerror(status)})")


class SelscanTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32),
                ("ndim", ctypes.c_int32), ("shape", ctypes.c_int64 * 4),
                ("stride", ctypes.c_int64 * 4)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libselscan.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m selective_state_space_selscan_b200.build` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(SelscanTensor)
        L.selscan_fwd.argtypes = [P, P, P, ctypes.c_int, P, P, P, P, P, P, P,
                                  ctypes.c_void_p]
        L.selscan_fwd_scalarA.argtypes = [P, P, P, ctypes.c_int, P, P, P, P, P,
                                          ctypes.c_int64, P, P, ctypes.c_void_p]
        L.selscan_check.argtypes = [ctypes.c_void_p]
        L.selscan_strerror.argtypes = [ctypes.c_int]
        L.selscan_strerror.restype = ctypes.c_char_p
        L.selscan_version.argtypes = []
        L.selscan_launch_count.argtypes = []
        L.selscan_launch_count.restype = ctypes.c_ulonglong
        for f in (L.selscan_fwd, L.selscan_fwd_scalarA, L.selscan_check,
                  L.selscan_version):
            f.restype = ctypes.c_int
        L.selscan_fwd_h0.argtypes = [P, P, P, ctypes.c_int, P, P, P, P, P, P, P, P,
                                     ctypes.c_void_p]
        L.selscan_fwd_h0.restype = ctypes.c_int
        L.selscan_fwd_scalarA_h0.argtypes = [P, P, P, ctypes.c_int, P, P, P, P, P,
                                             ctypes.c_int64, P, P, P, ctypes.c_void_p]
        L.selscan_fwd_scalarA_h0.restype = ctypes.c_int
        L.selscan_fwd_noalloc.argtypes = [P, P, P, ctypes.c_int, P, P, P, P, P, P, P,
                                          ctypes.c_void_p]
        L.selscan_fwd_noalloc.restype = ctypes.c_int
        L.selscan_step.argtypes = [P, P, P, P, ctypes.c_int, P, P, P, P, P, P,
                                   ctypes.c_void_p]
        L.selscan_step.restype = ctypes.c_int
        L.selscan_step_scalarA.argtypes = [P, P, P, P, ctypes.c_int, P, P, P, P, P,
                                           ctypes.c_int64, P, ctypes.c_void_p]
        L.selscan_step_scalarA.restype = ctypes.c_int
        L.selscan_bwd.argtypes = [P, P, P, ctypes.c_int] + [P] * 17 + [ctypes.c_void_p]
        L.selscan_bwd_scalarA.argtypes = ([P, P, P, ctypes.c_int] + [P] * 5 +
                                          [ctypes.c_int64] + [P] * 12 + [ctypes.c_void_p])
        L.selscan_bwd_scalarA.restype = ctypes.c_int
        L.selscan_bwd.restype = ctypes.c_int
        L.selscan_release_scratch.argtypes = []
        L.selscan_release_scratch.restype = ctypes.c_int
        L.selscan_debug_withhold_carry.argtypes = [ctypes.c_int]
        L.selscan_debug_withhold_carry.restype = None
        L.selscan_debug_diag_mode.argtypes = [ctypes.c_int]
        L.selscan_debug_diag_mode.restype = None
        L.selscan_debug_bwd_segments.argtypes = [ctypes.c_int]
        L.selscan_debug_bwd_segments.restype = None
        L.selscan_debug_fwd_segments.argtypes = [ctypes.c_int]
        L.selscan_debug_fwd_segments.restype = None
        L.selscan_debug_fwd_plan.argtypes = [ctypes.c_longlong] * 3
        L.selscan_debug_fwd_plan.restype = ctypes.c_longlong
        L.selscan_debug_bwd_plan.argtypes = [ctypes.c_longlong] * 3
        L.selscan_debug_bwd_plan.restype = ctypes.c_longlong
        _lib = L
    return _lib


def _strerror(status: int) -> str:
    try:
        return lib().selscan_strerror(int(status)).decode()
    except Exception:  # pragma: no cover - only when the library is absent
        return STATUS.get(status, "unknown")


def version() -> int:
    return lib().selscan_version()


def launch_count() -> int:
    """Kernels launched by the library in this process so far."""
    return int(lib().selscan_launch_count())


def release_scratch() -> None:
    """Hand back to the driver the scratch memory the library's pools keep
    between calls (synchronise the streams first to release all of it)."""
    st = lib().selscan_release_scratch()
    if st != 0:
        raise SelscanError(st, "selscan_release_scratch")


def describe(t, dtype_code=None) -> SelscanTensor | None:
    """selscan_tensor for a CUDA torch tensor (None stays None -> NULL).
    Host tensors are refused: the C ABI takes device pointers only, and
    there is no CPU implementation to fall back to."""
    if t is None:
        return None
    import torch
    if not t.is_cuda:
        raise ValueError(f"libselscan takes CUDA tensors only (got one on {t.device}); "
                         "there is no CPU implementation")
    d = SelscanTensor()
    d.data = t.data_ptr()
    if dtype_code is None:
        dtype_code = {torch.float32: SELSCAN_F32,
                      torch.bfloat16: SELSCAN_BF16}.get(t.dtype, -1)
    d.dtype = dtype_code
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _ref(d):
    return None if d is None else ctypes.byref(d)


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def selscan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                delta_softplus=True, out=None, last_state=None,
                return_last_state=True, stream=None, h0=None):
    """Diagonal-A selective scan forward through the C ABI.

    u, delta, z: (batch, D, L) bf16 or fp32 CUDA tensors (time stride 1);
    A: (D, N=16) fp32; B, C: (batch, N, L) same dtype as u; D, delta_bias:
    (D,) fp32; h0: optional initial state (batch, D, N) fp32 (selscan_fwd_h0).
    Returns (y, last_state); last_state is None unless requested.
    """
    import torch
    y = out if out is not None else torch.empty_like(u, memory_format=torch.contiguous_format)
    if last_state is None and return_last_state:
        last_state = torch.empty((u.shape[0], u.shape[1], A.shape[1]),
                                 dtype=torch.float32, device=u.device)
    descs = [describe(t) for t in (u, delta, delta_bias, A, B, C, D, z, y, last_state)]
    common = (_ref(descs[0]), _ref(descs[1]), _ref(descs[2]), int(bool(delta_softplus)),
              _ref(descs[3]), _ref(descs[4]), _ref(descs[5]), _ref(descs[6]), _ref(descs[7]))
    if h0 is None:
        rc = lib().selscan_fwd(*common, _ref(descs[8]), _ref(descs[9]), _stream_handle(stream))
        where = "selscan_fwd"
    else:
        hd = describe(h0)
        rc = lib().selscan_fwd_h0(*common, _ref(hd), _ref(descs[8]), _ref(descs[9]),
                                  _stream_handle(stream))
        where = "selscan_fwd_h0"
    if rc != 0:
        raise SelscanError(rc, where)
    return y, last_state


def selscan_fwd_noalloc(u, delta, A, B, C, out, D=None, z=None, delta_bias=None,
                        delta_softplus=True, last_state=None, stream=None):
    """selscan_fwd for callers that cannot allocate device memory during a
    call (fixed-footprint servers or real-time loops that reserve memory at
    start-up, or systems without the stream-ordered allocator that
    selscan_fwd uses for its scratch).  The library keeps the scratch in one
    static device array per GPU, shared by all calls: calls that overlap on
    the GPU race, so serialise them, and make the first call on a device
    before any stream capture (it looks up the array's address).

    ``out`` (the y buffer) and the optional ``last_state`` must be passed;
    nothing is allocated here either.  Returns (out, last_state).
    """
    descs = [describe(t) for t in (u, delta, delta_bias, A, B, C, D, z, out, last_state)]
    rc = lib().selscan_fwd_noalloc(_ref(descs[0]), _ref(descs[1]), _ref(descs[2]),
                                   int(bool(delta_softplus)), _ref(descs[3]),
                                   _ref(descs[4]), _ref(descs[5]), _ref(descs[6]),
                                   _ref(descs[7]), _ref(descs[8]), _ref(descs[9]),
                                   _stream_handle(stream))
    if rc != 0:
        raise SelscanError(rc, "selscan_fwd_noalloc")
    return out, last_state


def selscan_fwd_scalarA(x, dt, A, B, C, headdim, D=None, z=None, dt_bias=None,
                        dt_softplus=False, out=None, last_state=None,
                        return_last_state=True, stream=None, h0=None):
    """Scalar-A (Mamba-2 / SSD) scan forward through the C ABI.

    x, z: (batch, H*P, L) bf16; dt: (batch, H, L) fp32; A, D, dt_bias: (H,)
    fp32; B, C: (batch, G, N, L) bf16.  Returns (y, last_state (batch, H, P, N)).
    """
    import torch
    y = out if out is not None else torch.empty_like(x, memory_format=torch.contiguous_format)
    if last_state is None and return_last_state:
        last_state = torch.empty((x.shape[0], A.shape[0], headdim, B.shape[2]),
                                 dtype=torch.float32, device=x.device)
    descs = [describe(t) for t in (x, dt, dt_bias, A, B, C, D, z, y, last_state)]
    common = (_ref(descs[0]), _ref(descs[1]), _ref(descs[2]), int(bool(dt_softplus)),
              _ref(descs[3]), _ref(descs[4]), _ref(descs[5]), _ref(descs[6]), _ref(descs[7]),
              int(headdim))
    if h0 is None:
        rc = lib().selscan_fwd_scalarA(*common, _ref(descs[8]), _ref(descs[9]),
                                       _stream_handle(stream))
        where = "selscan_fwd_scalarA"
    else:
        hd = describe(h0)
        rc = lib().selscan_fwd_scalarA_h0(*common, _ref(hd), _ref(descs[8]), _ref(descs[9]),
                                          _stream_handle(stream))
        where = "selscan_fwd_scalarA_h0"
    if rc != 0:
        raise SelscanError(rc, where)
    return y, last_state


def selscan_step(state, u, delta, A, B, C, D=None, z=None, delta_bias=None,
                 delta_softplus=True, out=None, stream=None):
    """One decode step of the diagonal-A scan; ``state`` (batch, D, N) fp32
    is updated in place.  u, delta, z: (batch, D) bf16 or fp32 (any strides);
    B, C: (batch, N) or (batch, G, N).  Returns y (batch, D)."""
    import torch
    y = out if out is not None else torch.empty(u.shape, dtype=u.dtype, device=u.device)
    d = [describe(t) for t in (state, u, delta, delta_bias, A, B, C, D, z, y)]
    rc = lib().selscan_step(_ref(d[0]), _ref(d[1]), _ref(d[2]), _ref(d[3]),
                            int(bool(delta_softplus)), _ref(d[4]), _ref(d[5]), _ref(d[6]),
                            _ref(d[7]), _ref(d[8]), _ref(d[9]), _stream_handle(stream))
    if rc != 0:
        raise SelscanError(rc, "selscan_step")
    return y


def selscan_step_scalarA(state, x, dt, A, B, C, headdim, D=None, z=None, dt_bias=None,
                         dt_softplus=False, out=None, stream=None):
    """One decode step of the scalar-A (Mamba-2) scan; ``state`` (batch, H,
    P, N) fp32 is updated in place.  x, z: (batch, H*P); dt: (batch, H)
    fp32; B, C: (batch, N) or (batch, G, N).  Returns y (batch, H*P)."""
    import torch
    y = out if out is not None else torch.empty(x.shape, dtype=x.dtype, device=x.device)
    d = [describe(t) for t in (state, x, dt, dt_bias, A, B, C, D, z, y)]
    rc = lib().selscan_step_scalarA(_ref(d[0]), _ref(d[1]), _ref(d[2]), _ref(d[3]),
                                    int(bool(dt_softplus)), _ref(d[4]), _ref(d[5]),
                                    _ref(d[6]), _ref(d[7]), _ref(d[8]), int(headdim),
                                    _ref(d[9]), _stream_handle(stream))
    if rc != 0:
        raise SelscanError(rc, "selscan_step_scalarA")
    return y


def selscan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None,
                delta_softplus=True, h0=None, dlast=None, need_dh0=None, stream=None):
    """Gradients of selscan_fwd (diagonal A) for sum(dy * y) + sum(dlast *
    last_state).  Returns a dict: du, ddelta (like u), dz (like u, or None),
    dA (D, N), dB, dC (batch, N, L) fp32, dD, ddelta_bias (D) fp32 or None,
    dh0 (batch, D, N) fp32 or None (computed when h0 is given or need_dh0)."""
    import torch
    dev = u.device
    f32 = dict(dtype=torch.float32, device=dev)
    batch, dim, L = u.shape
    N = A.shape[1]
    out = {
        "du": torch.empty(u.shape, dtype=u.dtype, device=dev),
        "ddelta": torch.empty(u.shape, dtype=u.dtype, device=dev),
        "dz": torch.empty(u.shape, dtype=u.dtype, device=dev) if z is not None else None,
        "dA": torch.empty((dim, N), **f32),
        "dB": torch.empty((batch, N, L), **f32),
        "dC": torch.empty((batch, N, L), **f32),
        "dD": torch.empty((dim,), **f32) if D is not None else None,
        "ddelta_bias": torch.empty((dim,), **f32) if delta_bias is not None else None,
        "dh0": torch.empty((batch, dim, N), **f32)
        if (h0 is not None or need_dh0) else None,
    }
    ins = [describe(t) for t in (u, delta, delta_bias)]
    rest = [describe(t) for t in (A, B, C, D, z, h0, dy, dlast)]
    outs = [describe(out[k]) for k in ("du", "ddelta", "dA", "dB", "dC", "dD", "dz",
                                       "ddelta_bias", "dh0")]
    rc = lib().selscan_bwd(_ref(ins[0]), _ref(ins[1]), _ref(ins[2]), int(bool(delta_softplus)),
                           *[_ref(x) for x in rest], *[_ref(x) for x in outs],
                           _stream_handle(stream))
    if rc != 0:
        raise SelscanError(rc, "selscan_bwd")
    return out


def selscan_bwd_scalarA(x, dt, A, B, C, headdim, dy, D=None, z=None, dt_bias=None,
                        dt_softplus=False, h0=None, dlast=None, need_dh0=None, stream=None):
    """Gradients of selscan_fwd_scalarA for sum(dy * y) + sum(dlast *
    last_state).  Returns a dict: dx (like x), dz (like x, or None), ddt
    (batch, H, L) fp32, dA (H,), dB, dC (batch, G, N, L) fp32, dD, ddt_bias
    (H,) fp32 or None, dh0 (batch, H, P, N) fp32 or None (computed when h0 is
    given or need_dh0).  B / C may be (batch, N, L) (one group)."""
    import torch
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    batch, dim, L = x.shape
    H = A.shape[0]
    if B.dim() == 3:
        B = B.unsqueeze(1)
        C = C.unsqueeze(1)
    G, N = B.shape[1], B.shape[2]
    out = {
        "dx": torch.empty(x.shape, dtype=x.dtype, device=dev),
        "dz": torch.empty(x.shape, dtype=x.dtype, device=dev) if z is not None else None,
        "ddt": torch.empty((batch, H, L), **f32),
        "dA": torch.empty((H,), **f32),
        "dB": torch.empty((batch, G, N, L), **f32),
        "dC": torch.empty((batch, G, N, L), **f32),
        "dD": torch.empty((H,), **f32) if D is not None else None,
        "ddt_bias": torch.empty((H,), **f32) if dt_bias is not None else None,
        "dh0": torch.empty((batch, H, int(headdim), N), **f32)
        if (h0 is not None or need_dh0) else None,
    }
    ins = [describe(t) for t in (x, dt, dt_bias)]
    mid = [describe(t) for t in (A, B, C, D, z)]
    tail = [describe(t) for t in (h0, dy, dlast)]
    outs = [describe(out[k]) for k in ("dx", "ddt", "dA", "dB", "dC", "dD", "dz",
                                       "ddt_bias", "dh0")]
    rc = lib().selscan_bwd_scalarA(_ref(ins[0]), _ref(ins[1]), _ref(ins[2]),
                                   int(bool(dt_softplus)), *[_ref(t) for t in mid],
                                   ctypes.c_int64(int(headdim)), *[_ref(t) for t in tail],
                                   *[_ref(t) for t in outs], _stream_handle(stream))
    if rc != 0:
        raise SelscanError(rc, "selscan_bwd_scalarA")
    return out


def check(stream=None) -> None:
    """Synchronise ``stream`` and raise if a device-side wait timed out."""
    rc = lib().selscan_check(_stream_handle(stream))
    if rc != 0:
        raise SelscanError(rc, "selscan_check")


def debug_diag_mode(mode: int) -> None:
    """Test hook: 0 = chained carries, 1 = two-pass form, -1 = automatic."""
    lib().selscan_debug_diag_mode(int(mode))


def debug_bwd_segments(segs: int) -> None:
    """Test hook: time segments per channel tile in selscan_bwd (0: automatic)."""
    lib().selscan_debug_bwd_segments(int(segs))


def debug_fwd_segments(segs: int) -> None:
    """Test hook: time segments per channel tile in selscan_fwd (0: automatic)."""
    lib().selscan_debug_fwd_segments(int(segs))


def debug_fwd_plan(tiles: int, chunks: int, ctas: int) -> int:
    """Test hook: selscan_fwd's automatic segment count for ``tiles`` tiles,
    ``chunks`` 64-token chunks and ``ctas`` CTAs (negative: the two-pass
    form).  Host arithmetic only."""
    return int(lib().selscan_debug_fwd_plan(int(tiles), int(chunks), int(ctas)))


def debug_bwd_plan(tiles: int, nchunks: int, slots: int) -> int:
    """Test hook: the backward's segment count for ``tiles`` channel tiles,
    ``nchunks`` checkpoint chunks and ``slots`` resident warps (host
    arithmetic only, no GPU needed)."""
    return int(lib().selscan_debug_bwd_plan(int(tiles), int(nchunks), int(slots)))


def debug_withhold_carry(unit: int) -> None:
    """Test hook: withhold the carry flag of work unit ``unit`` (-1: off)."""
    lib().selscan_debug_withhold_carry(int(unit))
