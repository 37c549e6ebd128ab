"""GPU parity of the diagonal-A scan (selscan_fwd, through the C ABI) against
the fp64 oracle on the same seeded, dtype-rounded inputs.

Tolerances (relative L2 over the compared tensor, y and last_state checked
separately): 1e-5 for fp32 inputs, 5e-3 for bf16 inputs with fp32 state.
"""
import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 5e-3}


def _torch():
    import torch
    return torch


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def dev(a, dtype):
    torch = _torch()
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t.float()


def dev32(a):
    torch = _torch()
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).float().cuda()


def run_gpu(inp, **kw):
    import selective_state_space_selscan_b200 as ss
    dt = inp["dtype"]
    y, hs = ss.selscan_fwd(dev(inp["u"], dt), dev(inp["delta"], dt), dev32(inp["A"]),
                           dev(inp["B"], dt), dev(inp["C"], dt), D=dev32(inp["D"]),
                           z=dev(inp["z"], dt), delta_bias=dev32(inp["delta_bias"]),
                           delta_softplus=inp["softplus"], **kw)
    ss.check()
    return y.float().cpu().numpy(), hs.cpu().numpy()


def run_oracle(inp, channels=None):
    return oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                          z=inp["z"], delta_bias=inp["delta_bias"],
                          delta_softplus=inp["softplus"], channels=channels)


def assert_parity(inp, y, hs, y_ref, hs_ref, what=""):
    tol = TOL[inp["dtype"]]
    ey, eh = rel_l2(y, y_ref), rel_l2(hs, hs_ref)
    assert np.isfinite(y).all() and np.isfinite(hs).all(), what
    assert ey <= tol and eh <= tol, f"{what}: rel L2 y={ey:.3e} state={eh:.3e} (tol {tol})"
    return ey, eh


def test_config0_tiny_fp32_full():
    """Tiny fp32 config (B1 D64 N16 L256, seed 0), every output checked."""
    inp = synthetic.make_config(0)
    y, hs = run_gpu(inp)
    y_ref, hs_ref = run_oracle(inp)
    assert_parity(inp, y, hs, y_ref, hs_ref, "config 0")


@pytest.mark.parametrize("gate", [True, False])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ragged_tiles_and_tail(gate, dtype):
    """dim not a multiple of the 64-channel tile, L not a multiple of the
    chunk, several segments and batches (bf16: the two-pass form the library
    picks for so few tiles; fp32: the chained form forced, which keeps its
    spread of segments, where the automatic choice would take one)."""
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(3, 96 + 8, 16, 1000, dtype=dtype, seed=21, gate=gate)
    if dtype == "f32":
        ss.debug_diag_mode(0)
    try:
        y, hs = run_gpu(inp)
    finally:
        ss.debug_diag_mode(-1)
    y_ref, hs_ref = run_oracle(inp)
    assert_parity(inp, y, hs, y_ref, hs_ref, f"ragged gate={gate} {dtype}")


def test_general_A_and_mixed_structure():
    """A without the S4D-real structure (general exp path) on some channels
    and with it on others, inside the same warp and tile."""
    inp = synthetic.make_diag(2, 128, 16, 512, dtype="bf16", seed=22)
    rng = np.random.default_rng(5)
    A = inp["A"].copy()
    A[::3] = -rng.uniform(0.5, 12.0, (A[::3].shape)).astype(np.float32)
    A[64:] = -np.exp(rng.uniform(-1, 2.5, (64, 16))).astype(np.float32)
    inp["A"] = A
    y, hs = run_gpu(inp)
    y_ref, hs_ref = run_oracle(inp)
    assert_parity(inp, y, hs, y_ref, hs_ref, "general A")


def test_scaled_s4d_structure_per_channel():
    """A[d,n] = (n+1) * a_d with a different a_d per channel (structured path)."""
    inp = synthetic.make_diag(1, 64, 16, 768, dtype="bf16", seed=23, gate=False)
    a = np.random.default_rng(1).uniform(0.2, 3.0, 64).astype(np.float32)
    inp["A"] = (-(np.arange(1, 17, dtype=np.float32))[None, :] * a[:, None]).astype(np.float32)
    y, hs = run_gpu(inp)
    y_ref, hs_ref = run_oracle(inp)
    assert_parity(inp, y, hs, y_ref, hs_ref, "scaled S4D")


def test_no_bias_no_softplus_no_D():
    inp = synthetic.make_diag(2, 64, 16, 256, dtype="bf16", seed=24, D=False, bias=False)
    inp["delta"] = synthetic.round_bf16(np.abs(inp["delta"]) * 0.1)
    inp["softplus"] = False
    y, hs = run_gpu(inp)
    y_ref, hs_ref = run_oracle(inp)
    assert_parity(inp, y, hs, y_ref, hs_ref, "plain delta")


def test_strided_views_and_rank4_BC():
    """u and z as the two halves of one (batch, 2D, L) buffer, delta with a
    padded row stride, B/C given as (batch, 1, N, L)."""
    torch = _torch()
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(2, 64, 16, 320, dtype="bf16", seed=25)
    xz = torch.cat([dev(inp["u"], "bf16"), dev(inp["z"], "bf16")], dim=1)
    u, z = xz[:, :64], xz[:, 64:]
    dpad = torch.zeros(2, 64, 336, dtype=torch.bfloat16, device="cuda")
    dpad[:, :, :320] = dev(inp["delta"], "bf16")
    delta = dpad[:, :, :320]
    assert not u.is_contiguous() and not delta.is_contiguous()
    B4 = dev(inp["B"], "bf16").unsqueeze(1)
    C4 = dev(inp["C"], "bf16").unsqueeze(1)
    y, hs = ss.selscan_fwd(u, delta, dev32(inp["A"]), B4, C4, D=dev32(inp["D"]), z=z,
                           delta_bias=dev32(inp["delta_bias"]))
    ss.check()
    y_ref, hs_ref = run_oracle(inp)
    assert_parity(inp, y.float().cpu().numpy(), hs.cpu().numpy(), y_ref, hs_ref, "strided")


def test_output_into_strided_buffer_and_no_state():
    torch = _torch()
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(1, 64, 16, 256, dtype="bf16", seed=26)
    ybuf = torch.full((1, 64, 264), 7.0, dtype=torch.bfloat16, device="cuda")
    out = ybuf[:, :, :256]
    dt = "bf16"
    y, hs = ss.selscan_fwd(dev(inp["u"], dt), dev(inp["delta"], dt), dev32(inp["A"]),
                           dev(inp["B"], dt), dev(inp["C"], dt), D=dev32(inp["D"]),
                           z=dev(inp["z"], dt), delta_bias=dev32(inp["delta_bias"]),
                           out=out, return_last_state=False)
    ss.check()
    assert hs is None
    assert torch.all(ybuf[:, :, 256:] == 7.0), "wrote past the view"
    y_ref, _ = run_oracle(inp)
    assert rel_l2(y.float().cpu().numpy(), y_ref) <= TOL["bf16"]


def test_empty_inputs():
    torch = _torch()
    import selective_state_space_selscan_b200 as ss
    A = -torch.arange(1, 17, dtype=torch.float32, device="cuda").repeat(64, 1)
    e = torch.empty(2, 64, 0, dtype=torch.bfloat16, device="cuda")
    Bc = torch.empty(2, 16, 0, dtype=torch.bfloat16, device="cuda")
    st = torch.full((2, 64, 16), 3.0, device="cuda")
    y, hs = ss.selscan_fwd(e, e, A, Bc, Bc, last_state=st)
    ss.check()
    assert y.shape == (2, 64, 0) and torch.all(hs == 0)
    e0 = torch.empty(0, 64, 128, dtype=torch.bfloat16, device="cuda")
    B0 = torch.empty(0, 16, 128, dtype=torch.bfloat16, device="cuda")
    y, hs = ss.selscan_fwd(e0, e0, A, B0, B0)
    ss.check()
    assert y.shape == (0, 64, 128)


def test_repeatable_bitwise():
    inp = synthetic.make_diag(2, 192, 16, 2048, dtype="bf16", seed=27)
    y1, h1 = run_gpu(inp)
    y2, h2 = run_gpu(inp)
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)


def _per_channel_worst(got, ref):
    got = np.asarray(got, np.float64).reshape(-1, got.shape[-1])
    ref = np.asarray(ref, np.float64).reshape(-1, ref.shape[-1])
    den = np.linalg.norm(ref, axis=1)
    live = den > 0
    return float(np.max(np.linalg.norm(got - ref, axis=1)[live] / den[live]))


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_full_size_config_whole(cfg):
    """Full-size configs in the launch configuration the benchmark times,
    compared with the oracle on every channel, token and batch row (the
    oracle runs over channel ranges on several host threads), whole tensor
    and channel by channel."""
    import oracle_par
    inp = synthetic.make_config(cfg)
    y, hs = run_gpu(inp)
    y_ref, hs_ref = oracle_par.selscan(inp)
    assert_parity(inp, y, hs, y_ref, hs_ref, f"config {cfg}")
    tol = TOL[inp["dtype"]]
    cy, ch = _per_channel_worst(y, y_ref), _per_channel_worst(hs, hs_ref)
    assert cy <= tol and ch <= tol, f"config {cfg}: worst channel y={cy:.3e} state={ch:.3e}"


@pytest.mark.parametrize("mode", [0, 1])
def test_chained_and_two_pass_forms(mode):
    """Two channel tiles, 32 segments: the carries chained from segment to
    segment (mode 0) and the two-pass form (mode 1: segment aggregates, then
    the output pass) both reproduce the oracle, with an initial state."""
    import selective_state_space_selscan_b200 as ss
    torch = _torch()
    inp = synthetic.make_diag(1, 256, 16, 8192, dtype="bf16", seed=31)
    h0 = np.random.default_rng(4).standard_normal((1, 256, 16)).astype(np.float32)
    ss.debug_diag_mode(mode)
    try:
        y, hs = ss.selscan_fwd(dev(inp["u"], "bf16"), dev(inp["delta"], "bf16"), dev32(inp["A"]),
                               dev(inp["B"], "bf16"), dev(inp["C"], "bf16"), D=dev32(inp["D"]),
                               z=dev(inp["z"], "bf16"), delta_bias=dev32(inp["delta_bias"]),
                               h0=torch.from_numpy(h0).cuda())
        ss.check()
    finally:
        ss.debug_diag_mode(-1)
    y_ref, hs_ref = oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                   D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"], h0=h0)
    assert_parity(inp, y.float().cpu().numpy(), hs.cpu().numpy(), y_ref, hs_ref, f"mode {mode}")


def test_withheld_carry_times_out():
    """Failure detection without a GPU fault: one work unit withholds its
    carry flag, its successor gives up after the (short) wait limit, and
    selscan_check reports SELSCAN_ERR_TIMEOUT; the next call runs clean.
    Runs in a child process so that the short limit applies only there."""
    import os
    import subprocess
    import sys
    code = r'''
import numpy as np, torch, sys
sys.path.insert(0, sys.argv[1])
import selective_state_space_selscan_b200 as ss, synthetic
inp = synthetic.make_diag(1, 256, 16, 4096, dtype="bf16", seed=32)
cv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch.bfloat16)
f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().float()
args = (cv(inp["u"]), cv(inp["delta"]), f(inp["A"]), cv(inp["B"]), cv(inp["C"]))
kw = dict(D=f(inp["D"]), z=cv(inp["z"]), delta_bias=f(inp["delta_bias"]))
ss.debug_diag_mode(0)
ss.debug_withhold_carry(3)      # unit 3 = segment 1 of tile 1 (two tiles)
ss.selscan_fwd(*args, **kw)
try:
    ss.check()
    print("NO_TIMEOUT")
except ss.SelscanError as e:
    print("STATUS", e.name)
ss.debug_withhold_carry(-1)
y, hs = ss.selscan_fwd(*args, **kw)
ss.check()
print("CLEAN", bool(torch.isfinite(y.float()).all()))
'''
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SELSCAN_WAIT_TIMEOUT_MS="300")
    r = subprocess.run([sys.executable, "-c", code, root], capture_output=True, text=True,
                       env=env, timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "STATUS SELSCAN_ERR_TIMEOUT" in r.stdout, r.stdout
    assert "CLEAN True" in r.stdout, r.stdout


@pytest.mark.parametrize("gate", [False, True])
def test_two_pass_without_softplus(gate):
    """The two-pass form's instances without the softplus (raw positive step
    sizes, no bias), with and without the gate."""
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(1, 256, 16, 2048, dtype="bf16", seed=33, gate=gate, bias=False)
    inp["delta"] = synthetic.round_bf16(np.abs(inp["delta"]) * 0.05)
    inp["softplus"] = False
    ss.debug_diag_mode(1)
    try:
        y, hs = run_gpu(inp)
    finally:
        ss.debug_diag_mode(-1)
    y_ref, hs_ref = run_oracle(inp)
    assert_parity(inp, y, hs, y_ref, hs_ref, f"two-pass, no softplus, gate={gate}")
