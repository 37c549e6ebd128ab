"""GPU parity of the backward pass (selscan_bwd, through the C ABI) with the
fp64 oracle's gradients (oracle.selscan_bwd, itself pinned by finite
differences) on the same seeded inputs.

Tolerances, relative L2 per gradient: fp32 inputs 1e-4 (fp32 arithmetic
through a reverse recurrence and atomic sums); bf16 inputs: 5e-3 for du,
ddelta, dz (stored in bf16) and 2e-3 for the fp32 gradients (computed in
fp32 with the special-function unit's exp/log)."""
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


def run(inp, dy, dtype, h0=None, dlast=None, softplus=True):
    import selective_state_space_selscan_b200 as ss
    g = ss.selscan_bwd(_dev(inp["u"], dtype), _dev(inp["delta"], dtype), _f32(inp["A"]),
                       _dev(inp["B"], dtype), _dev(inp["C"], dtype), _dev(dy, dtype),
                       D=_f32(inp["D"]), z=_dev(inp["z"], dtype),
                       delta_bias=_f32(inp["delta_bias"]), delta_softplus=softplus,
                       h0=_f32(h0), dlast=_f32(dlast))
    ss.check()
    return {k: (None if v is None else v.float().cpu().numpy()) for k, v in g.items()}


def ref(inp, dy, h0=None, dlast=None, softplus=True):
    return oracle.selscan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                              D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                              delta_softplus=softplus, h0=h0, dlast=dlast)


def compare(got, want, dtype, skip=()):
    tol_lo = 5e-3 if dtype == "bf16" else 1e-4
    tol_32 = 2e-3 if dtype == "bf16" else 1e-4
    for k, w in want.items():
        if k in skip:
            continue
        if w is None:
            assert got[k] is None, k
            continue
        assert np.isfinite(got[k]).all(), k
        tol = tol_lo if k in ("du", "ddelta", "dz") else tol_32
        e = rel(got[k].reshape(w.shape), w)
        assert e <= tol, f"{k}: rel L2 {e:.3e} > {tol}"


def _dy(inp, seed):
    d = np.random.default_rng(seed).standard_normal(inp["u"].shape).astype(np.float32)
    return synthetic.round_bf16(d) if inp["dtype"] == "bf16" else d


def test_fp32_all_options_ragged():
    """fp32; 80 channels (a warp with dead lanes), L = 300 (ragged chunk);
    gate, D, bias, softplus, h0 and a final-state gradient."""
    inp = synthetic.make_diag(2, 80, 16, 300, dtype="f32", seed=81)
    rng = np.random.default_rng(82)
    h0 = rng.standard_normal((2, 80, 16)).astype(np.float32)
    dlast = rng.standard_normal((2, 80, 16)).astype(np.float32)
    dy = _dy(inp, 83)
    compare(run(inp, dy, "f32", h0, dlast), ref(inp, dy, h0, dlast), "f32")


@pytest.mark.parametrize("gate,softplus", [(True, True), (False, False)])
def test_bf16(gate, softplus):
    inp = synthetic.make_diag(2, 192, 16, 1024, dtype="bf16", seed=84, gate=gate)
    if not softplus:
        # raw step sizes used as given: small and positive, bf16-exact, no bias
        inp["delta"] = synthetic.round_bf16(np.abs(inp["delta"]) * 0.05)
        inp["delta_bias"] = None
    dy = _dy(inp, 85)
    # an initial state and a final-state gradient exercise the segment folds
    rng = np.random.default_rng(86)
    h0 = rng.standard_normal((2, 192, 16)).astype(np.float32) if gate else None
    dlast = rng.standard_normal((2, 192, 16)).astype(np.float32) if gate else None
    compare(run(inp, dy, "bf16", h0, dlast, softplus=softplus),
            ref(inp, dy, h0, dlast, softplus=softplus), "bf16")


def test_general_A_no_bias():
    """A without the S4D-real structure (one exponential per state)."""
    inp = synthetic.make_diag(1, 64, 16, 256, dtype="f32", seed=86, bias=False)
    inp["A"] = -np.exp(np.random.default_rng(87).uniform(-2, 1.5, (64, 16))).astype(np.float32)
    dy = _dy(inp, 88)
    compare(run(inp, dy, "f32"), ref(inp, dy), "f32")


def test_strided_views():
    """u and z as halves of one (batch, 2D, L) projection."""
    import torch
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(2, 64, 16, 128, dtype="bf16", seed=89)
    dy = _dy(inp, 90)
    xz = torch.cat([_dev(inp["u"], "bf16"), _dev(inp["z"], "bf16")], dim=1)
    g = ss.selscan_bwd(xz[:, :64], _dev(inp["delta"], "bf16"), _f32(inp["A"]),
                       _dev(inp["B"], "bf16"), _dev(inp["C"], "bf16"), _dev(dy, "bf16"),
                       D=_f32(inp["D"]), z=xz[:, 64:], delta_bias=_f32(inp["delta_bias"]))
    ss.check()
    got = {k: (None if v is None else v.float().cpu().numpy()) for k, v in g.items()}
    compare(got, ref(inp, dy), "bf16")


def test_larger_sampled_channels():
    """B4 D384 L4096 bf16: per-channel gradients on sampled channels (dB
    and dC sum over every channel and are checked on the small cases)."""
    inp = synthetic.make_diag(4, 384, 16, 4096, dtype="bf16", seed=91)
    dy = _dy(inp, 92)
    got = run(inp, dy, "bf16")
    for (a, b) in [(0, 8), (190, 198), (376, 384)]:
        sl = lambda x: None if x is None else x[:, a:b]
        sub = dict(inp, u=sl(inp["u"]), delta=sl(inp["delta"]), z=sl(inp["z"]),
                   A=inp["A"][a:b], D=inp["D"][a:b], delta_bias=inp["delta_bias"][a:b])
        want = ref(sub, dy[:, a:b])
        part = {"du": got["du"][:, a:b], "ddelta": got["ddelta"][:, a:b],
                "dz": got["dz"][:, a:b], "dA": got["dA"][a:b], "dD": got["dD"][a:b],
                "ddelta_bias": got["ddelta_bias"][a:b], "dh0": None}
        compare(part, {k: want[k] for k in part}, "bf16")


def test_full_size_config2_sampled():
    """The benchmark's workload, B4 D5120 L4096 bf16 with gate, D and bias,
    in the launch configuration it times.  Per-channel gradients are
    checked on channels sampled at the start, middle and end of d_inner.
    dB and dC sum over all channels, so a second call gets dy only on the
    sampled channels: every other channel then has a zero gradient state
    and adds exactly zero, and the oracle's sums over the sampled channels
    are the whole answer."""
    inp = synthetic.make_config(2)
    dy = _dy(inp, 93)
    dim = inp["u"].shape[1]
    ranges = [(0, 4), (dim // 2 - 2, dim // 2 + 2), (dim - 4, dim)]
    chans = np.concatenate([np.arange(a, b) for a, b in ranges])
    sub = dict(inp, u=inp["u"][:, chans], delta=inp["delta"][:, chans], z=inp["z"][:, chans],
               A=inp["A"][chans], D=inp["D"][chans], delta_bias=inp["delta_bias"][chans])
    want = ref(sub, np.ascontiguousarray(dy[:, chans]))
    got = run(inp, dy, "bf16")
    part = {"du": got["du"][:, chans], "ddelta": got["ddelta"][:, chans],
            "dz": got["dz"][:, chans], "dA": got["dA"][chans], "dD": got["dD"][chans],
            "ddelta_bias": got["ddelta_bias"][chans], "dh0": None}
    compare(part, {k: want[k] for k in part}, "bf16")
    dy_masked = np.zeros_like(dy)
    dy_masked[:, chans] = dy[:, chans]
    got = run(inp, dy_masked, "bf16")
    compare({"dB": got["dB"], "dC": got["dC"]}, {"dB": want["dB"], "dC": want["dC"]}, "bf16")
    others = np.setdiff1d(np.arange(dim), chans)[::97]
    assert not got["du"][:, others].any() and not got["dA"][others].any()


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_full_size_config_whole(cfg):
    """Configs 1-3 (B8 D1536 L2048, the benchmark's B4 D5120 L4096, B1 D2048
    L131072) over the whole tensor, in the launch configurations the library
    picks for them: every gradient of every channel and token against the
    oracle, which runs on channel ranges side by side (oracle_par.selscan_bwd;
    dB and dC are the sums of the ranges' parts)."""
    import oracle_par
    inp = synthetic.make_config(cfg)
    dy = _dy(inp, 94 + cfg)
    got = run(inp, dy, "bf16")
    want = oracle_par.selscan_bwd(inp, dy)
    compare(got, want, "bf16")


@pytest.mark.parametrize("segs", [1, 3, 16])
def test_forced_segment_counts(segs):
    """The same gradients whatever the number of time segments per tile:
    the segment folds (end states and start gradients of the earlier and
    later segments) against the oracle, with h0 and a final-state gradient;
    187 chunks, so the last segment is shorter than the others."""
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(2, 64, 16, 1496, dtype="bf16", seed=94)
    rng = np.random.default_rng(95)
    h0 = rng.standard_normal((2, 64, 16)).astype(np.float32)
    dlast = rng.standard_normal((2, 64, 16)).astype(np.float32)
    dy = _dy(inp, 96)
    ss.debug_bwd_segments(segs)
    try:
        got = run(inp, dy, "bf16", h0, dlast)
    finally:
        ss.debug_bwd_segments(0)
    compare(got, ref(inp, dy, h0, dlast), "bf16")


def test_empty_sequence():
    import torch
    import selective_state_space_selscan_b200 as ss
    u = torch.empty(2, 32, 0, dtype=torch.bfloat16, device="cuda")
    BC = torch.empty(2, 16, 0, dtype=torch.bfloat16, device="cuda")
    A = -torch.arange(1, 17, dtype=torch.float32, device="cuda").repeat(32, 1)
    dlast = torch.randn(2, 32, 16, device="cuda")
    g = ss.selscan_bwd(u, u, A, BC, BC, u, dlast=dlast, need_dh0=True)
    ss.check()
    assert torch.equal(g["dh0"], dlast) and torch.all(g["dA"] == 0)


def test_results_unchanged_after_release_scratch():
    """The scratch pool handed back between two calls: the second call maps
    fresh memory and still matches the oracle."""
    import torch
    import selective_state_space_selscan_b200 as ss
    inp = synthetic.make_diag(1, 96, 16, 512, dtype="f32", seed=87)
    dy = _dy(inp, 88)
    want = ref(inp, dy)
    compare(run(inp, dy, "f32"), want, "f32")
    torch.cuda.synchronize()
    ss.release_scratch()
    compare(run(inp, dy, "f32"), want, "f32")


def test_empty_batch_zeroes_parameter_gradients():
    """batch = 0 with channels present: dA, dD and d bias are sums over no
    batch row, so the call must write zeros into them, whatever the caller's
    buffers held (here NaN), through the C ABI."""
    import torch
    import selective_state_space_selscan_b200 as ss
    dev = "cuda"
    dim, N, L = 32, 16, 64
    u = torch.empty(0, dim, L, dtype=torch.bfloat16, device=dev)
    BC = torch.empty(0, N, L, dtype=torch.bfloat16, device=dev)
    A = -torch.arange(1, N + 1, dtype=torch.float32, device=dev).repeat(dim, 1)
    Dv = torch.ones(dim, device=dev)
    bias = torch.zeros(dim, device=dev)
    nan = lambda *s: torch.full(s, float("nan"), device=dev)
    dA, dD, dbias = nan(dim, N), nan(dim), nan(dim)
    du = torch.empty_like(u)
    dd = torch.empty_like(u)
    dB = torch.empty(0, N, L, device=dev)
    dC = torch.empty(0, N, L, device=dev)
    r = lambda t: ss._ref(ss.describe(t))
    rc = ss.lib().selscan_bwd(r(u), r(u), r(bias), 1, r(A), r(BC), r(BC), r(Dv), None, None,
                              r(u), None, r(du), r(dd), r(dA), r(dB), r(dC), r(dD), None,
                              r(dbias), None, ss._stream_handle(None))
    assert rc == 0
    ss.check()
    assert torch.all(dA == 0) and torch.all(dD == 0) and torch.all(dbias == 0)
