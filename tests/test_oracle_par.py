"""The threaded oracle harness used by the whole-tensor GPU parity tests
returns exactly what one single-threaded oracle call returns (CPU)."""
import numpy as np

import oracle
import oracle_par
import synthetic


def test_threaded_diag_equals_single_call():
    inp = synthetic.make_diag(2, 37, 16, 300, dtype="bf16", seed=61)
    h0 = np.random.default_rng(2).standard_normal((2, 37, 16)).astype(np.float32)
    y1, h1 = oracle.selscan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                            z=inp["z"], delta_bias=inp["delta_bias"], h0=h0)
    y2, h2 = oracle_par.selscan(inp, h0=h0, parts=5)
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)


def test_threaded_scalarA_equals_single_call():
    inp = synthetic.make_scalarA(2, 6, 8, 16, 200, seed=62)
    y1, h1 = oracle.selscan_scalarA(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                    inp["headdim"], D=inp["D"])
    y2, h2 = oracle_par.selscan_scalarA(inp, parts=4)
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)


def test_threaded_diag_bwd_equals_single_call():
    """Per-channel gradients are identical; dB and dC, sums over channels,
    agree up to the order of the fp64 additions."""
    inp = synthetic.make_diag(2, 37, 16, 300, dtype="bf16", seed=63)
    dy = np.random.default_rng(3).standard_normal(inp["u"].shape).astype(np.float32)
    g1 = oracle.selscan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                            D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"])
    g2 = oracle_par.selscan_bwd(inp, dy, parts=5)
    assert g1.keys() == g2.keys()
    for k, v in g1.items():
        if v is None:
            assert g2[k] is None, k
        elif k in ("dB", "dC"):
            assert np.allclose(g2[k], v, rtol=1e-12, atol=1e-12 * np.abs(v).max()), k
        else:
            assert np.array_equal(g2[k], v), k


def test_threaded_scalarA_bwd_equals_single_call():
    inp = synthetic.make_scalarA(2, 6, 8, 16, 96, seed=64, gate=True)
    dy = np.random.default_rng(4).standard_normal(inp["x"].shape).astype(np.float32)
    g1 = oracle.selscan_scalarA_bwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                    inp["headdim"], dy, D=inp["D"], z=inp["z"])
    g2 = oracle_par.selscan_scalarA_bwd(inp, dy, parts=4)
    assert g1.keys() == g2.keys()
    for k, v in g1.items():
        if v is None:
            assert g2[k] is None, k
        elif k in ("dB", "dC"):
            assert np.allclose(g2[k], v, rtol=1e-12, atol=1e-12 * np.abs(v).max()), k
        else:
            assert np.array_equal(g2[k], v), k
