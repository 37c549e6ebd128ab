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
