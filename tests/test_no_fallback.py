"""The product path has no CPU fallback: the binding raises when
libselscan.so is missing, refuses host tensors before any library call
(the C ABI takes device pointers only), and never imports the oracle."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _python(code):
    r = subprocess.run([sys.executable, "-c", f"import sys; sys.path.insert(0, {ROOT!r})\n" + code],
                       capture_output=True, text=True, timeout=300)
    return r.stdout + r.stderr


def test_missing_library_raises():
    out = _python(
        "import selective_state_space_selscan_b200 as ss\n"
        "ss.LIB_PATH = '/nonexistent/libselscan.so'\n"
        "ss._lib = None\n"
        "try:\n"
        "    ss.lib()\n"
        "except RuntimeError as e:\n"
        "    print('RAISED:', e)\n")
    assert "RAISED:" in out and "no fallback" in out, out


def test_host_tensors_are_refused():
    import torch
    import selective_state_space_selscan_b200 as ss
    u = torch.zeros(1, 32, 16, dtype=torch.bfloat16)
    A = -torch.ones(32, 16)
    bc = torch.zeros(1, 16, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        ss.selscan_fwd(u, u, A, bc, bc)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        ss.selscan_bwd(u, u, A, bc, bc, u)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        ss.selscan_step(torch.zeros(1, 32, 16), u[..., 0], u[..., 0], A, bc[..., 0], bc[..., 0])


def test_product_package_does_not_import_the_oracle():
    out = _python(
        "import selective_state_space_selscan_b200 as ss\n"
        "ss.lib()\n"
        "print('oracle loaded:', 'oracle' in sys.modules)\n")
    assert "oracle loaded: False" in out, out
