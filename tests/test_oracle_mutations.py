"""Every pin suite of the oracle must catch a plausible mistake in it.

Each case below plants one mistake in a temporary copy of the oracle's C
source: a wrong index, a dropped term, a swapped operand or a wrong sign.
The copy compiles into its own build folder, and the committed oracle is not
touched.  The case then runs the pin suite that should catch the mistake,
and that suite must fail.  Unmutated control copies must pass, so a failure
always means a caught mistake and never a broken copy.  All cases run on the
CPU, in parallel subprocesses.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "selscan_oracle.c")
FWD = "tests/test_oracle_pins.py"
BWD = "tests/test_oracle_bwd_pins.py"

# name: (pin suite, exact text in the oracle, the mistake that replaces it)
MUTATIONS = {
    "B index t-1": (
        FWD, "const double bbar_x = dt * Bg[n * L + t] * x;",
        "const double bbar_x = dt * Bg[n * L + (t > 0 ? t - 1 : 0)] * x;"),
    "bias added after the softplus": (
        FWD,
        "double dt = delta[row + t] + (delta_bias ? delta_bias[d] : 0.0);\n"
        "                if (softplus_flag)\n"
        "                    dt = oracle_softplus(dt);",
        "double dt = delta[row + t];\n"
        "                if (softplus_flag)\n"
        "                    dt = oracle_softplus(dt);\n"
        "                dt += (delta_bias ? delta_bias[d] : 0.0);"),
    "D skip dropped": (
        FWD, "double out = acc + (D ? D[d] * x : 0.0);\n                if (z)",
        "double out = acc;\n                if (z)"),
    "gate applied before the D skip": (
        FWD,
        "double out = acc + (D ? D[d] * x : 0.0);\n"
        "                if (z)\n"
        "                    out *= oracle_silu(z[row + t]);",
        "double out = acc;\n"
        "                if (z)\n"
        "                    out *= oracle_silu(z[row + t]);\n"
        "                out += (D ? D[d] * x : 0.0);"),
    "B read in place of C": (
        FWD, "acc += Cg[n * L + t] * h[n];\n                }",
        "acc += Bg[n * L + t] * h[n];\n                }"),
    "sign of A flipped": (
        FWD, "const double abar = exp(dt * A[d * N + n]);",
        "const double abar = exp(-dt * A[d * N + n]);"),
    "SSD causal mask off by one": (
        FWD, "for (int64_t j = 0; j <= i; ++j) {  /* token t0+j */",
        "for (int64_t j = 0; j < i; ++j) {  /* token t0+j */"),
    "SSD state decay across chunks dropped": (
        FWD, "double acc = exp(a * S_end) * hprev[n * headdim + p];",
        "double acc = hprev[n * headdim + p];"),
    "scalar-A step bias dropped": (
        FWD, "double step = dth[t] + (dt_bias ? dt_bias[hh] : 0.0);",
        "double step = dth[t];"),
    "backward: A factor dropped from ddelta": (
        BWD, "ddt += g[n] * (a * abar * h_prev[n] + Bg[n * L + t] * x);",
        "ddt += g[n] * (abar * h_prev[n] + Bg[n * L + t] * x);"),
    "backward: dC from the previous state": (
        BWD, "dCg[n * L + t] += dout * h_t[n];", "dCg[n * L + t] += dout * h_prev[n];"),
    "backward: step size dropped from dB": (
        BWD, "dBg[n * L + t] += g[n] * dt * x;", "dBg[n * L + t] += g[n] * x;"),
    "backward: decay applied before adding dout C": (
        BWD,
        "g[n] += dout * Cg[n * L + t];\n"
        "                    dCg[n * L + t] += dout * h_t[n];",
        "g[n] *= exp(dt * a);\n"
        "                    g[n] += dout * Cg[n * L + t];\n"
        "                    dCg[n * L + t] += dout * h_t[n];"),
    "backward: sigmoid of the softplus with the wrong sign": (
        BWD, "dDelta = ddt / (1.0 + exp(-(delta[row + t] + bias)));",
        "dDelta = ddt / (1.0 + exp(delta[row + t] + bias));"),
}


def _copy_and_run(base, name, suite, source):
    d = os.path.join(base, "".join(c if c.isalnum() else "_" for c in name))
    skip = shutil.ignore_patterns("_build", "__pycache__")
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"), ignore=skip)
    with open(os.path.join(d, "oracle", "selscan_oracle.c"), "w") as f:
        f.write(source)
    shutil.copytree(os.path.join(ROOT, "synthetic"), os.path.join(d, "synthetic"), ignore=skip)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(d, "tests", "golden"))
    for f in ("conftest.py", os.path.basename(suite)):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(d, "tests", f))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        suite], cwd=d, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-1500:] + r.stderr[-500:]


def test_planted_mistakes_fail_the_pins(tmp_path):
    src = open(SRC).read()
    jobs = {"control (forward pins)": (FWD, src), "control (backward pins)": (BWD, src)}
    for name, (suite, old, new) in MUTATIONS.items():
        assert src.count(old) == 1, f"{name}: the text to mutate is no longer in the oracle"
        jobs[name] = (suite, src.replace(old, new))
    workers = max(2, min(8, os.cpu_count() or 2))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        futures = {n: ex.submit(_copy_and_run, str(tmp_path), n, s, c)
                   for n, (s, c) in jobs.items()}
        results = {n: f.result() for n, f in futures.items()}
    for name in ("control (forward pins)", "control (backward pins)"):
        assert results[name][0] == 0, f"{name} failed:\n{results[name][1]}"
    missed = [n for n in MUTATIONS if results[n][0] == 0]
    assert not missed, f"mistakes no pin caught: {missed}"
