"""Comparison metrics and tolerances for CUDA-vs-oracle parity.

Bars (fp16 inputs, fp32 accumulation, compared with the FP64 oracle):
  max_abs  = max |gpu - ref|                      <= 4e-3
  rel_fro  = ||gpu - ref||_F / ||ref||_F          <= 1e-3
  max |gpu_lse - ref_lse|                          <= 1e-3

Every check also records its measured values against its bars (``MARGINS``);
``conftest.py`` prints them at the end of the run, so the margin behind each
passing test is visible in the log.
"""
import os

import numpy as np

MAX_ABS = 4e-3
REL_FRO = 1e-3
LSE_ABS = 1e-3

# (test id, what, metric name, measured value, bar)
MARGINS = []


def _test_id():
    cur = os.environ.get("PYTEST_CURRENT_TEST", "")
    return cur.split(" ")[0] if cur else "(outside pytest)"


def record(what, name, value, bar):
    MARGINS.append((_test_id(), what, name, float(value), float(bar)))


def metrics(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = gpu - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff)) / den if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_out_close(gpu, ref, what="out", max_abs=MAX_ABS, rel_fro=REL_FRO):
    assert np.all(np.isfinite(np.asarray(gpu, dtype=np.float64))), f"{what}: non-finite values"
    ma, rf = metrics(gpu, ref)
    record(what, "max_abs", ma, max_abs)
    record(what, "rel_fro", rf, rel_fro)
    assert ma <= max_abs and rf <= rel_fro, f"{what}: max_abs={ma:.3e} rel_fro={rf:.3e}"
    return ma, rf


def assert_lse_close(gpu, ref, what="lse", tol=LSE_ABS):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    both_inf = np.isneginf(gpu) & np.isneginf(ref)
    d = np.where(both_inf, 0.0, np.abs(gpu - ref))
    m = float(np.max(d)) if d.size else 0.0
    record(what, "dlse", m, tol)
    assert m <= tol, f"{what}: max |dLSE| = {m:.3e}"
    return m


def fp16_ulp(x):
    """Spacing of fp16 numbers at |x| (subnormal spacing below 2^-14)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return 2.0 ** (e - 10)


def summary_lines():
    """One line per test: the worst measured/bar ratio of each metric, then the
    same for every check whose label names a 32768-token workload."""
    by_test = {}
    for tid, what, name, val, bar in MARGINS:
        t = by_test.setdefault(tid, {})
        cur = t.get(name)
        if cur is None or val / bar > cur[0] / cur[1]:
            t[name] = (val, bar)
    order = ("max_abs", "rel_fro", "dlse", "elem_bound")

    def fmt(t):
        return "  ".join(f"{n} {t[n][0]:.2e} ({t[n][0] / t[n][1]:.2f} of bar)" for n in order if n in t)

    lines = [f"{tid.split('::', 1)[-1]}: {fmt(t)}" for tid, t in by_test.items()]
    big = {}
    for tid, what, name, val, bar in MARGINS:
        if "32k" in what or "32768" in what:
            big.setdefault(what, {})[name] = (val, bar)
    if big:
        lines.append("-- checks on the 32768-token workloads --")
        lines += [f"{what}: {fmt(t)}" for what, t in big.items()]
    return lines
