"""The pins catch plausible mistakes in the oracle.

Each case plants one single-line mistake in a scratch copy of oracle/cf_oracle.c
(on the CPU, in a temporary directory), builds it, and runs the oracle's pin
tests against that build: at least one pin must fail.  The unmodified source
must pass the same run, so a failure is the mistake's doing.
"""
import concurrent.futures
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "cf_oracle.c")
PINS = [os.path.join(ROOT, "tests", "test_oracle_quant.py"), os.path.join(ROOT, "tests", "test_oracle_lowrank.py"),
        os.path.join(ROOT, "tests", "test_oracle_attention.py")]

# (name, text in cf_oracle.c, replacement, replace every occurrence)
MUTATIONS = [
    ("residual sign", "float diff = bf16_to_float(x[i0 + j]) - bf16_to_float(base[i0 + j]);",
     "float diff = bf16_to_float(base[i0 + j]) - bf16_to_float(x[i0 + j]);", False),
    ("error feedback dropped", "a[j] = diff + err[i0 + j];", "a[j] = diff;", False),
    ("new error sign", "for (int j = 0; j < G; ++j) err[i0 + j] = a[j] - d[j];",
     "for (int j = 0; j < G; ++j) err[i0 + j] = d[j] - a[j];", False),
    ("round half away from zero", "float r = rintf(y);", "float r = roundf(y);", False),
    ("MSB-first packing", "int64_t bit = i * k + b;", "int64_t bit = i * k + (k - 1 - b);", True),
    ("levels per side", "return k >= 2 ? (1 << (k - 1)) - 1 : 1;", "return k >= 2 ? (1 << (k - 1)) : 1;", False),
    ("sign of zero", "unsigned c = (a[j] >= 0.0f) ? 1u : 0u;", "unsigned c = (a[j] > 0.0f) ? 1u : 0u;", False),
    ("cache not accumulated", "cache[i] = cache[i] + dv;", "cache[i] = dv;", False),
    ("bf16 ties rounded up", "return (uint16_t)((u + 0x7fffu + lsb) >> 16);", "return (uint16_t)((u + 0x8000u) >> 16);",
     False),
    ("A^T dropped from the iteration", "mat_AtP(m, n, r, A, P, Q);", "(void)P;", False),
    ("Cholesky divisor", "R[p * r + q] = v / R[p * r + p];", "R[p * r + q] = v / diag;", False),
    ("zero-group threshold at FLT_MIN", "CFO_SCALE_MIN = 7.52316384526264e-37f;", "CFO_SCALE_MIN = 1.17549435e-38f;",
     False),
    ("zero-group threshold inclusive", "} else if (s < CFO_SCALE_MIN) {", "} else if (s <= CFO_SCALE_MIN) {", False),
    ("attention scale 1/64", "w[j] = s / 8.0;", "w[j] = s / 64.0;", False),
    ("softmax max not taken out", "w[j] = exp(w[j] - mx);", "w[j] = exp(w[j]);", False),
    ("softmax not normalised", "out[i * cols + c0 + c] = o / z;", "out[i * cols + c0 + c] = o;", False),
    ("log-sum-exp without the maximum", "lse[i * (cols / 64) + h] = mx + log(z);",
     "lse[i * (cols / 64) + h] = log(z);", False),
    ("log-sum-exp in base 2", "lse[i * (cols / 64) + h] = mx + log(z);",
     "lse[i * (cols / 64) + h] = mx + log2(z);", False),
]


def _build(text, out):
    import oracle

    src = out + ".c"
    with open(src, "w") as f:
        f.write(text)
    subprocess.check_call(["gcc", *oracle._CFLAGS, "-o", out, src, "-lm"])
    return out


def _run_pins(lib):
    env = dict(os.environ, CF_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-800:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    original = open(SRC).read()
    libs = {"unmodified": _build(original, str(tmp_path / "orig.so"))}
    for i, (name, old, new, every) in enumerate(MUTATIONS):
        assert old in original, name
        text = original.replace(old, new) if every else original.replace(old, new, 1)
        libs[name] = _build(text, str(tmp_path / f"mut{i}.so"))
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = dict(zip(libs, ex.map(_run_pins, libs.values())))
    rc, out = results.pop("unmodified")
    assert rc == 0, out
    survivors = [name for name, (rc, _) in results.items() if rc == 0]
    assert not survivors, f"mistakes no pin catches: {survivors}"
