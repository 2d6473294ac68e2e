"""Planted mistakes in a copy of the oracle (CPU only).

Each mutant below is a plausible error in oracle/gla_oracle.c: a wrong gate
sign, a dropped or misplaced term, an exclusive instead of inclusive
diagonal, a wrong scan-order map, an off-by-one in the in-chunk log-gate
sums.  For every one, the pins of tests/test_oracle_pins.py must fail; the
unmodified copy must pass.  The mutants are built in a temporary directory,
so the committed oracle is never touched.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = "gla_oracle.c"

# (name, [(original text, replacement), ...]); every original must occur once.
MUTANTS = [
    ("gate sign", [("const double a = exp(lat[i]);", "const double a = exp(-lat[i]);")]),
    ("write term dropped",
     [("Si[j] = a * Si[j] + kt[i] * vt[j];", "Si[j] = a * Si[j];")]),
    ("gate applied after the write",
     [("Si[j] = a * Si[j] + kt[i] * vt[j];", "Si[j] = a * (Si[j] + kt[i] * vt[j]);")]),
    ("output reads the state before the write",
     [("ot[j] += qt[i] * Si[j];", "ot[j] += qt[i] * (Si[j] - kt[i] * vt[j]);")]),
    ("reversed scans reverse each row",
     [("memcpy(dst + (size_t)p * d, tmp + (size_t)(n - 1 - p) * d,",
       "memcpy(dst + (size_t)p * d, tmp + (size_t)((p / gw) * gw + (gw - 1 - p % gw)) * d,"),
      ("memcpy(tmp + (size_t)(n - 1 - p) * d, src + (size_t)p * d,",
       "memcpy(tmp + (size_t)((p / gw) * gw + (gw - 1 - p % gw)) * d, src + (size_t)p * d,")]),
    ("top-to-bottom scans without the transpose",
     [("    if (direction == 2 || direction == 3) {\n        /* transpose",
       "    if (direction == 3) {\n        /* transpose"),
      ("    if (direction == 2 || direction == 3) {\n        for (int y = 0; y < gh; ++y)\n"
       "            for (int x = 0; x < gw; ++x)\n                memcpy(dst +",
       "    if (direction == 3) {\n        for (int y = 0; y < gh; ++y)\n"
       "            for (int x = 0; x < gw; ++x)\n                memcpy(dst +")]),
    ("chunk log-gate sums skip the chunk's first token",
     [("acc += la[(size_t)(t0 + u) * dk + i];", "acc += (u > 0) ? la[(size_t)(t0 + u) * dk + i] : 0.0;")]),
    ("chunk state contribution decays the wrong way",
     [("exp(g[i] - b[(size_t)w * dk + i])", "exp(b[(size_t)w * dk + i] - g[i])")]),
    ("in-chunk scores without the diagonal",
     [("for (int w = 0; w <= u; ++w) {", "for (int w = 0; w < u; ++w) {")]),
    ("inter-chunk term with the exclusive gate sum",
     [("q[(size_t)t * dk + i] * exp(b[(size_t)u * dk + i]);",
       "q[(size_t)t * dk + i] * exp(u > 0 ? b[(size_t)(u - 1) * dk + i] : 0.0);")]),
    ("boundary state not decayed",
     [("S[(size_t)i * dv + j] = gam * S[(size_t)i * dv + j] + dS[(size_t)i * dv + j];",
       "S[(size_t)i * dv + j] = S[(size_t)i * dv + j] + dS[(size_t)i * dv + j];")]),
]


def _run_pins(tmp, edits):
    """Copy the oracle and the pin tests into tmp, apply edits, run the pins;
    return pytest's exit code."""
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(tmp, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    os.makedirs(os.path.join(tmp, "tests"))
    shutil.copy(os.path.join(ROOT, "tests", "test_oracle_pins.py"), os.path.join(tmp, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(tmp, "tests", "golden"))
    path = os.path.join(tmp, "oracle", SRC)
    with open(path) as f:
        text = f.read()
    for old, new in edits:
        assert text.count(old) == 1, f"mutation anchor not found exactly once: {old[:60]!r}"
        text = text.replace(old, new)
    with open(path, "w") as f:
        f.write(text)
    env = dict(os.environ, PYTHONPATH=tmp, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(tmp, "tests", "test_oracle_pins.py")],
                       cwd=tmp, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:] + r.stderr[-2000:]


def test_unmodified_copy_passes(tmp_path):
    rc, log = _run_pins(str(tmp_path), [])
    assert rc == 0, log


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, edits):
    rc, log = _run_pins(str(tmp_path), edits)
    assert rc == 1, f"mutant '{name}' survived the pins (pytest exit {rc}):\n{log}"
