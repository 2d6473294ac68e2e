"""Pins for the output-tail oracle (oracle/output_tail.py), CPU only.

Each pin is independent of the oracle's code:
- a hand-worked example with closed-form values (tests/golden/output_tail_hand.json);
- the whole tail against torch's CPU primitives (rms_norm, silu) in float64;
- the invariants the RMS norm fixes (scale invariance, odd symmetry, unit RMS);
- the gate's zero;
- the locality of each head.
Planted mistakes in a copy of the oracle must fail them (the last tests).
"""
import json
import os
import shutil
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle.output_tail as ot

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden", "output_tail_hand.json")


def _inputs(B=2, H=3, gh=4, gw=5, dv=8, seed=0):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B, H, gh, gw, dv)), r.standard_normal((B, gh, gw, H * dv)),
            1.0 + 0.1 * r.standard_normal((H, dv)))


def test_hand_worked_example():
    with open(GOLDEN) as f:
        doc = json.load(f)
    for c in doc["cases"]:
        y = ot.forward(np.array(c["o"]), np.array(c["z"]), np.array(c["w"]), c["eps"])
        assert np.allclose(y, np.array(c["expected_y"]), rtol=0, atol=1e-12), (c["eps"], y)


@pytest.mark.parametrize("eps", [0.0, 1e-5, 0.5])
def test_matches_torch_primitives(eps):
    o, z, w = _inputs(seed=1)
    B, H, gh, gw, dv = o.shape
    ot_ = torch.from_numpy(o)
    parts = []
    for h in range(H):
        n = torch.nn.functional.rms_norm(ot_[:, h], (dv,), weight=torch.from_numpy(w[h]), eps=eps)
        zh = torch.from_numpy(z[..., h * dv:(h + 1) * dv])
        parts.append(n * torch.nn.functional.silu(zh))
    ref = torch.cat(parts, dim=-1).numpy()
    assert np.allclose(ot.forward(o, z, w, eps), ref, rtol=1e-12, atol=1e-12)


def test_scale_invariance_and_odd_symmetry():
    o, z, w = _inputs(seed=2)
    y = ot.forward(o, z, w, 0.0)
    assert np.allclose(ot.forward(7.5 * o, z, w, 0.0), y, rtol=1e-12, atol=1e-12)
    assert np.allclose(ot.forward(1e-3 * o, z, w, 0.0), y, rtol=1e-10, atol=1e-12)
    assert np.allclose(ot.forward(-o, z, w, 0.0), -y, rtol=1e-12, atol=1e-12)


def test_unit_rms_with_a_constant_gate():
    """w = 1 and z = ln 3 everywhere (SiLU = (3/4) ln 3): every head's row of
    y / ((3/4) ln 3) has mean square 1 when eps = 0."""
    o, _, _ = _inputs(seed=3)
    B, H, gh, gw, dv = o.shape
    z = np.full((B, gh, gw, H * dv), np.log(3.0))
    y = ot.forward(o, z, np.ones((H, dv)), 0.0) / (0.75 * np.log(3.0))
    ms = (y.reshape(B, gh, gw, H, dv) ** 2).mean(axis=-1)
    assert np.allclose(ms, 1.0, rtol=1e-12)


def test_zero_gate_gives_zero():
    o, z, w = _inputs(seed=4)
    assert np.all(ot.forward(o, np.zeros_like(z), w) == 0.0)


def test_each_head_touches_only_its_channels():
    o, z, w = _inputs(seed=5)
    dv = o.shape[-1]
    y = ot.forward(o, z, w)
    o2 = o.copy()
    o2[:, 1] = 3.0 * np.roll(o2[:, 1], 1, axis=-1) + 0.25
    y2 = ot.forward(o2, z, w)
    changed = np.any(y2 != y, axis=(0, 1, 2))
    assert changed[dv:2 * dv].all()
    assert not changed[:dv].any() and not changed[2 * dv:].any()


# Planted mistakes: (name, original text, replacement); each original must
# occur once in oracle/output_tail.py.
MUTANTS = [
    ("norm over all heads instead of per head",
     "ms = np.mean(oh * oh, axis=-1, keepdims=True)",
     "ms = np.mean(oh * oh, axis=(-2, -1), keepdims=True)"),
    ("sum of squares instead of the mean",
     "ms = np.mean(oh * oh, axis=-1, keepdims=True)",
     "ms = np.sum(oh * oh, axis=-1, keepdims=True)"),
    ("eps outside the square root",
     "n = oh / np.sqrt(ms + eps) * w",
     "n = oh / (np.sqrt(ms) + eps) * w"),
    ("sigmoid gate instead of SiLU",
     "y = n * (zh / (1.0 + np.exp(-zh)))",
     "y = n * (1.0 / (1.0 + np.exp(-zh)))"),
    ("heads merged channel-major",
     "return y.reshape(B, gh, gw, H * dv)",
     "return np.swapaxes(y, -1, -2).reshape(B, gh, gw, H * dv)"),
    ("gate read with the heads interleaved",
     "zh = z.reshape(B, gh, gw, H, dv)",
     "zh = np.swapaxes(z.reshape(B, gh, gw, dv, H), -1, -2)"),
    ("norm weight of the wrong head",
     "n = oh / np.sqrt(ms + eps) * w",
     "n = oh / np.sqrt(ms + eps) * w[::-1]"),
]


def _run_pins(tmp, edit):
    os.makedirs(os.path.join(tmp, "oracle"))
    shutil.copy(os.path.join(ROOT, "oracle", "output_tail.py"), os.path.join(tmp, "oracle", "output_tail.py"))
    open(os.path.join(tmp, "oracle", "__init__.py"), "w").close()
    os.makedirs(os.path.join(tmp, "tests", "golden"))
    shutil.copy(os.path.abspath(__file__), os.path.join(tmp, "tests", "test_pins.py"))
    shutil.copy(GOLDEN, os.path.join(tmp, "tests", "golden"))
    path = os.path.join(tmp, "oracle", "output_tail.py")
    if edit:
        old, new = edit
        with open(path) as f:
            text = f.read()
        assert text.count(old) == 1, f"mutation anchor not found exactly once: {old!r}"
        with open(path, "w") as f:
            f.write(text.replace(old, new))
    env = dict(os.environ, PYTHONPATH=tmp, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "-k", "not mutant and not unmodified",
                        os.path.join(tmp, "tests", "test_pins.py")],
                       cwd=tmp, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:] + r.stderr[-2000:]


def test_unmodified_copy_passes(tmp_path):
    rc, log = _run_pins(str(tmp_path), None)
    assert rc == 0, log


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    rc, log = _run_pins(str(tmp_path), (old, new))
    assert rc == 1, f"mutant '{name}' survived (pytest exit {rc}):\n{log}"
