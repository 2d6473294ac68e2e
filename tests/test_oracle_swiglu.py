"""Pins for the Spatial SwiGLU oracle (oracle/swiglu.py), CPU only.

Each pin is independent of the oracle's code: a hand-worked 2x2 example
(tests/golden/swiglu_2x2.json), the depthwise convolution against
scipy.signal.correlate2d, the whole block against torch's CPU primitives
(linear, grouped conv2d, silu) in float64, the translation a single
off-centre tap must produce, the closed form of a constant field with its
border, and the gate's zero.  Planted mistakes in a copy of the oracle must
fail them (see the last tests).
"""
import json
import os
import shutil
import subprocess
import sys

import numpy as np
import pytest
import scipy.signal
import torch

import oracle.swiglu as sw

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden", "swiglu_2x2.json")


def rand_block(rng, B, gh, gw, C, F):
    return (rng.standard_normal((B, gh, gw, C)), rng.standard_normal((2 * F, C)),
            rng.standard_normal(2 * F), rng.standard_normal((F, 3, 3)),
            rng.standard_normal(F), rng.standard_normal((C, F)), rng.standard_normal(C))


def rel(a, b):
    d = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (d if d > 0 else 1.0))


def test_hand_worked_2x2():
    with open(GOLDEN) as f:
        gd = json.load(f)
    x = np.array(gd["x"], float)[None, :, :, None]
    y = sw.forward(x, np.array(gd["w_gu"], float), np.array(gd["b_gu"], float),
                   np.array(gd["w_dw"], float), np.array(gd["b_dw"], float),
                   np.array(gd["w_down"], float), np.array(gd["b_down"], float))
    assert np.allclose(y[0, :, :, 0], np.array(gd["expected_y"]), rtol=0, atol=1e-9)


@pytest.mark.parametrize("grid", [(1, 1), (2, 3), (5, 4), (7, 9)])
def test_depthwise_is_correlate2d(grid):
    rng = np.random.default_rng(1)
    gh, gw = grid
    B, C, F = 2, 3, 5
    args = rand_block(rng, B, gh, gw, C, F)
    g, u, v, h, y = sw.forward(*args, parts=True)
    w_dw, b_dw = args[3], args[4]
    for b in range(B):
        for f in range(F):
            ref = scipy.signal.correlate2d(u[b, :, :, f], w_dw[f], mode="same",
                                           boundary="fill", fillvalue=0.0) + b_dw[f]
            assert np.allclose(v[b, :, :, f], ref, rtol=1e-13, atol=1e-12)


@pytest.mark.parametrize("shape", [(1, 4, 6, 8, 12), (2, 5, 3, 6, 10), (1, 1, 1, 4, 4)])
def test_block_matches_torch_cpu_primitives(shape):
    B, gh, gw, C, F = shape
    rng = np.random.default_rng(2)
    x, w_gu, b_gu, w_dw, b_dw, w_down, b_down = rand_block(rng, B, gh, gw, C, F)
    T = lambda a: torch.from_numpy(np.asarray(a, np.float64))  # noqa: E731
    gu = torch.nn.functional.linear(T(x), T(w_gu), T(b_gu))
    g, u = gu[..., :F], gu[..., F:]
    v = torch.nn.functional.conv2d(u.permute(0, 3, 1, 2), T(w_dw)[:, None], T(b_dw),
                                   padding=1, groups=F).permute(0, 2, 3, 1)
    ref = torch.nn.functional.linear(torch.nn.functional.silu(g) * v, T(w_down), T(b_down))
    y = sw.forward(x, w_gu, b_gu, w_dw, b_dw, w_down, b_down)
    assert rel(y, ref.numpy()) < 1e-12


def test_single_tap_translates():
    """Only the top-left tap set: v[y, x] = u[y - 1, x - 1], zero on the first
    row and column (fixes the orientation of the cross-correlation)."""
    rng = np.random.default_rng(3)
    B, gh, gw, C, F = 1, 4, 5, 3, 2
    x, w_gu, b_gu, _, _, w_down, b_down = rand_block(rng, B, gh, gw, C, F)
    w_dw = np.zeros((F, 3, 3))
    w_dw[:, 0, 0] = 1.0
    g, u, v, h, y = sw.forward(x, w_gu, b_gu, w_dw, np.zeros(F), w_down, b_down, parts=True)
    assert np.all(v[:, 0, :, :] == 0) and np.all(v[:, :, 0, :] == 0)
    assert np.array_equal(v[:, 1:, 1:, :], u[:, :-1, :-1, :])


def test_constant_field_border():
    """x = 0: u is the constant b_u per channel, so v = b_dw + b_u * (sum of the
    taps that fall inside the grid): 4 at a corner, 6 on an edge, 9 inside."""
    rng = np.random.default_rng(4)
    gh, gw, C, F = 4, 5, 3, 2
    _, w_gu, b_gu, _, b_dw, w_down, b_down = rand_block(rng, 1, gh, gw, C, F)
    w_dw = np.ones((F, 3, 3))
    g, u, v, h, y = sw.forward(np.zeros((1, gh, gw, C)), w_gu, b_gu, w_dw, b_dw, w_down,
                               b_down, parts=True)
    bu = b_gu[F:]
    for (yy, xx), n in {(0, 0): 4, (0, 2): 6, (2, 0): 6, (3, 4): 4, (1, 2): 9, (2, 3): 9}.items():
        assert np.allclose(v[0, yy, xx], b_dw + n * bu, rtol=1e-14, atol=1e-14)


def test_gate_zero_gives_bias():
    """SiLU(0) = 0: with a zero gate the block returns b_down whatever the value."""
    rng = np.random.default_rng(5)
    B, gh, gw, C, F = 1, 3, 3, 4, 6
    x, w_gu, b_gu, w_dw, b_dw, w_down, b_down = rand_block(rng, B, gh, gw, C, F)
    w_gu[:F] = 0.0
    b_gu[:F] = 0.0
    y = sw.forward(x, w_gu, b_gu, w_dw, b_dw, w_down, b_down)
    assert np.array_equal(y, np.broadcast_to(b_down, y.shape))


MUTANTS = [
    ("convolution instead of cross-correlation",
     "v += w_dw[:, a, c] * up[:, a:a + gh, c:c + gw, :]",
     "v += w_dw[:, 2 - a, 2 - c] * up[:, a:a + gh, c:c + gw, :]"),
    ("gate and value swapped", "g, u = gu[..., :F], gu[..., F:]", "u, g = gu[..., :F], gu[..., F:]"),
    ("sigmoid gate instead of SiLU", "h = g / (1.0 + np.exp(-g)) * v", "h = 1.0 / (1.0 + np.exp(-g)) * v"),
    ("depthwise bias dropped", "v = np.broadcast_to(b_dw, u.shape).copy()", "v = np.zeros(u.shape)"),
    ("wrap-around instead of zero padding",
     "up[:, 1:gh + 1, 1:gw + 1, :] = u",
     "up[:, 1:gh + 1, 1:gw + 1, :] = u; up[:, 0] = up[:, gh]; up[:, gh + 1] = up[:, 1]"),
    ("taps transposed", "v += w_dw[:, a, c] * up", "v += w_dw[:, c, a] * up"),
    ("value bias in the padding",
     "up = np.zeros((B, gh + 2, gw + 2, F))",
     "up = np.zeros((B, gh + 2, gw + 2, F)) + b_gu[F:]"),
]


def _run_pins(tmp, edit):
    os.makedirs(os.path.join(tmp, "oracle"))
    shutil.copy(os.path.join(ROOT, "oracle", "swiglu.py"), os.path.join(tmp, "oracle", "swiglu.py"))
    open(os.path.join(tmp, "oracle", "__init__.py"), "w").close()
    os.makedirs(os.path.join(tmp, "tests", "golden"))
    shutil.copy(os.path.abspath(__file__), os.path.join(tmp, "tests", "test_pins.py"))
    shutil.copy(GOLDEN, os.path.join(tmp, "tests", "golden"))
    path = os.path.join(tmp, "oracle", "swiglu.py")
    if edit:
        old, new = edit
        text = open(path).read()
        assert text.count(old) == 1, old
        open(path, "w").write(text.replace(old, new))
    env = dict(os.environ, PYTHONPATH=tmp, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "-k", "not mutant and not unmodified",
                        os.path.join(tmp, "tests", "test_pins.py")],
                       cwd=tmp, env=env, capture_output=True, text=True, timeout=300)
    return r.returncode, r.stdout[-1500:] + r.stderr[-1500:]


def test_unmodified_copy_passes(tmp_path):
    rc, log = _run_pins(str(tmp_path), None)
    assert rc == 0, log


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    rc, log = _run_pins(str(tmp_path), (old, new))
    assert rc == 1, f"mutant '{name}' survived (pytest exit {rc}):\n{log}"
