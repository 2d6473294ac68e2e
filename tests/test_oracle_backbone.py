"""Pins for the backbone-layer oracle (oracle/backbone.py), CPU only.

Each pin is independent of the oracle's code:
- the layer and a 5-layer stack against a restatement with torch's float64
  primitives (layer_norm, linear, logsigmoid, rms_norm, silu, grouped conv2d)
  and a token-by-token recurrence that walks scan orders listed position by
  position;
- the identity the residual layout gives when both branches' output maps are
  zero;
- the geometry of the scan directions: rotating the grid by 180 degrees turns
  a right-to-left scan into a left-to-right one, and transposing it turns
  top-to-bottom into left-to-right, provided the convolution taps turn with
  the grid.
Planted mistakes in a copy of the oracle must fail them (the last tests).
"""
import os
import shutil
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

import oracle.backbone as bb
from recurrent_vision_backbone_chunkwise_b200.inputs import make_backbone_params

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _params(C=128, F=256, n=1, seed=0):
    return [{k: v.double().numpy() for k, v in p.items()} for p in make_backbone_params(C, F, n, "f16", seed)]


def _x(B=1, gh=3, gw=4, C=128, seed=0):
    return np.random.default_rng(seed).standard_normal((B, gh, gw, C))


def _scan_positions(gh, gw, direction):
    rows = [(y, x) for y in range(gh) for x in range(gw)]
    cols = [(y, x) for x in range(gw) for y in range(gh)]
    return {0: rows, 1: rows[::-1], 2: cols, 3: cols[::-1]}[direction]


def _torch_layer(x, p, direction):
    x = torch.from_numpy(np.asarray(x, dtype=np.float64))
    P = {k: torch.from_numpy(np.asarray(v, dtype=np.float64)) for k, v in p.items()}
    B, gh, gw, C = x.shape
    H, d = C // 64, 64
    F = P["w_dw"].shape[0]
    x1 = Fn.layer_norm(x, (C,), P["ln1_w"], P["ln1_b"], eps=1e-6)
    q = Fn.linear(x1, P["w_q"])
    k = Fn.linear(x1, P["w_k"]) / 8.0
    v = Fn.linear(x1, P["w_v"])
    la = Fn.logsigmoid(Fn.linear(x1, P["w_a"], P["b_a"])) / 16.0
    z = Fn.linear(x1, P["w_z"])
    o = torch.zeros(B, gh, gw, H * d, dtype=torch.float64)
    for b in range(B):
        for h in range(H):
            c = slice(h * d, (h + 1) * d)
            S = torch.zeros(d, d, dtype=torch.float64)
            for (yy, xx) in _scan_positions(gh, gw, direction):
                S = torch.exp(la[b, yy, xx, c])[:, None] * S + torch.outer(k[b, yy, xx, c], v[b, yy, xx, c])
                o[b, yy, xx, c] = q[b, yy, xx, c] @ S
    t = torch.cat([Fn.rms_norm(o[..., h * d:(h + 1) * d], (d,), P["w_n"][h], eps=1e-5) for h in range(H)], -1)
    t = t * Fn.silu(z)
    xm = x + Fn.linear(t, P["w_o"])
    x2 = Fn.layer_norm(xm, (C,), P["ln2_w"], P["ln2_b"], eps=1e-6)
    gu = Fn.linear(x2, P["w_gu"], P["b_gu"])
    g, u = gu[..., :F], gu[..., F:]
    vc = Fn.conv2d(u.permute(0, 3, 1, 2), P["w_dw"][:, None], P["b_dw"], padding=1, groups=F).permute(0, 2, 3, 1)
    return (xm + Fn.linear(Fn.silu(g) * vc, P["w_down"], P["b_down"])).numpy()


def _close(a, b, tol=1e-10):
    return np.max(np.abs(a - b)) <= tol * max(1.0, np.max(np.abs(b)))


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_layer_matches_torch_restatement(direction):
    p = _params(seed=1)[0]
    x = _x(B=2, gh=3, gw=4, seed=2)
    assert _close(bb.layer_forward(x, p, direction), _torch_layer(x, p, direction))


def test_stack_cycles_the_directions():
    layers = _params(n=5, seed=3)
    x = _x(gh=4, gw=3, seed=4)
    ref = x
    for l, p in enumerate(layers):
        ref = _torch_layer(ref, p, l % 4)
    assert _close(bb.backbone_forward(x, layers), ref)


def test_zero_output_maps_give_the_identity():
    p = _params(seed=5)[0]
    p["w_o"] = np.zeros_like(p["w_o"])
    p["w_down"] = np.zeros_like(p["w_down"])
    p["b_down"] = np.zeros_like(p["b_down"])
    x = _x(seed=6)
    for direction in range(4):
        assert np.array_equal(bb.layer_forward(x, p, direction), x)


def _rot180(a):
    return a[:, ::-1, ::-1, :].copy()


def _turned(p, how):
    q = dict(p)
    q["w_dw"] = p["w_dw"][:, ::-1, ::-1].copy() if how == "rot180" else np.swapaxes(p["w_dw"], 1, 2).copy()
    return q


@pytest.mark.parametrize("d_from,d_to", [(1, 0), (3, 2)])
def test_rotating_the_grid_reverses_the_scan(d_from, d_to):
    p = _params(seed=7)[0]
    x = _x(gh=3, gw=5, seed=8)
    lhs = bb.layer_forward(x, p, d_from)
    rhs = _rot180(bb.layer_forward(_rot180(x), _turned(p, "rot180"), d_to))
    assert _close(lhs, rhs)


def test_transposing_the_grid_turns_columns_into_rows():
    p = _params(seed=9)[0]
    x = _x(gh=3, gw=5, seed=10)
    xt = np.swapaxes(x, 1, 2).copy()
    lhs = bb.layer_forward(x, p, 2)
    rhs = np.swapaxes(bb.layer_forward(xt, _turned(p, "transpose"), 0), 1, 2)
    assert _close(lhs, rhs)


# Planted mistakes: (name, original text, replacement); each original must
# occur once in oracle/backbone.py.
MUTANTS = [
    ("mixer residual dropped", 'xm = x + t @ P["w_o"].T', 'xm = t @ P["w_o"].T'),
    ("second norm with the first norm's weights", 'x2 = layer_norm(xm, P["ln2_w"], P["ln2_b"])',
     'x2 = layer_norm(xm, P["ln1_w"], P["ln1_b"])'),
    ("keys not scaled", 'k = _heads(x1 @ P["w_k"].T, H) / np.sqrt(HEAD_DIM)', 'k = _heads(x1 @ P["w_k"].T, H)'),
    ("gates without 1/tau", 'P["b_a"]), H) / TAU', 'P["b_a"]), H)'),
    ("direction cycle off by one", "x = layer_forward(x, p, l % 4)", "x = layer_forward(x, p, (l + 1) % 4)"),
    ("output gate from the un-normalised input", 'z = x1 @ P["w_z"].T', 'z = x @ P["w_z"].T'),
    ("heads split channel-major", "t.reshape(B, gh, gw, H, HD // H)",
     "np.swapaxes(t.reshape(B, gh, gw, HD // H, H), -1, -2)"),
    ("variance about zero instead of the mean", "var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)",
     "var = (x ** 2).mean(axis=-1, keepdims=True)"),
]


def _run_pins(tmp, edit):
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(tmp, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    pkg = os.path.join(tmp, "recurrent_vision_backbone_chunkwise_b200")
    os.makedirs(pkg)
    open(os.path.join(pkg, "__init__.py"), "w").close()
    shutil.copy(os.path.join(ROOT, "recurrent_vision_backbone_chunkwise_b200", "inputs.py"), pkg)
    os.makedirs(os.path.join(tmp, "tests"))
    shutil.copy(os.path.abspath(__file__), os.path.join(tmp, "tests", "test_pins.py"))
    path = os.path.join(tmp, "oracle", "backbone.py")
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
                       cwd=tmp, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-2000:] + r.stderr[-2000:]


def test_unmodified_copy_passes(tmp_path):
    rc, log = _run_pins(str(tmp_path), None)
    assert rc == 0, log


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    rc, log = _run_pins(str(tmp_path), (old, new))
    assert rc == 1, f"mutant '{name}' survived (pytest exit {rc}):\n{log}"
