"""Pins for the GLA gradient oracle (oracle/backward.py, gla_backward.c), CPU only.

Each pin is independent of the oracle's code:
- scalar examples worked by hand with the chain rule: three tokens in all
  four directions (tests/golden/backward_scalar_1x3.json) and the two column
  scans of a 2x2 grid (tests/golden/backward_scalar_2x2_columns.json);
- central finite differences of the forward oracle (itself pinned in
  test_oracle_pins.py), as directional derivatives in all four directions and
  element by element on a tiny plane;
- torch autograd through the brute-force quadratic form (explicit gate
  products, scan orders listed position by position);
- the final-state gradient entering the same way.
The chunked reorganisation of the gradients (oracle.backward.chunkwise_backward)
is checked against them for many chunk lengths.
Planted mistakes in a copy of the oracle must fail them (the last tests).
"""
import os
import shutil
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import oracle.backward as ob

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _case(B=1, H=2, gh=3, gw=4, dk=3, dv=2, seed=0):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, H, gh, gw, dk))
    k = r.standard_normal((B, H, gh, gw, dk))
    v = r.standard_normal((B, H, gh, gw, dv))
    la = -0.5 * np.abs(r.standard_normal((B, H, gh, gw, dk)))
    dO = r.standard_normal((B, H, gh, gw, dv))
    dS = r.standard_normal((B, H, dk, dv))
    return q, k, v, la, dO, dS


def _golden_scalar(name="backward_scalar_1x3.json"):
    import json

    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        g = json.load(f)
    shape = (1, 1, g["grid"][0], g["grid"][1], 1)
    q, k, v = (np.array(g[n], dtype=np.float64).reshape(shape) for n in ("q", "k", "v"))
    la = np.log(np.array(g["alpha"], dtype=np.float64)).reshape(shape)
    dO = np.array(g["d_out"], dtype=np.float64).reshape(shape)
    dS = np.full((1, 1, 1, 1), g["d_final_state"])
    return g, (q, k, v, la, dO, dS)


@pytest.mark.parametrize("name,direction", [("backward_scalar_1x3.json", d) for d in range(4)] +
                         [("backward_scalar_2x2_columns.json", d) for d in (2, 3)])
def test_hand_worked_scalar_gradients(name, direction):
    g, (q, k, v, la, dO, dS) = _golden_scalar(name)
    exp = next(e for e in g["expected"].values() if direction in e["directions"])
    o, S = oracle.forward(q, k, v, la, direction)
    assert np.allclose(o.ravel(), exp["out"], rtol=0, atol=1e-12)
    assert abs(float(S.ravel()[0]) - exp["final_state"]) <= 1e-12
    grads = ob.backward(q, k, v, la, dO, direction, d_final_state=dS)
    for name, got in zip(("dq", "dk", "dv", "dlog_alpha"), grads):
        assert np.allclose(np.asarray(got).ravel(), exp[name], rtol=0, atol=1e-12), name
    # the chunked reorganisation at a chunk shorter than the scan
    grads_c = ob.chunkwise_backward(q, k, v, la, dO, direction, chunk=2, d_final_state=dS)
    for name, got in zip(("dq", "dk", "dv", "dlog_alpha"), grads_c):
        assert np.allclose(np.asarray(got).ravel(), exp[name], rtol=0, atol=1e-12), name


def _loss(q, k, v, la, dO, dS, direction):
    o, S = oracle.forward(q, k, v, la, direction)
    return float(np.sum(dO * o) + (0.0 if dS is None else np.sum(dS * S)))


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
@pytest.mark.parametrize("with_state", [False, True])
def test_directional_derivatives_match_finite_differences(direction, with_state):
    q, k, v, la, dO, dS = _case(seed=direction + 10 * with_state)
    dS = dS if with_state else None
    grads = ob.backward(q, k, v, la, dO, direction, dS)
    r = np.random.default_rng(99)
    args = [q, k, v, la]
    eps = 1e-6
    for idx in range(4):
        delta = r.standard_normal(args[idx].shape)
        plus = [a.copy() for a in args]
        minus = [a.copy() for a in args]
        plus[idx] += eps * delta
        minus[idx] -= eps * delta
        fd = (_loss(*plus, dO, dS, direction) - _loss(*minus, dO, dS, direction)) / (2 * eps)
        an = float(np.sum(grads[idx] * delta))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (idx, fd, an)


def test_every_element_matches_finite_differences():
    q, k, v, la, dO, dS = _case(B=1, H=1, gh=2, gw=3, dk=2, dv=2, seed=5)
    for direction in range(4):
        grads = ob.backward(q, k, v, la, dO, direction, dS)
        args = [q, k, v, la]
        for idx in range(4):
            fd = np.zeros_like(args[idx])
            for pos in np.ndindex(args[idx].shape):
                plus = [a.copy() for a in args]
                minus = [a.copy() for a in args]
                plus[idx][pos] += 1e-6
                minus[idx][pos] -= 1e-6
                fd[pos] = (_loss(*plus, dO, dS, direction) - _loss(*minus, dO, dS, direction)) / 2e-6
            assert np.allclose(grads[idx], fd, rtol=1e-6, atol=1e-7), (direction, idx)


def _scan_positions(gh, gw, direction):
    rows = [(y, x) for y in range(gh) for x in range(gw)]
    cols = [(y, x) for x in range(gw) for y in range(gh)]
    return {0: rows, 1: rows[::-1], 2: cols, 3: cols[::-1]}[direction]


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_autograd_of_the_quadratic_form(direction):
    """o_t = sum_{s<=t} q_t diag(prod_{u=s+1..t} alpha_u) k_s^T v_s and
    S_final = sum_s diag(prod_{u>s} alpha_u) k_s^T v_s, written with explicit
    products, differentiated by torch."""
    q, k, v, la, dO, dS = _case(B=1, H=1, gh=3, gw=3, dk=2, dv=3, seed=20 + direction)
    tq, tk, tv, tla = (torch.tensor(a, requires_grad=True) for a in (q, k, v, la))
    pos = _scan_positions(3, 3, direction)
    n = len(pos)
    loss = torch.zeros((), dtype=torch.float64)
    alpha = torch.exp(tla)
    for t in range(n):
        yt, xt = pos[t]
        o_t = torch.zeros(3, dtype=torch.float64)
        for s in range(t + 1):
            ys, xs = pos[s]
            g = torch.ones(2, dtype=torch.float64)
            for u in range(s + 1, t + 1):
                g = g * alpha[0, 0, pos[u][0], pos[u][1]]
            o_t = o_t + (tq[0, 0, yt, xt] * g * tk[0, 0, ys, xs]).sum() * tv[0, 0, ys, xs]
        loss = loss + (torch.from_numpy(dO[0, 0, yt, xt]) * o_t).sum()
    S = torch.zeros(2, 3, dtype=torch.float64)
    for s in range(n):
        ys, xs = pos[s]
        g = torch.ones(2, dtype=torch.float64)
        for u in range(s + 1, n):
            g = g * alpha[0, 0, pos[u][0], pos[u][1]]
        S = S + torch.outer(g * tk[0, 0, ys, xs], tv[0, 0, ys, xs])
    loss = loss + (torch.from_numpy(dS[0, 0]) * S).sum()
    loss.backward()
    grads = ob.backward(q, k, v, la, dO, direction, dS)
    for got, ref in zip(grads, (tq.grad, tk.grad, tv.grad, tla.grad)):
        assert np.allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
@pytest.mark.parametrize("chunk", [1, 5, 16, 64, 1000])
def test_chunkwise_backward_equals_the_token_backward(direction, chunk):
    """The chunked reorganisation (boundary states, reverse scan of the state
    gradients, per-chunk matrix products, log-gates through the cumulative
    sum) gives the token-by-token gradients for any chunk length, including
    ones that do not divide the token count and one longer than the scan."""
    q, k, v, la, dO, dS = _case(B=2, H=1, gh=5, gw=7, dk=3, dv=4, seed=30 + direction)
    for state in (None, dS):
        ref = ob.backward(q, k, v, la, dO, direction, state)
        got = ob.chunkwise_backward(q, k, v, la, dO, direction, chunk, state)
        for a, b in zip(got, ref):
            assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(b))


# Planted mistakes: (name, original text, replacement); each original must
# occur once in oracle/gla_backward.c.
MUTANTS = [
    ("state gradient not decayed", "for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] *= a;",
     "for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] *= 1.0;"),
    ("gate gradient without the alpha factor", "dla[(size_t)t * dk + i] = exp(la[(size_t)t * dk + i]) * sa;",
     "dla[(size_t)t * dk + i] = sa;"),
    ("gate gradient against the updated state", "sa += G[(size_t)i * dv + j] * Sp[(size_t)i * dv + j];",
     "sa += G[(size_t)i * dv + j] * St[(size_t)i * dv + j];"),
    ("query gradient against the previous state", "sq += gt[j] * St[(size_t)i * dv + j];",
     "sq += gt[j] * Sp[(size_t)i * dv + j];"),
    ("value gradient through the query", "for (int i = 0; i < dk; ++i) s += kt[i] * G[(size_t)i * dv + j];",
     "for (int i = 0; i < dk; ++i) s += qt[i] * G[(size_t)i * dv + j];"),
    ("final-state gradient ignored", "if (dS) memcpy(G, dS, SZ * sizeof(double));", ""),
    ("column scans read without the transpose",
     "const int r = (direction == 2 || direction == 3) ? (q % gh) * gw + q / gh : q;\n"
     "        memcpy(dst + (size_t)p * d, src + (size_t)r * d",
     "const int r = q;\n        memcpy(dst + (size_t)p * d, src + (size_t)r * d"),
]


def _run_pins(tmp, edit):
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(tmp, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    os.makedirs(os.path.join(tmp, "tests"))
    shutil.copy(os.path.abspath(__file__), os.path.join(tmp, "tests", "test_pins.py"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(tmp, "tests", "golden"))
    path = os.path.join(tmp, "oracle", "gla_backward.c")
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
