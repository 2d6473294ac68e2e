"""Pins for the fp64 oracle, each independent of the oracle's own code.

The oracle (oracle/gla_oracle.c) runs the token-by-token recurrence of GTR's
gated linear attention ("GTR: Gated Token Recurrence for Efficient Dense
Prediction", x-techcon article, section 架构) with the scan directions built
by explicit transposes/reversals.  Nothing on the pages prints tensors for
this operator, so it is pinned here against what the mathematics fixes:

* a hand-worked 2x2-grid example (tests/golden/hand_2x2.json), all 4 scans;
* the brute-force quadratic form with an explicit product loop over gates
  and scan orders built from index formulas (not from the oracle's copies);
* the all-gates-one special case = causal linear attention tril(QK^T)V;
* the chunkwise reorganisation (section 算子) at many chunk sizes;
* the flip identities R->L(X) = flip(L->R(flip X)), B->T(X) = flip(T->B(flip X));
* memoryless gates, a single token, the scalar recurrence, the transpose
  identity, and linearity in v.

d_k != d_v wherever possible, so a transposed operand cannot pass.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def scan_order(gh: int, gw: int, direction: int):
    """Raster index of each scan position, from the index formulas."""
    n = gh * gw
    order = []
    for p in range(n):
        pp = n - 1 - p if direction in (1, 3) else p
        if direction in (0, 1):
            r = pp
        else:
            y, x = pp % gh, pp // gh
            r = y * gw + x
        order.append(r)
    return order


def rand_case(rng, B, H, gh, gw, dk, dv, gate_scale=1.0):
    q = rng.standard_normal((B, H, gh, gw, dk))
    k = rng.standard_normal((B, H, gh, gw, dk))
    v = rng.standard_normal((B, H, gh, gw, dv))
    la = -gate_scale * rng.exponential(1.0, (B, H, gh, gw, dk))
    return q, k, v, la


def brute_plane(q, k, v, la, order):
    """o_t = sum_{s<=t} q_t diag(prod_{u=s+1..t} alpha_u) k_s^T v_s, explicit loops.

    q,k,la: [N, dk]; v: [N, dv] in raster order; order: scan -> raster."""
    n = len(order)
    dk, dv = q.shape[1], v.shape[1]
    alpha = np.exp(la)
    out = np.zeros((n, dv))
    for ti in range(n):
        t = order[ti]
        acc = np.zeros(dv)
        for si in range(ti + 1):
            s = order[si]
            decay = np.ones(dk)
            for ui in range(si + 1, ti + 1):
                decay = decay * alpha[order[ui]]
            acc += float(np.sum(q[t] * decay * k[s])) * v[s]
        out[t] = acc
    final = np.zeros((dk, dv))
    for si in range(n):
        s = order[si]
        decay = np.ones(dk)
        for ui in range(si + 1, n):
            decay = decay * alpha[order[ui]]
        final += np.outer(decay * k[s], v[s])
    return out, final


def rel(a, b):
    d = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (d if d > 0 else 1.0))


# ---------------------------------------------------------------- golden


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_hand_worked_2x2(direction):
    g = json.load(open(os.path.join(GOLDEN, "hand_2x2.json")))
    gh, gw = g["grid"]
    q = np.array(g["q"], float).reshape(1, 1, gh, gw, g["d_k"])
    k = np.array(g["k"], float).reshape(1, 1, gh, gw, g["d_k"])
    v = np.array(g["v"], float).reshape(1, 1, gh, gw, g["d_v"])
    la = np.log(np.array(g["alpha"], float)).reshape(1, 1, gh, gw, g["d_k"])
    exp = g["expected"][str(direction)]
    assert scan_order(gh, gw, direction) == exp["scan_order"]
    out, fs = oracle.forward(q, k, v, la, direction)
    np.testing.assert_allclose(out.reshape(-1), np.array(exp["out"], float), rtol=1e-14, atol=1e-13)
    np.testing.assert_allclose(fs.reshape(-1), np.array(exp["final_state"], float).reshape(-1),
                               rtol=1e-14, atol=1e-13)


# ---------------------------------------------------------------- C1 brute force


@pytest.mark.parametrize("grid", [(2, 3), (3, 2), (4, 4), (5, 7)])
@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_brute_force_quadratic_form(grid, direction):
    rng = np.random.default_rng(100 + 10 * direction + grid[0] * grid[1])
    gh, gw = grid
    q, k, v, la = rand_case(rng, 1, 2, gh, gw, 5, 3, gate_scale=0.7)
    out, fs = oracle.forward(q, k, v, la, direction)
    order = scan_order(gh, gw, direction)
    for h in range(2):
        n = gh * gw
        ref, ref_fs = brute_plane(q[0, h].reshape(n, 5), k[0, h].reshape(n, 5),
                                  v[0, h].reshape(n, 3), la[0, h].reshape(n, 5), order)
        assert rel(out[0, h].reshape(n, 3), ref) < 1e-12
        assert rel(fs[0, h], ref_fs) < 1e-12


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_brute_force_16x16_prefix_logs(direction):
    """16x16 grid, d=64: closed form with gate products from prefix sums of logs."""
    rng = np.random.default_rng(7 + direction)
    gh = gw = 16
    dk, dv = 64, 48
    q, k, v, la = rand_case(rng, 1, 1, gh, gw, dk, dv, gate_scale=1.0 / 16)
    out, fs = oracle.forward(q, k, v, la, direction)
    n = gh * gw
    order = np.array(scan_order(gh, gw, direction))
    Q = q[0, 0].reshape(n, dk)[order]
    K = k[0, 0].reshape(n, dk)[order]
    V = v[0, 0].reshape(n, dv)[order]
    c = np.cumsum(la[0, 0].reshape(n, dk)[order], axis=0)  # c_t = sum_{u<=t} log a_u
    ref = np.zeros((n, dv))
    for t in range(n):
        w = np.exp(c[t][None, :] - c[: t + 1])  # prod_{u=s+1..t} alpha_u, s<=t
        a = np.sum(Q[t][None, :] * w * K[: t + 1], axis=1)
        ref[t] = a @ V[: t + 1]
    got = out[0, 0].reshape(n, dv)[order]
    assert rel(got, ref) < 1e-12
    wf = np.exp(c[-1][None, :] - c)
    assert rel(fs[0, 0], (wf * K).T @ V) < 1e-12


# ---------------------------------------------------------------- C2 gates = 1


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_all_gates_one_is_causal_linear_attention(direction):
    rng = np.random.default_rng(3)
    gh, gw, dk, dv = 6, 9, 16, 24
    q, k, v, _ = rand_case(rng, 2, 1, gh, gw, dk, dv)
    la = np.zeros_like(q)
    out, fs = oracle.forward(q, k, v, la, direction)
    n = gh * gw
    order = np.array(scan_order(gh, gw, direction))
    for b in range(2):
        Q = q[b, 0].reshape(n, dk)[order]
        K = k[b, 0].reshape(n, dk)[order]
        V = v[b, 0].reshape(n, dv)[order]
        ref = np.tril(Q @ K.T) @ V
        assert rel(out[b, 0].reshape(n, dv)[order], ref) < 1e-12
        assert rel(fs[b, 0], K.T @ V) < 1e-12


# ---------------------------------------------------------------- C3 chunk invariance


@pytest.mark.parametrize("chunk", [1, 7, 16, 32, 48, 64, 128, 256])
@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_chunkwise_equals_recurrence(chunk, direction):
    rng = np.random.default_rng(11)
    q, k, v, la = rand_case(rng, 1, 2, 16, 16, 24, 20, gate_scale=0.25)
    out, fs = oracle.forward(q, k, v, la, direction)
    oc, fc = oracle.chunkwise(q, k, v, la, direction, chunk)
    assert rel(oc, out) < 1e-11
    assert rel(fc, fs) < 1e-11


def test_chunkwise_ragged_tail_strong_gates():
    """N = 40*40 = 1600 is not a multiple of 128: the last chunk is partial."""
    rng = np.random.default_rng(12)
    q, k, v, la = rand_case(rng, 1, 1, 40, 40, 8, 8, gate_scale=2.0)
    for direction in range(4):
        out, fs = oracle.forward(q, k, v, la, direction)
        oc, fc = oracle.chunkwise(q, k, v, la, direction, 128)
        assert rel(oc, out) < 1e-11
        assert rel(fc, fs) < 1e-11


# ---------------------------------------------------------------- C4 flips


def flip(x):
    """Reverse the whole token sequence of the raster (the grid turned 180 deg)."""
    return np.ascontiguousarray(x[:, :, ::-1, ::-1, :])


@pytest.mark.parametrize("grid", [(5, 7), (16, 16), (3, 1), (1, 6)])
def test_flip_identities(grid):
    rng = np.random.default_rng(21)
    gh, gw = grid
    q, k, v, la = rand_case(rng, 2, 2, gh, gw, 6, 4, gate_scale=0.5)
    for fwd_dir, rev_dir in ((0, 1), (2, 3)):
        o_rev, f_rev = oracle.forward(q, k, v, la, rev_dir)
        o_f, f_f = oracle.forward(flip(q), flip(k), flip(v), flip(la), fwd_dir)
        assert rel(o_rev, flip(o_f)) < 1e-14
        assert rel(f_rev, f_f) < 1e-14


def test_reverse_is_not_row_reversal():
    """R->L is the full reversal, not a per-row mirror with rows kept in order."""
    rng = np.random.default_rng(22)
    q, k, v, la = rand_case(rng, 1, 1, 4, 5, 3, 3, gate_scale=0.3)
    o1, _ = oracle.forward(q, k, v, la, 1)
    mirrored = lambda x: np.ascontiguousarray(x[:, :, :, ::-1, :])
    o_m, _ = oracle.forward(mirrored(q), mirrored(k), mirrored(v), mirrored(la), 0)
    assert rel(o1, mirrored(o_m)) > 1e-3


# ---------------------------------------------------------------- C5 extras


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_memoryless_gates(direction):
    rng = np.random.default_rng(31)
    q, k, v, _ = rand_case(rng, 1, 1, 7, 5, 8, 6)
    la = np.full_like(q, -80.0)
    out, fs = oracle.forward(q, k, v, la, direction)
    ref = np.sum(q * k, axis=-1, keepdims=True) * v
    assert rel(out, ref) < 1e-12
    last = scan_order(7, 5, direction)[-1]
    kk, vv = k[0, 0].reshape(35, 8)[last], v[0, 0].reshape(35, 6)[last]
    assert rel(fs[0, 0], np.outer(kk, vv)) < 1e-12


def test_single_token():
    rng = np.random.default_rng(32)
    q, k, v, la = rand_case(rng, 3, 2, 1, 1, 5, 7)
    for direction in range(4):
        out, fs = oracle.forward(q, k, v, la, direction)
        ref = np.sum(q * k, axis=-1, keepdims=True) * v
        assert rel(out, ref) < 1e-14
        assert rel(fs, np.einsum("bhyxi,bhyxj->bhij", k, v)) < 1e-14


def test_scalar_recurrence_closed_form():
    rng = np.random.default_rng(33)
    gh, gw = 8, 9
    q, k, v, la = rand_case(rng, 1, 1, gh, gw, 1, 1, gate_scale=0.4)
    out, fs = oracle.forward(q, k, v, la, 0)
    n = gh * gw
    qq, kk, vv, ll = (x.reshape(n) for x in (q, k, v, la))
    c = np.cumsum(ll)
    ref = np.array([qq[t] * np.sum(np.exp(c[t] - c[: t + 1]) * kk[: t + 1] * vv[: t + 1])
                    for t in range(n)])
    assert rel(out.reshape(n), ref) < 1e-12


@pytest.mark.parametrize("rev", [False, True])
def test_column_scan_is_row_scan_of_transpose(rev):
    rng = np.random.default_rng(34)
    q, k, v, la = rand_case(rng, 1, 2, 5, 8, 4, 3, gate_scale=0.3)
    tr = lambda x: np.ascontiguousarray(np.swapaxes(x, 2, 3))
    o_col, f_col = oracle.forward(q, k, v, la, 3 if rev else 2)
    o_row, f_row = oracle.forward(tr(q), tr(k), tr(v), tr(la), 1 if rev else 0)
    assert rel(o_col, tr(o_row)) < 1e-14
    assert rel(f_col, f_row) < 1e-14


def test_linear_in_v_and_q():
    rng = np.random.default_rng(35)
    q, k, v, la = rand_case(rng, 1, 1, 6, 6, 5, 4, gate_scale=0.5)
    v2 = rng.standard_normal(v.shape)
    o1, f1 = oracle.forward(q, k, v, la, 2)
    o2, f2 = oracle.forward(q, k, v2, la, 2)
    o12, f12 = oracle.forward(3.0 * q, k, v + v2, la, 2)
    assert rel(o12, 3.0 * (o1 + o2)) < 1e-13
    assert rel(f12, f1 + f2) < 1e-13


def test_argument_errors():
    z = np.zeros((1, 1, 2, 2, 3))
    with pytest.raises(ValueError):
        oracle.forward(z, z, z, z, 4)
    with pytest.raises(ValueError):
        oracle.forward(z, z[..., :2], z, z, 0)
