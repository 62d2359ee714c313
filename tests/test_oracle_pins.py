"""Pins for the fp64 oracle: checks against results fixed by the mathematics.

None of these re-types the oracle's recurrence.  Each check uses a different
route to the same number:
  * a brute-force quadratic form, o_t = sum_{s<=t} (q~_t * exp(G_t - G_s)) . k_s v_s,
    with G the inclusive prefix sum of the gates along the scan (the
    "parallel form" of gated linear attention, Yang et al., cited on the
    mlsanity index page of GTR);
  * closed forms: zero gates give causal linear attention (Katharopoulos et
    al., same reference list), a constant gate gives RetNet-style geometric
    weights (Sun et al., same list), closed gates give a memoryless readout;
  * invariants: a single token, linearity in v, homogeneity in q, chunk-size
    independence of the chunkwise schedule (GTR project page, "A Kernel That
    Makes Recurrence Fast": same state update, different schedule);
  * the four scan orders (ai.info summary, "Methodology in Plain English")
    built from numpy reshapes and reversals instead of the oracle's index
    arithmetic, and the equivariances between them.
Sizes use d_k != d_v so that a transposed operand cannot pass.
"""
import json
import os

import numpy as np
import pytest

from recurrent_vision_backbone_key_b200.synthetic import make_inputs

pytestmark = pytest.mark.filterwarnings("ignore")


def scan_perm(direction, H, W):
    """Row-major token index visited at each scan step, from numpy reshapes."""
    grid = np.arange(H * W).reshape(H, W)
    if direction == 0:
        return grid.reshape(-1)
    if direction == 1:
        return grid.reshape(-1)[::-1]
    if direction == 2:
        return grid.T.reshape(-1)
    if direction == 3:
        return grid.T.reshape(-1)[::-1]
    raise ValueError(direction)


def brute_force(q, k, v, g, H, W, direction):
    """Quadratic (parallel) form, one (b, h) slice at a time, in float64."""
    q, k, v, g = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g))
    B, N, heads, dk = q.shape
    out = np.zeros(v.shape)
    perm = scan_perm(direction, H, W)
    for b in range(B):
        for h in range(heads):
            Q = q[b, perm, h, :] / np.sqrt(dk)
            K = k[b, perm, h, :]
            V = v[b, perm, h, :]
            G = np.cumsum(g[b, perm, h, :], axis=0)
            O = np.zeros((N, v.shape[3]))
            for t in range(N):
                w = np.exp(G[t][None, :] - G[: t + 1])          # (t+1, dk)
                a = (Q[t][None, :] * w * K[: t + 1]).sum(axis=1)  # (t+1,)
                O[t] = a @ V[: t + 1]
            out[b, perm, h, :] = O
    return out


def rand_inputs(B, H, W, heads, dk, dv, seed, gate="mild"):
    q, k, v, g = make_inputs(B, H, W, heads, dk, dv, seed=seed, gate=gate)
    return (q.float().numpy().astype(np.float64), k.float().numpy().astype(np.float64),
            v.float().numpy().astype(np.float64), g.numpy().astype(np.float64))


def rel_err(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
@pytest.mark.parametrize("H,W", [(1, 1), (3, 5), (6, 4), (8, 8)])
def test_serial_matches_brute_force(oracle_mod, direction, H, W):
    q, k, v, g = rand_inputs(2, H, W, 2, 3, 5, seed=11 + direction)
    # widen the gate range so decay matters over a few tokens
    g = g * 8.0
    ref = brute_force(q, k, v, g, H, W, direction)
    out = oracle_mod.gla_serial(q, k, v, g, H, W, direction)
    assert rel_err(out, ref) < 1e-12


@pytest.mark.parametrize("direction", [0, 2])
def test_serial_brute_force_strong_decay(oracle_mod, direction):
    q, k, v, g = rand_inputs(1, 5, 7, 3, 4, 6, seed=5, gate="strong")
    ref = brute_force(q, k, v, g, 5, 7, direction)
    out = oracle_mod.gla_serial(q, k, v, g, 5, 7, direction)
    assert rel_err(out, ref) < 1e-12


def test_zero_gates_is_causal_linear_attention(oracle_mod):
    H, W, dk, dv = 4, 6, 5, 3
    q, k, v, _ = rand_inputs(2, H, W, 2, dk, dv, seed=3)
    g = np.zeros_like(q)
    out = oracle_mod.gla_serial(q, k, v, g, H, W, 0)
    for b in range(2):
        for h in range(2):
            Q, K, V = q[b, :, h] / np.sqrt(dk), k[b, :, h], v[b, :, h]
            ref = np.tril(Q @ K.T) @ V
            np.testing.assert_allclose(out[b, :, h], ref, rtol=1e-12, atol=1e-12)


def test_constant_gate_is_geometric_decay(oracle_mod):
    H, W, dk, dv = 3, 7, 4, 6
    c = -0.37
    q, k, v, _ = rand_inputs(1, H, W, 1, dk, dv, seed=4)
    g = np.full_like(q, c)
    out = oracle_mod.gla_serial(q, k, v, g, H, W, 0)
    N = H * W
    t = np.arange(N)
    D = np.where(t[:, None] >= t[None, :], np.exp(c * (t[:, None] - t[None, :])), 0.0)
    Q, K, V = q[0, :, 0] / np.sqrt(dk), k[0, :, 0], v[0, :, 0]
    ref = ((Q @ K.T) * D) @ V
    np.testing.assert_allclose(out[0, :, 0], ref, rtol=1e-12, atol=1e-12)


def test_closed_gates_are_memoryless(oracle_mod):
    H, W, dk, dv = 5, 5, 3, 4
    q, k, v, _ = rand_inputs(1, H, W, 2, dk, dv, seed=6)
    g = np.full_like(q, -np.inf)
    for direction in range(4):
        out = oracle_mod.gla_serial(q, k, v, g, H, W, direction)
        ref = ((q / np.sqrt(dk)) * k).sum(-1, keepdims=True) * v
        np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-14)


def test_single_token(oracle_mod):
    q, k, v, g = rand_inputs(3, 1, 1, 2, 7, 2, seed=8)
    out = oracle_mod.gla_serial(q, k, v, g, 1, 1, 0)
    ref = ((q / np.sqrt(7)) * k).sum(-1, keepdims=True) * v
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-14)


def test_linearity_and_homogeneity(oracle_mod):
    H, W = 4, 5
    q, k, v1, g = rand_inputs(1, H, W, 2, 3, 4, seed=9)
    _, _, v2, _ = rand_inputs(1, H, W, 2, 3, 4, seed=10)
    f = lambda qq, vv: oracle_mod.gla_serial(qq, k, vv, g, H, W, 2)
    np.testing.assert_allclose(f(q, 2.5 * v1 - 0.75 * v2), 2.5 * f(q, v1) - 0.75 * f(q, v2),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(f(-3.0 * q, v1), -3.0 * f(q, v1), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
@pytest.mark.parametrize("direction", [0, 3])
def test_chunked_equals_serial(oracle_mod, chunk, direction):
    # 7 x 9 = 63 tokens: a ragged last chunk for every chunk size but 1
    H, W = 7, 9
    q, k, v, g = rand_inputs(2, H, W, 2, 5, 3, seed=20 + chunk)
    ref = oracle_mod.gla_serial(q, k, v, g, H, W, direction)
    out, dS, gamma, S_enter = oracle_mod.gla_chunked(q, k, v, g, H, W, direction, chunk)
    assert rel_err(out, ref) < 1e-12


def test_chunked_strong_decay_equals_serial(oracle_mod):
    H, W = 9, 10
    q, k, v, g = rand_inputs(1, H, W, 2, 6, 4, seed=31, gate="strong")
    ref = oracle_mod.gla_serial(q, k, v, g, H, W, 1)
    out, *_ = oracle_mod.gla_chunked(q, k, v, g, H, W, 1, 16)
    assert rel_err(out, ref) < 1e-12


@pytest.mark.parametrize("chunk", [4, 16])
def test_chunk_intermediates(oracle_mod, chunk):
    """S_enter equals the serial state at chunk boundaries; dS_c is the state
    reached from zero over chunk c alone; gamma_c the product of the gates."""
    H, W, dk, dv = 5, 7, 3, 4
    q, k, v, g = rand_inputs(1, H, W, 2, dk, dv, seed=40)
    direction = 2
    out, states = oracle_mod.gla_serial(q, k, v, g, H, W, direction, chunk=chunk,
                                        return_states=True)
    _, dS, gamma, S_enter = oracle_mod.gla_chunked(q, k, v, g, H, W, direction, chunk)
    nc = dS.shape[2]
    np.testing.assert_allclose(S_enter, states[:, :, :nc], rtol=1e-12, atol=1e-13)
    perm = scan_perm(direction, H, W)
    N = H * W
    for h in range(2):
        for c in range(nc):
            toks = perm[c * chunk: min(N, (c + 1) * chunk)]
            # dS_c: recurrence over this chunk alone from a zero state, done as
            # a product of per-token decays (not as an exp of a prefix sum)
            S = np.zeros((dk, dv))
            for p in toks:
                S = np.exp(g[0, p, h])[:, None] * S + np.outer(k[0, p, h], v[0, p, h])
            np.testing.assert_allclose(dS[0, h, c], S, rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(gamma[0, h, c], np.prod(np.exp(g[0, toks, h]), axis=0),
                                       rtol=1e-12)


def test_scan_index_bijection_and_definition(oracle_mod):
    for H, W in [(1, 1), (1, 7), (6, 1), (3, 5), (8, 8), (40, 40)]:
        N = H * W
        for d in range(4):
            seq = np.array([oracle_mod.scan_index(d, t, H, W) for t in range(N)])
            np.testing.assert_array_equal(np.sort(seq), np.arange(N))
            np.testing.assert_array_equal(seq, scan_perm(d, H, W))


@pytest.mark.parametrize("H,W", [(3, 5), (6, 4)])
def test_direction_equivariances(oracle_mod, H, W):
    """R->L is L->R on the 180-degree-rotated grid, T->B is L->R on the
    transposed grid, B->T is T->B on the rotated grid."""
    q, k, v, g = rand_inputs(1, H, W, 2, 3, 4, seed=50)
    f = lambda d, X, h, w: oracle_mod.gla_serial(*X, h, w, d)
    X = (q, k, v, g)
    rot = lambda a: a[:, ::-1]
    tr = lambda a, h, w: a.reshape(a.shape[0], h, w, *a.shape[2:]).transpose(0, 2, 1, 3, 4).reshape(a.shape)
    # R->L
    np.testing.assert_allclose(f(1, X, H, W), rot(f(0, tuple(rot(a) for a in X), H, W)),
                               rtol=1e-12, atol=1e-13)
    # T->B on H x W == transpose back of L->R on the W x H transposed grid
    Xt = tuple(tr(a, H, W) for a in X)
    o_t2b = f(2, X, H, W)
    np.testing.assert_allclose(o_t2b, tr(f(0, Xt, W, H), W, H), rtol=1e-12, atol=1e-13)
    # B->T == rotate of T->B on rotated inputs
    np.testing.assert_allclose(f(3, X, H, W), rot(f(2, tuple(rot(a) for a in X), H, W)),
                               rtol=1e-12, atol=1e-13)


def test_golden_regression(oracle_mod):
    """The oracle still reproduces the values its committed generator wrote."""
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")
    with open(path) as f:
        gold = json.load(f)
    w = gold["workload"]
    q, k, v, g = make_inputs(w["B"], w["grid_h"], w["grid_w"], w["heads"], w["d_k"], w["d_v"],
                             seed=w["seed"], gate=w["gate"])
    for key, direction in (("l2r", 0), ("t2b", 2)):
        out = oracle_mod.gla_serial(q, k, v, g, w["grid_h"], w["grid_w"], direction)
        ref = np.array(gold[key]).reshape(out.shape)
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-15)
