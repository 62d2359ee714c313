"""Pins for the oracle's extra operations, each against a result that does not
come from the oracle itself:

  * state carried in and out (ai.info summary, "Future Directions": carrying
    the state across frames):
      - an independent numpy quadratic form with the initial-state term,
        o_t = sum_{s<=t} (q~_t * exp(G_t - G_s)) . k_s v_s + (q~_t * exp(G_t)) S_0,
        S_N = diag(exp(G_N)) S_0 + sum_s diag(exp(G_N - G_s)) k_s^T v_s;
      - splitting the scan: the scan over a grid equals the scan over its
        first rows (columns for T->B) followed by the scan over the rest
        started from the first part's final state;
      - with k = 0 only the initial state is read out, decayed;
  * the output gate on the RMS-normalised output (ai.info summary,
    "Methodology in Plain English"): torch's rms_norm and silu in float64,
    scale invariance of the normalisation, constant rows, a zero gate;
  * Spatial SwiGLU's 3x3 depthwise convolution (same section; GTR project
    page, "Spatial SwiGLU"): torch's grouped conv2d in float64, a delta
    kernel, zero padding at the border.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from test_oracle_pins import rand_inputs, rel_err, scan_perm

pytestmark = pytest.mark.filterwarnings("ignore")


def brute_force_state(q, k, v, g, S0, H, W, direction):
    """Quadratic form with an initial state, one (b, h) slice at a time."""
    B, N, heads, dk = q.shape
    dv = v.shape[3]
    out = np.zeros((B, N, heads, dv))
    SN = np.zeros((B, heads, dk, dv))
    perm = scan_perm(direction, H, W)
    for b in range(B):
        for h in range(heads):
            Q = q[b, perm, h, :] / np.sqrt(dk)
            K, V = k[b, perm, h, :], v[b, perm, h, :]
            G = np.cumsum(g[b, perm, h, :], axis=0)
            for t in range(N):
                w = np.exp(G[t][None, :] - G[: t + 1])
                a = (Q[t][None, :] * w * K[: t + 1]).sum(axis=1)
                out[b, perm[t], h, :] = a @ V[: t + 1] + (Q[t] * np.exp(G[t])) @ S0[b, h]
            wN = np.exp(G[-1][None, :] - G)                      # (N, dk)
            SN[b, h] = np.exp(G[-1])[:, None] * S0[b, h] + (K * wN).T @ V
    return out, SN


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_state_in_and_out_matches_brute_force(oracle_mod, direction):
    H, W, heads, dk, dv = 5, 6, 2, 3, 5
    q, k, v, g = rand_inputs(2, H, W, heads, dk, dv, seed=40 + direction)
    g = g * 8.0
    S0 = np.random.default_rng(direction).standard_normal((2, heads, dk, dv))
    out, SN = oracle_mod.gla_serial_state(q, k, v, g, H, W, direction, S0)
    ref_out, ref_SN = brute_force_state(q, k, v, g, S0, H, W, direction)
    assert rel_err(out, ref_out) < 1e-12
    assert rel_err(SN, ref_SN) < 1e-12


def test_zero_initial_state_is_the_plain_recurrence(oracle_mod):
    q, k, v, g = rand_inputs(1, 6, 7, 2, 4, 6, seed=3)
    out, _ = oracle_mod.gla_serial_state(q, k, v, g, 6, 7, 2, None)
    out0, _ = oracle_mod.gla_serial_state(q, k, v, g, 6, 7, 2, np.zeros((1, 2, 4, 6)))
    plain = oracle_mod.gla_serial(q, k, v, g, 6, 7, 2)
    assert np.array_equal(out, plain) and np.array_equal(out0, plain)


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_split_scan_carries_the_state(oracle_mod, direction):
    """Scanning the whole grid equals scanning a prefix of the scan order and
    then the rest from the prefix's final state."""
    H, W, heads, dk, dv = 6, 5, 2, 4, 3
    q, k, v, g = rand_inputs(1, H, W, heads, dk, dv, seed=50 + direction)
    full, SN_full = oracle_mod.gla_serial_state(q, k, v, g, H, W, direction)

    def part(x, sl, hh, ww):  # [1, H*W, heads, d] -> sub-grid in row-major order
        d = x.shape[-1]
        return np.ascontiguousarray(x.reshape(1, H, W, heads, d)[:, sl[0], sl[1]].reshape(1, hh * ww, heads, d))

    if direction in (0, 1):  # row-major orders: split rows
        cut = 2
        first, second = (slice(0, cut), slice(None)), (slice(cut, H), slice(None))
        shp1, shp2 = (cut, W), (H - cut, W)
    else:                    # column-major orders: split columns
        cut = 2
        first, second = (slice(None), slice(0, cut)), (slice(None), slice(cut, W))
        shp1, shp2 = (H, cut), (H, W - cut)
    if direction in (1, 3):  # reversed orders visit the second part first
        first, second, shp1, shp2 = second, first, shp2, shp1
    X1 = [part(x, first, *shp1) for x in (q, k, v, g)]
    X2 = [part(x, second, *shp2) for x in (q, k, v, g)]
    o1, S1 = oracle_mod.gla_serial_state(*X1, shp1[0], shp1[1], direction)
    o2, S2 = oracle_mod.gla_serial_state(*X2, shp2[0], shp2[1], direction, S1)
    assert rel_err(o1, part(full, first, *shp1)) < 1e-12
    assert rel_err(o2, part(full, second, *shp2)) < 1e-12
    assert rel_err(S2, SN_full) < 1e-12


def test_initial_state_readout_with_no_keys(oracle_mod):
    """k = 0: the state never changes except by decay, o_t = q~_t exp(G_t) S_0."""
    H, W, heads, dk, dv = 4, 4, 1, 3, 2
    q, k, v, g = rand_inputs(1, H, W, heads, dk, dv, seed=9)
    k = np.zeros_like(k)
    S0 = np.arange(dk * dv, dtype=np.float64).reshape(1, 1, dk, dv) - 2.5
    out, SN = oracle_mod.gla_serial_state(q, k, v, g, H, W, 0, S0)
    G = np.cumsum(g[0, :, 0, :], axis=0)
    ref = (q[0, :, 0, :] / np.sqrt(dk) * np.exp(G)) @ S0[0, 0]
    assert rel_err(out[0, :, 0, :], ref) < 1e-13
    assert rel_err(SN[0, 0], np.exp(G[-1])[:, None] * S0[0, 0]) < 1e-13


def _gate_ref_torch(o, r, w, eps):
    ot, rt, wt = (torch.from_numpy(np.asarray(x, dtype=np.float64)) for x in (o, r, w))
    return (F.rms_norm(ot, (ot.shape[-1],), weight=wt, eps=eps) * F.silu(rt)).numpy()


@pytest.mark.parametrize("dv", [16, 64, 128])
def test_output_gate_matches_torch(oracle_mod, dv):
    rng = np.random.default_rng(dv)
    o = rng.standard_normal((3, 7, 2, dv)) * 0.3
    r = rng.standard_normal((3, 7, 2, dv)) * 2.0
    w = rng.standard_normal(dv)
    for eps in (1e-5, 1e-2):
        y = oracle_mod.output_gate(o, r, w, eps)
        assert rel_err(y, _gate_ref_torch(o, r, w, eps)) < 1e-13


def test_output_gate_closed_forms(oracle_mod):
    rng = np.random.default_rng(1)
    dv = 32
    o = rng.standard_normal((5, dv))
    r = rng.standard_normal((5, dv))
    w = rng.standard_normal(dv)
    # without eps the normalisation is scale invariant
    assert rel_err(oracle_mod.output_gate(7.5 * o, r, w, 0.0), oracle_mod.output_gate(o, r, w, 0.0)) < 1e-13
    # a constant row c: o / rms(o) = sign(c), so y = sign(c) w silu(r) (eps = 0)
    c = np.full((2, dv), -3.0)
    c[1] = 0.25
    y = oracle_mod.output_gate(c, r[:2], w, 0.0)
    silu = r[:2] / (1.0 + np.exp(-r[:2]))
    assert rel_err(y, np.sign(c) * w * silu) < 1e-14
    # a zero gate closes the output
    assert np.array_equal(oracle_mod.output_gate(o, np.zeros_like(r), w, 1e-5), np.zeros_like(o))


def _sswiglu_ref_torch(a, b, wc, bias, H, W):
    B, N, C = a.shape
    bt = torch.from_numpy(b).reshape(B, H, W, C).permute(0, 3, 1, 2)
    conv = F.conv2d(bt, torch.from_numpy(wc)[:, None], None if bias is None else torch.from_numpy(bias),
                    padding=1, groups=C)
    conv = conv.permute(0, 2, 3, 1).reshape(B, N, C)
    return (F.silu(torch.from_numpy(a)) * conv).numpy()


@pytest.mark.parametrize("H,W", [(1, 1), (1, 5), (4, 1), (5, 7)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_sswiglu_matches_torch_depthwise_conv(oracle_mod, H, W, with_bias):
    rng = np.random.default_rng(H * 10 + W)
    B, C = 2, 6
    a = rng.standard_normal((B, H * W, C))
    b = rng.standard_normal((B, H * W, C))
    wc = rng.standard_normal((C, 3, 3))
    bias = rng.standard_normal(C) if with_bias else None
    y = oracle_mod.sswiglu(a, b, wc, bias, H, W)
    assert rel_err(y, _sswiglu_ref_torch(a, b, wc, bias, H, W)) < 1e-13


def test_sswiglu_delta_kernel_and_padding(oracle_mod):
    rng = np.random.default_rng(2)
    B, H, W, C = 1, 4, 5, 3
    a = rng.standard_normal((B, H * W, C))
    b = rng.standard_normal((B, H * W, C))
    silu = a / (1.0 + np.exp(-a))
    delta = np.zeros((C, 3, 3))
    delta[:, 1, 1] = 1.0
    assert rel_err(oracle_mod.sswiglu(a, b, delta, None, H, W), silu * b) < 1e-15
    # a single value at the top-left corner reaches only its 2x2 neighbourhood
    b1 = np.zeros_like(b)
    b1[0, 0, :] = 1.0
    ones = np.ones((C, 3, 3))
    y = oracle_mod.sswiglu(np.full_like(a, 50.0), b1, ones, None, H, W).reshape(H, W, C)
    reach = np.zeros((H, W), dtype=bool)
    reach[:2, :2] = True
    assert np.allclose(y[reach], 50.0) and np.all(y[~reach] == 0.0)
