"""GPU parity of the state-carrying and the gated forward against the oracle.

  * gtr_gla_forward_state: the recurrence from a given S_0, with the final
    state S_N returned (ai.info summary, "Future Directions": carrying the
    state across frames).  Outputs at the forward's bar, max |o_gpu - o_ref|
    <= 2e-3 max |o_ref|; the final state at the same relative bar, the bound
    the chunk summaries and boundary states of the three-phase schedule are
    held to (fp16 rounding of the decay-scaled key operand, fp32
    accumulation).
  * gtr_gla_forward_gated: the output gate on the RMS-normalised output
    (same page, "Methodology in Plain English"), against the oracle's gate
    applied to the oracle's fp64 output.  Bound: 5e-3 max |y_ref|.  The gate
    divides each row by its own rms, so a row's error relative to its rms is
    what carries over: at most the forward's 2e-3 for the numerator, as much
    again through the rms itself, plus one fp16 rounding of the result
    (2^-11 ~ 4.9e-4); 2 * 2e-3 + 4.9e-4 < 5e-3.
  * gtr_gla_forward_bf16: bf16 q, k, v and out (ai.info summary, "Future
    Directions": other precisions), at the bar scaled by the ratio of unit
    roundoffs (BF16_TOL below), and the pages' deployment shape d_k = 32,
    d_v = 64 at the batched size.
"""
import numpy as np
import pytest
import torch

from recurrent_vision_backbone_key_b200 import gtr_gla
from recurrent_vision_backbone_key_b200.synthetic import make_inputs
from gpu_util import compare, gpu_inputs

pytestmark = pytest.mark.gpu

GATE_TOL = 5e-3
WALK_SHAPES = [(32, 64), (64, 64), (128, 128), (64, 128), (128, 64)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gtr_gla.load()


def _state(B, heads, dk, dv, seed, scale=1.0):
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn((B, heads, dk, dv), generator=gen, dtype=torch.float64) * scale).float()


def run_state(q, k, v, g, S0, H, W, direction, want_sn=True):
    B, N, heads, dk = q.shape
    dv = v.shape[3]
    out = torch.full_like(v, float("nan"))
    SN = torch.full((B, heads, dk, dv), float("nan"), device="cuda") if want_sn else None
    gtr_gla.check(gtr_gla.gtr_gla_forward_state(q, k, v, g, S0, B, heads, H, W, dk, dv, direction, 64, out, SN))
    torch.cuda.synchronize()
    return out, SN


@pytest.mark.parametrize("dk,dv", WALK_SHAPES)
def test_state_in_and_out_against_oracle(oracle_mod, dk, dv):
    for (B, H, W, heads) in [(2, 7, 19, 3), (1, 16, 16, 2)]:
        q, k, v, g = gpu_inputs(B, H, W, heads, dk, dv, seed=dk + dv + H)
        S0 = _state(B, heads, dk, dv, seed=H, scale=0.5)
        for direction in range(4):
            out, SN = run_state(q, k, v, g, S0.cuda(), H, W, direction)
            ref_out, ref_SN = oracle_mod.gla_serial_state(q.cpu(), k.cpu(), v.cpu(), g.cpu(), H, W, direction,
                                                          S0.double().numpy())
            compare(out, ref_out)
            compare(SN, ref_SN)


def test_state_chained_calls_equal_one_call(oracle_mod):
    """Two calls over the top and bottom halves of a grid (L->R), the second
    started from the first one's final state, give the single call's
    outputs and final state; also the oracle's."""
    B, H, W, heads, dk, dv = 2, 24, 20, 4, 64, 64
    q, k, v, g = gpu_inputs(B, H, W, heads, dk, dv, seed=5)
    full, SN_full = run_state(q, k, v, g, None, H, W, 0)
    half = H // 2 * W
    top = [x[:, :half].contiguous() for x in (q, k, v, g)]
    bot = [x[:, half:].contiguous() for x in (q, k, v, g)]
    o1, S1 = run_state(*top, None, H // 2, W, 0)
    o2, S2 = run_state(*bot, S1, H - H // 2, W, 0)
    compare(torch.cat([o1, o2], dim=1), full.float().cpu().numpy())
    compare(S2, SN_full.double().cpu().numpy())
    ref_out, ref_SN = oracle_mod.gla_serial_state(q.cpu(), k.cpu(), v.cpu(), g.cpu(), H, W, 0)
    compare(torch.cat([o1, o2], dim=1), ref_out)
    compare(S2, ref_SN)


def test_state_in_place_and_null(oracle_mod):
    B, H, W, heads, dk, dv = 2, 9, 11, 3, 128, 128
    q, k, v, g = gpu_inputs(B, H, W, heads, dk, dv, seed=8)
    S0 = _state(B, heads, dk, dv, seed=1)
    buf = S0.cuda()
    out = torch.empty_like(v)
    gtr_gla.check(gtr_gla.gtr_gla_forward_state(q, k, v, g, buf, B, heads, H, W, dk, dv, 2, 64, out, buf))
    torch.cuda.synchronize()
    ref_out, ref_SN = oracle_mod.gla_serial_state(q.cpu(), k.cpu(), v.cpu(), g.cpu(), H, W, 2, S0.double().numpy())
    compare(out, ref_out)
    compare(buf, ref_SN)
    # no initial and no final state: the plain walk, bit for bit
    o0, _ = run_state(q, k, v, g, None, H, W, 2, want_sn=False)
    plain = gtr_gla.forward(q, k, v, g, H, W, direction=2, chunk=64, schedule="walk_tcgen05")
    torch.cuda.synchronize()
    assert torch.equal(o0, plain)


def test_state_empty_grid_copies_the_state():
    B, heads, dk, dv = 2, 3, 64, 64
    S0 = _state(B, heads, dk, dv, seed=3).cuda()
    SN = torch.zeros_like(S0)
    z = torch.empty((B, 0, heads, dk), dtype=torch.float16, device="cuda")
    zg = torch.empty((B, 0, heads, dk), dtype=torch.float32, device="cuda")
    zo = torch.empty((B, 0, heads, dv), dtype=torch.float16, device="cuda")
    # empty tensors may share a null data pointer: use distinct dummies
    dummy = [torch.empty(16, dtype=torch.float32, device="cuda") for _ in range(5)]
    st = gtr_gla.gtr_gla_forward_state(dummy[0], dummy[1], dummy[2], dummy[3], S0, B, heads, 0, 7, dk, dv, 0,
                                       64, dummy[4], SN)
    assert st == 0, gtr_gla.last_error()
    torch.cuda.synchronize()
    assert torch.equal(SN, S0)
    del z, zg, zo


def gate_inputs(B, N, heads, dv, seed):
    gen = torch.Generator().manual_seed(seed)
    r = (torch.randn((B, N, heads, dv), generator=gen) * 2.0).half()
    w = (1.0 + 0.2 * torch.randn(dv, generator=gen)).float()
    return r, w


@pytest.mark.parametrize("dk", [32, 64, 128])
@pytest.mark.parametrize("gate_kind", ["mild", "strong"])
def test_gated_against_oracle(oracle_mod, dk, gate_kind):
    dv, eps = 64, 1e-5
    for (B, H, W, heads) in [(2, 7, 19, 3), (1, 20, 20, 2)]:
        q, k, v, g = gpu_inputs(B, H, W, heads, dk, dv, seed=dk + H, gate=gate_kind)
        r, w = gate_inputs(B, H * W, heads, dv, seed=H)
        for direction in range(4):
            out = torch.full_like(v, float("nan"))
            gtr_gla.check(gtr_gla.gtr_gla_forward_gated(q, k, v, g, r.cuda(), w.cuda(), eps, B, heads, H, W, dk,
                                                        dv, direction, 64, out))
            torch.cuda.synchronize()
            o_ref = oracle_mod.gla_serial(q.cpu(), k.cpu(), v.cpu(), g.cpu(), H, W, direction)
            y_ref = oracle_mod.output_gate(o_ref, r, w, eps)
            compare(out, y_ref, tol=GATE_TOL)


def test_gated_full_size_sampled(oracle_mod):
    """The batched shape (B32, 40x40, 12 heads, d = 64) through the gated
    call, 24 sampled sequences against the oracle."""
    B, H, W, heads, d = 32, 40, 40, 12, 64
    q, k, v, g = make_inputs(B, H, W, heads, d, d, seed=12, device="cuda")
    r, w = gate_inputs(B, H * W, heads, d, seed=12)
    r, w = r.cuda(), w.cuda()
    out = torch.empty_like(v)
    gtr_gla.check(gtr_gla.gtr_gla_forward_gated(q, k, v, g, r, w, 1e-5, B, heads, H, W, d, d, 2, 64, out))
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    picks = {(0, 0), (B - 1, heads - 1)}
    while len(picks) < 24:
        picks.add((int(rng.integers(B)), int(rng.integers(heads))))
    for b, h in sorted(picks):
        sl = lambda x: x[b:b + 1, :, h:h + 1, :].cpu()
        o_ref = oracle_mod.gla_serial(sl(q), sl(k), sl(v), sl(g), H, W, 2)
        compare(out[b:b + 1, :, h:h + 1, :], oracle_mod.output_gate(o_ref, sl(r), w.cpu(), 1e-5), tol=GATE_TOL)


def test_state_and_gate_reject_unsupported():
    q, k, v, g = gpu_inputs(1, 4, 4, 1, 16, 16, seed=1)
    out = torch.empty_like(v)
    assert gtr_gla.gtr_gla_forward_state(q, k, v, g, None, 1, 1, 4, 4, 16, 16, 0, 64, out, None) == 2
    q, k, v, g = gpu_inputs(1, 4, 4, 1, 64, 128, seed=1)
    out = torch.empty_like(v)
    r = torch.zeros_like(v)
    w = torch.ones(128, device="cuda")
    assert gtr_gla.gtr_gla_forward_gated(q, k, v, g, r, w, 1e-5, 1, 1, 4, 4, 64, 128, 0, 64, out) == 2
    assert "d_v = 64" in gtr_gla.last_error()


# bf16 I/O: the forward's bar scaled from fp16 to bf16 unit roundoff.  The
# fp16 bar, 2e-3 of max |o_ref|, is about 4 units of fp16 roundoff (2^-11);
# bf16 rounds 8 times coarser (2^-8 against 2^-11), so the same number of
# units is 8 * 2e-3 = 1.6e-2 of max |o_ref|.
BF16_TOL = 1.6e-2


@pytest.mark.parametrize("dk,dv", WALK_SHAPES)
def test_bf16_against_oracle(oracle_mod, dk, dv):
    for (B, H, W, heads) in [(2, 7, 19, 3), (1, 16, 24, 2)]:
        q, k, v, g = make_inputs(B, H, W, heads, dk, dv, seed=dk + dv + W, dtype=torch.bfloat16)
        qd, kd, vd, gd = (x.cuda() for x in (q, k, v, g))
        for direction in range(4):
            out = torch.full_like(vd, float("nan"))
            gtr_gla.check(gtr_gla.gtr_gla_forward_bf16(qd, kd, vd, gd, B, heads, H, W, dk, dv, direction, 64, out))
            torch.cuda.synchronize()
            compare(out, oracle_mod.gla_serial(q, k, v, g, H, W, direction), tol=BF16_TOL)


def test_bf16_special_gates(oracle_mod):
    B, H, W, heads, dk, dv = 2, 10, 13, 2, 64, 64
    q, k, v, g = make_inputs(B, H, W, heads, dk, dv, seed=3, dtype=torch.bfloat16)
    cases = {"open": torch.zeros_like(g), "closed": torch.full_like(g, -1.0e4),
             "strong": make_inputs(B, H, W, heads, dk, dv, seed=3, gate="strong")[3]}
    for name, gg in cases.items():
        out = torch.empty_like(v).cuda()
        gtr_gla.check(gtr_gla.gtr_gla_forward_bf16(q.cuda(), k.cuda(), v.cuda(), gg.cuda(), B, heads, H, W, dk, dv,
                                                   2, 64, out))
        torch.cuda.synchronize()
        compare(out, oracle_mod.gla_serial(q, k, v, gg, H, W, 2), tol=BF16_TOL)


def test_deployment_shape_full_size_sampled(oracle_mod):
    """The pages' deployment shape (d_k = 32, d_v = 64, chunk 64) at the
    batched size, fp16 through AUTO and bf16, 24 sampled sequences each."""
    from recurrent_vision_backbone_key_b200.synthetic import WORKLOADS, make_workload_inputs
    w = WORKLOADS["deploy_batched"]
    for dtype, tol in ((torch.float16, 2e-3), (torch.bfloat16, BF16_TOL)):
        q, k, v, g = make_workload_inputs(w, seed=5, device="cuda", dtype=dtype)
        out = torch.empty_like(v)
        if dtype == torch.float16:
            gtr_gla.check(gtr_gla.gtr_gla_forward(q, k, v, g, w.B, w.heads, w.grid_h, w.grid_w, w.d_k, w.d_v, 2,
                                                  64, out))
        else:
            gtr_gla.check(gtr_gla.gtr_gla_forward_bf16(q, k, v, g, w.B, w.heads, w.grid_h, w.grid_w, w.d_k, w.d_v,
                                                       2, 64, out))
        torch.cuda.synchronize()
        rng = np.random.default_rng(1)
        picks = {(0, 0), (w.B - 1, w.heads - 1)}
        while len(picks) < 24:
            picks.add((int(rng.integers(w.B)), int(rng.integers(w.heads))))
        for b, h in sorted(picks):
            sl = lambda x: x[b:b + 1, :, h:h + 1, :].cpu()
            compare(out[b:b + 1, :, h:h + 1, :], oracle_mod.gla_serial(sl(q), sl(k), sl(v), sl(g), w.grid_h,
                                                                       w.grid_w, 2), tol=tol)


def _picks(B, heads, n, seed):
    rng = np.random.default_rng(seed)
    picks = {(0, 0), (B - 1, heads - 1)}
    while len(picks) < n:
        picks.add((int(rng.integers(B)), int(rng.integers(heads))))
    return sorted(picks)


def test_bf16_batched_full_size_sampled(oracle_mod):
    """bf16 I/O at the batched size (d = 64, the launch the bf16 bench line
    times), L->R and T->B, 24 sampled sequences each."""
    from recurrent_vision_backbone_key_b200.synthetic import WORKLOADS, make_workload_inputs
    w = WORKLOADS["batched"]
    q, k, v, g = make_workload_inputs(w, seed=6, device="cuda", dtype=torch.bfloat16)
    out = torch.empty_like(v)
    for direction in (0, 2):
        gtr_gla.check(gtr_gla.gtr_gla_forward_bf16(q, k, v, g, w.B, w.heads, w.grid_h, w.grid_w, w.d_k, w.d_v,
                                                   direction, 64, out))
        torch.cuda.synchronize()
        for b, h in _picks(w.B, w.heads, 24, seed=direction + 11):
            sl = lambda x: x[b:b + 1, :, h:h + 1, :].cpu()
            compare(out[b:b + 1, :, h:h + 1, :], oracle_mod.gla_serial(sl(q), sl(k), sl(v), sl(g), w.grid_h,
                                                                       w.grid_w, direction), tol=BF16_TOL)


def test_state_batched_full_size_sampled(oracle_mod):
    """State in and out at the batched size (the launch the state bench line
    times), T->B, 24 sampled sequences: outputs and final states."""
    from recurrent_vision_backbone_key_b200.synthetic import WORKLOADS, make_workload_inputs
    w = WORKLOADS["batched"]
    q, k, v, g = make_workload_inputs(w, seed=8, device="cuda")
    S0 = _state(w.B, w.heads, w.d_k, w.d_v, seed=9, scale=0.5)
    out, SN = run_state(q, k, v, g, S0.cuda(), w.grid_h, w.grid_w, 2)
    for b, h in _picks(w.B, w.heads, 24, seed=13):
        sl = lambda x: x[b:b + 1, :, h:h + 1, :].cpu()
        ref_out, ref_SN = oracle_mod.gla_serial_state(sl(q), sl(k), sl(v), sl(g), w.grid_h, w.grid_w, 2,
                                                      S0[b:b + 1, h:h + 1].double().numpy())
        compare(out[b:b + 1, :, h:h + 1, :], ref_out)
        compare(SN[b:b + 1, h:h + 1], ref_SN)
