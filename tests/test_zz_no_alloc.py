"""gtr_gla_forward_noalloc: the forward for callers that cannot let the
library allocate device memory while they run (hosts that own all device
memory through their own allocator or budget, real-time loops that forbid
allocation after start-up).  Its scratch is a fixed 16 MiB array inside the
library that every call reuses, so the tests call it through the C ABI
several times in a row, on problems of different sizes, and check every
result against gtr_gla_forward and against the fp64 oracle within the
forward's tolerance; a problem too large for the fixed scratch is refused
without a launch.

This file is collected last on purpose and works in a fresh process too.
"""
import numpy as np
import pytest
import torch

from recurrent_vision_backbone_key_b200 import build as libbuild
from recurrent_vision_backbone_key_b200 import gtr_gla
from recurrent_vision_backbone_key_b200.synthetic import make_inputs

pytestmark = pytest.mark.gpu

REL_TOL = 2e-3  # the forward's parity tolerance: max|diff| <= 2e-3 * max|reference|


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    libbuild.build()
    gtr_gla.load()


def _rel(a, b):
    a = a.float().cpu().numpy().astype(np.float64) if hasattr(a, "cpu") else np.asarray(a)
    b = b.float().cpu().numpy().astype(np.float64) if hasattr(b, "cpu") else np.asarray(b)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def _noalloc(q, k, v, g, B, heads, H, W, dk, dv, direction, chunk):
    out = torch.full_like(v, float("nan"))
    st = gtr_gla.gtr_gla_forward_noalloc(q, k, v, g, B, heads, H, W, dk, dv, direction, chunk, out)
    assert st == 0, (gtr_gla.gtr_gla_status_string(st), gtr_gla.last_error())
    torch.cuda.synchronize()
    return out


def test_noalloc_matches_forward_and_oracle_on_consecutive_calls(oracle_mod):
    """Four calls in a row: the GTR-S-like 40x40 grid (6 heads, d=64) twice
    with other inputs and directions, then a d_k=d_v=128 problem (the widest
    shared-memory layout of the CUDA-core output kernel), then a smaller grid
    again, so leftover scratch contents of a larger call are never read."""
    cases = [
        (1, 40, 40, 6, 64, 64, 0, 1),
        (1, 40, 40, 6, 64, 64, 2, 2),
        (1, 32, 32, 2, 128, 128, 3, 3),
        (2, 9, 13, 3, 32, 64, 1, 4),
    ]
    for call, (B, H, W, heads, dk, dv, direction, seed) in enumerate(cases):
        qc, kc, vc, gc = make_inputs(B, H, W, heads, dk, dv, seed=seed)
        q, k, v, g = (x.cuda() for x in (qc, kc, vc, gc))
        out = _noalloc(q, k, v, g, B, heads, H, W, dk, dv, direction, 64)
        assert torch.isfinite(out).all(), f"call {call}"
        ref = torch.empty_like(v)
        gtr_gla.check(gtr_gla.gtr_gla_forward(q, k, v, g, B, heads, H, W, dk, dv, direction, 64, ref))
        torch.cuda.synchronize()
        assert _rel(out, ref) <= REL_TOL, f"call {call} against gtr_gla_forward"
        exact = oracle_mod.gla_serial(qc, kc, vc, gc, H, W, direction)
        assert _rel(out, exact) <= REL_TOL, f"call {call} against the oracle"


def test_noalloc_refuses_oversized_problem():
    # batched 32 x 40x40 x 12 heads x d=64 needs ~158 MB of chunk states
    q = torch.empty((32, 1600, 12, 64), dtype=torch.float16, device="cuda")
    g = torch.empty((32, 1600, 12, 64), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    before = gtr_gla.gtr_gla_launch_count()
    st = gtr_gla.gtr_gla_forward_noalloc(q, q, q, g, 32, 12, 40, 40, 64, 64, 0, 64, out)
    assert st == 2  # GTR_ERR_UNSUPPORTED_SHAPE
    assert "16 MiB" in gtr_gla.last_error()
    assert gtr_gla.gtr_gla_launch_count() == before
