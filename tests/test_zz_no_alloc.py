"""gtr_gla_forward_noalloc: the forward for callers that cannot let the
library allocate device memory while they run (hosts that own all device
memory through their own allocator or budget, real-time loops that forbid
allocation after start-up).  Its scratch is a fixed 16 MiB array inside the
library, so the test checks, through the C ABI, that two calls in a row give
the same result as gtr_gla_forward within the parity tolerance, and that a
problem too large for the fixed scratch is refused without a launch.

This file is collected last on purpose and works in a fresh process too.
"""
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
    return ((a.float() - b.float()).abs().max() / b.float().abs().max().clamp_min(1e-30)).item()


def test_noalloc_matches_forward_on_two_calls():
    # GTR-S-like 640x640 grid (40x40 tokens, 6 heads, d=64) fits the scratch.
    H, W, heads, d = 40, 40, 6, 64
    for call, (seed, direction) in enumerate([(1, 0), (2, 2)]):
        q, k, v, g = (x.cuda() for x in make_inputs(1, H, W, heads, d, d, seed=seed))
        ref = torch.empty_like(v)
        gtr_gla.check(gtr_gla.gtr_gla_forward(q, k, v, g, 1, heads, H, W, d, d, direction, 64, ref))
        out = torch.full_like(v, float("nan"))
        st = gtr_gla.gtr_gla_forward_noalloc(q, k, v, g, 1, heads, H, W, d, d, direction, 64, out)
        assert st == 0, gtr_gla.gtr_gla_status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all(), f"call {call}"
        assert _rel(out, ref) <= REL_TOL, f"call {call}"


def test_noalloc_refuses_oversized_problem():
    # batched 32 x 40x40 x 12 heads x d=64 needs ~158 MB of chunk states
    q = torch.empty((32, 1600, 12, 64), dtype=torch.float16, device="cuda")
    g = torch.empty((32, 1600, 12, 64), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    before = gtr_gla.gtr_gla_launch_count()
    st = gtr_gla.gtr_gla_forward_noalloc(q, q, q, g, 32, 12, 40, 40, 64, 64, 0, 64, out)
    assert st == 2  # GTR_ERR_UNSUPPORTED_SHAPE
    assert gtr_gla.gtr_gla_launch_count() == before
