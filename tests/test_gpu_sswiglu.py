"""GPU parity of Spatial SwiGLU's gating with its fused 3x3 depthwise
convolution against the fp64 oracle (ai.info summary of GTR, "Methodology in
Plain English"; GTR project page, "Spatial SwiGLU").

Bar: max |y_gpu - y_ref| <= 2e-3 max |y_ref|, the forward's bar: fp16 inputs
are exact in the oracle, the nine taps accumulate in fp32, the result is
rounded once to fp16 (2^-11 relative).  Grids that do not fill the 8 x 16
tiles, channel counts that do not fill the 64-channel blocks, 1-token-wide
grids (every neighbour is padding), with and without bias."""
import ctypes

import pytest
import torch

from recurrent_vision_backbone_key_b200 import build as libbuild
from recurrent_vision_backbone_key_b200 import gtr_gla
from recurrent_vision_backbone_key_b200.synthetic import SSWIGLU_WORKLOADS, make_sswiglu_inputs
from gpu_util import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gtr_gla.load()


def run(a, v, w, bias, H, W, lib=None):
    B, N, C = a.shape
    out = torch.full_like(a, float("nan"))
    if lib is None:
        gtr_gla.check(gtr_gla.gtr_sswiglu_forward(a, v, w, bias, B, H, W, C, out))
    else:
        p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
        assert lib.gtr_sswiglu_forward(p(a), p(v), p(w), p(bias), B, H, W, C, p(out), None) == 0
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("H,W", [(1, 1), (1, 37), (37, 1), (7, 9), (8, 16), (17, 33), (40, 40)])
@pytest.mark.parametrize("C", [8, 64, 72, 200])
@pytest.mark.parametrize("with_bias", [True, False])
def test_sswiglu_against_oracle(oracle_mod, H, W, C, with_bias):
    a, v, w, b = make_sswiglu_inputs(2, H, W, C, seed=H * 100 + W + C, bias=with_bias)
    out = run(a.cuda(), v.cuda(), w.cuda(), None if b is None else b.cuda(), H, W)
    compare(out, oracle_mod.sswiglu(a, v, w, b, H, W))


def test_sswiglu_full_size_sampled(oracle_mod):
    """The bench workload (B32, 40x40, C = 768): batch items 0 and 31 in
    full against the oracle."""
    wl = SSWIGLU_WORKLOADS["sswiglu_batched"]
    a, v, w, b = make_sswiglu_inputs(wl.B, wl.grid_h, wl.grid_w, wl.C, seed=4, device="cuda")
    out = run(a, v, w, b, wl.grid_h, wl.grid_w)
    for bi in (0, wl.B - 1):
        ref = oracle_mod.sswiglu(a[bi:bi + 1].cpu(), v[bi:bi + 1].cpu(), w.cpu(), b.cpu(), wl.grid_h, wl.grid_w)
        compare(out[bi:bi + 1], ref)


def test_sswiglu_bounds_checked(oracle_mod):
    """Through the bounds-checked build: no skipped access, same result."""
    libbuild.build(checked=True)
    clib = gtr_gla.load_checked()
    gtr_gla.bounds_report(clib, clear=True)
    for (H, W, C) in [(7, 9, 72), (1, 37, 8), (17, 33, 200)]:
        a, v, w, b = make_sswiglu_inputs(2, H, W, C, seed=C)
        out = run(a.cuda(), v.cuda(), w.cuda(), b.cuda(), H, W, lib=clib)
        cnt, site, idx, lim = gtr_gla.bounds_report(clib, clear=True)
        assert cnt == 0, (site, idx, lim)
        compare(out, oracle_mod.sswiglu(a, v, w, b, H, W))
