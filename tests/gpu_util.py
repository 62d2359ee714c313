"""Helpers shared by the GPU parity tests (CUDA path vs fp64 oracle)."""
import numpy as np
import torch

from recurrent_vision_backbone_key_b200 import gtr_gla
from recurrent_vision_backbone_key_b200.synthetic import make_inputs

# Tolerance of the forward: max |o_gpu - o_ref| <= REL_TOL * max |o_ref| over
# the compared outputs (fp16 inputs and outputs, fp32 accumulation).
REL_TOL = 2e-3


def gpu_inputs(B, H, W, heads, dk, dv, seed, gate="mild", device="cuda"):
    """Seeded inputs drawn on the CPU generator (small) and moved to the GPU."""
    q, k, v, g = make_inputs(B, H, W, heads, dk, dv, seed=seed, gate=gate, device="cpu")
    return tuple(x.to(device) for x in (q, k, v, g))


def run_forward(q, k, v, g, H, W, direction, chunk, schedule=0):
    out = gtr_gla.forward(q, k, v, g, H, W, direction=direction, chunk=chunk, schedule=schedule)
    torch.cuda.synchronize()
    return out


def compare(out_gpu, ref, tol=REL_TOL):
    """Returns (rel_err, cosine) and asserts rel_err <= tol."""
    o = out_gpu.detach().float().cpu().numpy().astype(np.float64) if hasattr(out_gpu, "detach") \
        else np.asarray(out_gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert o.shape == r.shape, (o.shape, r.shape)
    assert np.isfinite(o).all(), "non-finite GPU output"
    scale = max(np.abs(r).max(), 1e-30)
    err = np.abs(o - r).max() / scale
    cos = float((o * r).sum() / max(np.sqrt((o * o).sum() * (r * r).sum()), 1e-300))
    assert err <= tol, f"rel err {err:.3e} > {tol:.1e} (cosine {cos:.6f})"
    return err, cos


def slice_of(x, b, h):
    """[B,N,heads,d] -> [1,N,1,d] CPU float64 copy of one (b, h) sequence."""
    return x[b:b + 1, :, h:h + 1, :].detach().float().cpu().numpy().astype(np.float64)


def sample_slices(B, heads, n, seed):
    """n distinct (b, h) pairs: (0, 0), the last one, then seeded random ones."""
    rng = np.random.default_rng(seed)
    picks = [(0, 0), (B - 1, heads - 1)]
    while len(picks) < min(n, B * heads):
        p = (int(rng.integers(B)), int(rng.integers(heads)))
        if p not in picks:
            picks.append(p)
    return picks[: min(n, B * heads)]
