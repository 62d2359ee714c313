"""Seeded synthetic inputs for the key-gated GLA token mixer.

This module only draws random numbers; it holds none of the mixer's
arithmetic.  Both the CUDA path (tests, benchmark, smoke check) and the CPU
oracle take their inputs from here, so the two always see the same values.

Recipe (the pages measure on COCO-style 640x640 and 1280x1280 images; here
only their stride-16 token-grid shapes are reproduced, with synthetic values):
  * q ~ N(0, 1), v ~ N(0, 1), rounded to fp16;
  * k ~ N(0, 1) / sqrt(d_k) drawn in fp32, then rounded to fp16;
  * log-gates g = logsigmoid(N(0, 1)) / 16 in fp32 ("mild"), or
    g = logsigmoid(N(-2, 1)) in fp32 ("strong" decay);
  * draw order q, k, v, g, each of shape [B, N, heads, d], N = grid_h*grid_w
    in row-major spatial order.
Two generators are offered: a CPU ``torch.Generator`` (small cases that the
oracle runs in full) and a CUDA ``torch.Generator`` (large cases, where the
oracle gets the sampled slices copied back from the device).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    """One GLA forward problem: sizes and the input recipe."""
    name: str
    B: int
    grid_h: int
    grid_w: int
    heads: int
    d_k: int
    d_v: int
    chunk: int = 64
    gate: str = "mild"
    directions: tuple = (0,)

    @property
    def N(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def token_heads(self) -> int:
        return self.B * self.N * self.heads

    def algorithmic_bytes(self) -> int:
        """q, k, v, out in fp16 plus g in fp32, each read or written once."""
        th = self.token_heads
        return th * (2 * self.d_k + 2 * self.d_k + 2 * self.d_v + 4 * self.d_k + 2 * self.d_v)

    def algorithmic_flops(self) -> int:
        """4*dk*dv (chunk summary + state readout) + C*(dk+dv) (causal half of
        the intra-chunk score and score-value products) per token-head."""
        return self.token_heads * (4 * self.d_k * self.d_v + self.chunk * (self.d_k + self.d_v))


# The workloads named for this operator: the tiny parity case, the GTR-S-like
# 640^2 latency case, the 1280^2 case, the batched throughput case and the
# resolution sweep (d=128).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 8, 8, 1, 16, 16, 16, "mild", (0,)),
    "gtr_s_640": Workload("gtr_s_640", 1, 40, 40, 6, 64, 64, 64, "mild", (0, 1, 2, 3)),
    "highres_1280": Workload("highres_1280", 1, 80, 80, 6, 64, 64, 64, "mild", (0, 1, 2, 3)),
    "batched": Workload("batched", 32, 40, 40, 12, 64, 64, 64, "mild", (0, 2)),
    # the pages' deployment shape (d_k = 32, d_v = 64, chunk 64) at the batched size
    "deploy_batched": Workload("deploy_batched", 32, 40, 40, 12, 32, 64, 64, "mild", (0, 2)),
}
for _g in (32, 64, 128, 256):
    for _b in (1, 8):
        for _gate in ("mild", "strong"):
            _n = f"sweep_b{_b}_{_g}_{_gate}"
            WORKLOADS[_n] = Workload(_n, _b, _g, _g, 8, 128, 128, 64, _gate, (0, 1, 2, 3))


def make_inputs(B, grid_h, grid_w, heads, d_k, d_v, seed=0, gate="mild", device="cpu",
                dtype=torch.float16):
    """Return (q, k, v, g): q, k, v in ``dtype`` (fp16, or bf16 for the bf16
    variant), g fp32; each [B, N, heads, d].

    ``device='cpu'`` draws with a seeded CPU generator; a CUDA device draws
    with a seeded generator on that device (values differ between the two).
    """
    N = grid_h * grid_w
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(int(seed))
    shp_k = (B, N, heads, d_k)
    shp_v = (B, N, heads, d_v)
    q = torch.randn(shp_k, generator=gen, device=dev, dtype=torch.float32).to(dtype)
    k = (torch.randn(shp_k, generator=gen, device=dev, dtype=torch.float32)
         / math.sqrt(d_k)).to(dtype)
    v = torch.randn(shp_v, generator=gen, device=dev, dtype=torch.float32).to(dtype)
    z = torch.randn(shp_k, generator=gen, device=dev, dtype=torch.float32)
    if gate == "mild":
        g = F.logsigmoid(z) / 16.0
    elif gate == "strong":
        g = F.logsigmoid(z - 2.0)
    else:
        raise ValueError(f"unknown gate recipe {gate!r}")
    return q, k, v, g.contiguous()


def make_workload_inputs(w: Workload, seed=0, device="cpu", dtype=torch.float16):
    return make_inputs(w.B, w.grid_h, w.grid_w, w.heads, w.d_k, w.d_v, seed, w.gate, device, dtype)


@dataclass(frozen=True)
class SSwiGLUWorkload:
    """One Spatial SwiGLU gating problem: [B, H*W, C] branches on an H x W grid."""
    name: str
    B: int
    grid_h: int
    grid_w: int
    C: int

    @property
    def N(self) -> int:
        return self.grid_h * self.grid_w

    def algorithmic_bytes(self) -> int:
        """a and v read, out written (fp16), the filter and bias read once."""
        return self.B * self.N * self.C * 6 + self.C * (9 + 1) * 4


# The batched grid (B32, 40x40) with a channel width equal to the mixer's
# token width (12 heads x 64): the pages give no block widths.
SSWIGLU_WORKLOADS = {
    "sswiglu_batched": SSwiGLUWorkload("sswiglu_batched", 32, 40, 40, 768),
}


def make_sswiglu_inputs(B, grid_h, grid_w, C, seed=0, device="cpu", bias=True):
    """(a, v, w, bias): a, v ~ N(0, 1) fp16 [B, H*W, C]; the 3x3 depthwise
    filter w ~ N(0, 1/9) fp32 [C, 3, 3]; bias ~ N(0, 0.1^2) fp32 [C] or None."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(int(seed))
    N = grid_h * grid_w
    a = torch.randn((B, N, C), generator=gen, device=dev).to(torch.float16)
    v = torch.randn((B, N, C), generator=gen, device=dev).to(torch.float16)
    w = torch.randn((C, 3, 3), generator=gen, device=dev) / 3.0
    b = torch.randn((C,), generator=gen, device=dev) * 0.1 if bias else None
    return a, v, w.contiguous(), b
