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
}
for _g in (32, 64, 128, 256):
    for _b in (1, 8):
        for _gate in ("mild", "strong"):
            _n = f"sweep_b{_b}_{_g}_{_gate}"
            WORKLOADS[_n] = Workload(_n, _b, _g, _g, 8, 128, 128, 64, _gate, (0, 1, 2, 3))


def make_inputs(B, grid_h, grid_w, heads, d_k, d_v, seed=0, gate="mild", device="cpu"):
    """Return (q, k, v, g): fp16, fp16, fp16, fp32 tensors [B, N, heads, d].

    ``device='cpu'`` draws with a seeded CPU generator; a CUDA device draws
    with a seeded generator on that device (values differ between the two).
    """
    N = grid_h * grid_w
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(int(seed))
    shp_k = (B, N, heads, d_k)
    shp_v = (B, N, heads, d_v)
    q = torch.randn(shp_k, generator=gen, device=dev, dtype=torch.float32).to(torch.float16)
    k = (torch.randn(shp_k, generator=gen, device=dev, dtype=torch.float32)
         / math.sqrt(d_k)).to(torch.float16)
    v = torch.randn(shp_v, generator=gen, device=dev, dtype=torch.float32).to(torch.float16)
    z = torch.randn(shp_k, generator=gen, device=dev, dtype=torch.float32)
    if gate == "mild":
        g = F.logsigmoid(z) / 16.0
    elif gate == "strong":
        g = F.logsigmoid(z - 2.0)
    else:
        raise ValueError(f"unknown gate recipe {gate!r}")
    return q, k, v, g.contiguous()


def make_workload_inputs(w: Workload, seed=0, device="cpu"):
    return make_inputs(w.B, w.grid_h, w.grid_w, w.heads, w.d_k, w.d_v, seed, w.gate, device)
