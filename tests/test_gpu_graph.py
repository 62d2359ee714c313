"""The forward captured in a CUDA graph and replayed, against the oracle.

The three-phase schedules launch their scan and output phase with
programmatic stream serialization (the phase starts while the one ahead of
it finishes and waits for it before reading its results), and the walk is
launched the same way after whatever precedes it on the stream.  Captured
into a graph those launches become programmatic edges; a replay must give
the oracle's outputs, and a replay after the input buffers were rewritten in
place must give the oracle's outputs for the new inputs (the graph reads the
live buffers).  Bar: the forward's, max |o_gpu - o_ref| <= 2e-3 max |o_ref|.
"""
import pytest
import torch

from recurrent_vision_backbone_key_b200 import gtr_gla
from gpu_util import compare, gpu_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gtr_gla.load()


@pytest.mark.parametrize("schedule", ["auto", "three_phase_mma", "three_phase", "walk_tcgen05", "fused"])
def test_forward_replayed_from_cuda_graph(oracle_mod, schedule):
    B, H, W, heads, d = 2, 24, 20, 3, 64
    direction = 2
    q, k, v, g = gpu_inputs(B, H, W, heads, d, d, seed=71)
    out = torch.full_like(v, float("nan"))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        # first call outside the capture: the stream's workspace and status word exist
        gtr_gla.forward(q, k, v, g, H, W, direction=direction, schedule=schedule, out=out, stream=side)
    side.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        gtr_gla.forward(q, k, v, g, H, W, direction=direction, schedule=schedule, out=out, stream=side)
    for seed in (71, 72):
        q2, k2, v2, g2 = gpu_inputs(B, H, W, heads, d, d, seed=seed)
        for dst, src in ((q, q2), (k, k2), (v, v2), (g, g2)):
            dst.copy_(src)
        out.fill_(float("nan"))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        ref = oracle_mod.gla_serial(q2.cpu(), k2.cpu(), v2.cpu(), g2.cpu(), H, W, direction)
        compare(out.cpu(), ref)
    del graph


@pytest.mark.parametrize("schedule", ["walk_tcgen05", "three_phase_mma", "three_phase"])
def test_forward_after_a_producer_kernel(oracle_mod, schedule):
    """The forward's q written by a kernel just ahead of it on the same
    stream: the first kernel of the call waits for that grid before it reads
    global memory and lets the next one start only then (the output phase of
    the three-phase schedules reads q before its own wait)."""
    B, H, W, heads, d = 4, 40, 40, 12, 64
    q, k, v, g = gpu_inputs(B, H, W, heads, d, d, seed=73)
    qn = torch.full_like(q, float("nan"))
    out = torch.empty_like(v)
    st = torch.cuda.current_stream()
    for _ in range(3):
        qn.fill_(float("nan"))
        torch.mul(q, 1.0, out=qn)  # a kernel producing q immediately before the forward
        gtr_gla.forward(qn, k, v, g, H, W, direction=0, schedule=schedule, out=out, stream=st)
    torch.cuda.synchronize()
    ref = oracle_mod.gla_serial(q.cpu(), k.cpu(), v.cpu(), g.cpu(), H, W, 0)
    compare(out.cpu(), ref)
