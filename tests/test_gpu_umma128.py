"""The chained tcgen05 kernel at d_k = d_v = 128 (GTR_SCHED_FUSED_TCGEN05)
against the fp64 oracle.

At d = 128 each (sequence, chunk) is two CTAs, one per 64 value columns,
each with its own chain of 128 x 64 state slices through the ring.  Bar: the
forward's, max |o_gpu - o_ref| <= 2e-3 max |o_ref| (fp16 I/O, fp32
accumulation).  Covered: every scan order on ragged grids (the last chunk
short), the gate regimes that send chunks to the exact score path (open,
closed, strong, mixed, large |q~|), the full-size B8 64x64 sweep workload
on sampled sequences, the bounded wait of the chain, and agreement with the
mma.sync kernel.
"""
import pytest
import torch

from recurrent_vision_backbone_key_b200 import gtr_gla
from recurrent_vision_backbone_key_b200.synthetic import WORKLOADS, make_workload_inputs
from gpu_util import compare, gpu_inputs, run_forward
from test_gpu_parity import _sampled_check

pytestmark = pytest.mark.gpu
D = 128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gtr_gla.load()


def oracle_full(oracle_mod, q, k, v, g, H, W, direction):
    return oracle_mod.gla_serial(q.cpu(), k.cpu(), v.cpu(), g.cpu(), H, W, direction)


def test_plan_is_the_chained_tcgen05_kernel():
    assert gtr_gla.gtr_gla_plan(2, 2, 17, 23, D, D, 64, gtr_gla.SCHEDULES["fused_tcgen05"], 148) == 4


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
@pytest.mark.parametrize("H,W", [(17, 23), (8, 8), (1, 129), (24, 24)])
def test_ragged_grids_all_directions(oracle_mod, direction, H, W):
    q, k, v, g = gpu_inputs(2, H, W, 3, D, D, seed=H * 100 + W + direction)
    out = run_forward(q, k, v, g, H, W, direction, 64, "fused_tcgen05")
    compare(out, oracle_full(oracle_mod, q, k, v, g, H, W, direction))


def test_special_gates(oracle_mod):
    H, W = 10, 13
    q, k, v, g = gpu_inputs(2, H, W, 2, D, D, seed=23)
    cases = {
        "mild": g,
        "open": torch.zeros_like(g),
        "closed": torch.full_like(g, -1.0e4),
        "strong": gpu_inputs(2, H, W, 2, D, D, seed=23, gate="strong")[3],
        "mixed": torch.where(torch.rand_like(g) < 0.97, g, g * 60.0),
    }
    for name, gg in cases.items():
        for direction in range(4):
            out = run_forward(q, k, v, gg, H, W, direction, 64, "fused_tcgen05")
            compare(out, oracle_full(oracle_mod, q, k, v, gg, H, W, direction))
    # |q~| above 16 in a few tokens: those chunks take the exact score path
    gen = torch.Generator(device="cuda").manual_seed(6)
    big = torch.rand(q.shape[:3], device="cuda", generator=gen) < 0.05
    qb = torch.where(big[..., None], q.float() * 300.0, q.float()).half()
    for direction in (0, 2):
        out = run_forward(qb, k, v, g, H, W, direction, 64, "fused_tcgen05")
        compare(out, oracle_full(oracle_mod, qb, k, v, g, H, W, direction))


@pytest.mark.parametrize("direction", [0, 3])
def test_sweep_b8_64_full_size_sampled(oracle_mod, direction):
    w = WORKLOADS["sweep_b8_64_mild"]
    q, k, v, g = make_workload_inputs(w, seed=70 + direction, device="cuda")
    out = run_forward(q, k, v, g, w.grid_h, w.grid_w, direction, w.chunk, "fused_tcgen05")
    assert torch.isfinite(out).all()
    _sampled_check(oracle_mod, w, q, k, v, g, out, direction, 6, seed=direction)
    ref = run_forward(q, k, v, g, w.grid_h, w.grid_w, direction, w.chunk, "fused")
    assert ((out.float() - ref.float()).abs().max() / ref.float().abs().max()).item() < 2e-3


def test_bounded_wait_times_out_cleanly(oracle_mod):
    """A tile that never publishes: its successors' waits give up after the
    spin limit, the status word reports GTR_ERR_TIMEOUT, the kernel finishes,
    and the next call is correct."""
    H, W, heads = 16, 16, 2
    q, k, v, g = gpu_inputs(1, H, W, heads, D, D, seed=31)
    out = torch.zeros_like(v)
    st = gtr_gla.gtr_gla_debug_forward_fused(q, k, v, g, 1, heads, H, W, D, D, 0, 64, "fused_tcgen05",
                                             1, 1, 2000, out)
    assert st == 0
    assert gtr_gla.gtr_gla_get_last_device_status() == 6  # GTR_ERR_TIMEOUT
    assert gtr_gla.gtr_gla_get_last_device_status() == 0
    out2 = run_forward(q, k, v, g, H, W, 0, 64, "fused_tcgen05")
    compare(out2, oracle_full(oracle_mod, q, k, v, g, H, W, 0))
