"""GPU parity: the CUDA path against the fp64 oracle on the same seeded inputs.

Bar: max |o_gpu - o_ref| <= 2e-3 * max |o_ref| (fp16 I/O, fp32 accumulate),
and bit-exact agreement of the scan-order index maps.  Small cases are
compared in full; the full-size workloads are compared on sampled (b, h)
sequences that the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

from recurrent_vision_backbone_key_b200 import gtr_gla
from recurrent_vision_backbone_key_b200.synthetic import WORKLOADS, make_workload_inputs, make_inputs
from gpu_util import REL_TOL, compare, gpu_inputs, run_forward, sample_slices, slice_of

pytestmark = pytest.mark.gpu

SCHEDULES = ["auto", "fused", "fused_tcgen05", "three_phase", "three_phase_simt", "walk_tcgen05", "three_phase_mma"]
# the shapes of the tcgen05 walk kernel and of the tcgen05 three-phase phases
WALK_SHAPES = [(32, 64), (64, 64), (128, 128), (64, 128), (128, 64), (32, 128)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gtr_gla.load()


def oracle_full(oracle_mod, q, k, v, g, H, W, direction):
    return oracle_mod.gla_serial(q.cpu(), k.cpu(), v.cpu(), g.cpu(), H, W, direction)


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_tiny(oracle_mod, schedule):
    w = WORKLOADS["tiny"]
    q, k, v, g = gpu_inputs(w.B, w.grid_h, w.grid_w, w.heads, w.d_k, w.d_v, seed=0)
    out = run_forward(q, k, v, g, w.grid_h, w.grid_w, 0, w.chunk, schedule)
    compare(out, oracle_full(oracle_mod, q, k, v, g, w.grid_h, w.grid_w, 0))


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("direction", [0, 1, 2, 3])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_ragged_grid(oracle_mod, schedule, direction, chunk):
    # 7 x 9 = 63 tokens (ragged last chunk), 9 x 15 = 135 tokens (several chunks)
    for (H, W) in [(7, 9), (9, 15)]:
        q, k, v, g = gpu_inputs(2, H, W, 3, 32, 64, seed=100 + direction + chunk)
        out = run_forward(q, k, v, g, H, W, direction, chunk, schedule)
        compare(out, oracle_full(oracle_mod, q, k, v, g, H, W, direction))


@pytest.mark.parametrize("dk", [16, 32, 64, 128])
@pytest.mark.parametrize("dv", [16, 32, 64, 128])
def test_all_head_dims(oracle_mod, dk, dv):
    H, W = 5, 23  # 115 tokens
    q, k, v, g = gpu_inputs(1, H, W, 2, dk, dv, seed=dk * 1000 + dv)
    for schedule in SCHEDULES:
        for chunk in (16, 64):
            out = run_forward(q, k, v, g, H, W, 3, chunk, schedule)
            compare(out, oracle_full(oracle_mod, q, k, v, g, H, W, 3))


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("shape", [(1, 1), (1, 37), (37, 1), (2, 2), (16, 16)])
def test_degenerate_grids(oracle_mod, schedule, shape):
    H, W = shape
    q, k, v, g = gpu_inputs(2, H, W, 2, 64, 64, seed=H * 100 + W)
    for direction in range(4):
        out = run_forward(q, k, v, g, H, W, direction, 64, schedule)
        compare(out, oracle_full(oracle_mod, q, k, v, g, H, W, direction))


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_special_gates(oracle_mod, schedule):
    H, W = 12, 11
    q, k, v, g = gpu_inputs(1, H, W, 2, 64, 32, seed=7)
    cases = {
        "open": torch.zeros_like(g),                      # causal linear attention
        "closed": torch.full_like(g, -1.0e4),             # memoryless
        "strong": gpu_inputs(1, H, W, 2, 64, 32, seed=7, gate="strong")[3],
        "mixed": torch.where(torch.rand_like(g) < 0.5, torch.zeros_like(g), g * 40.0),
    }
    for name, gg in cases.items():
        out = run_forward(q, k, v, gg, H, W, 2, 64, schedule)
        compare(out, oracle_full(oracle_mod, q, k, v, gg, H, W, 2))


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_gtr_s_640_all_directions(oracle_mod, direction):
    w = WORKLOADS["gtr_s_640"]
    q, k, v, g = gpu_inputs(w.B, w.grid_h, w.grid_w, w.heads, w.d_k, w.d_v, seed=direction)
    ref = oracle_full(oracle_mod, q, k, v, g, w.grid_h, w.grid_w, direction)
    for schedule in SCHEDULES:
        out = run_forward(q, k, v, g, w.grid_h, w.grid_w, direction, w.chunk, schedule)
        compare(out, ref)


@pytest.mark.parametrize("dk,dv,chunk", [(32, 64, 32), (64, 64, 64), (128, 128, 64), (32, 64, 64)])
def test_phases_against_oracle_intermediates(oracle_mod, dk, dv, chunk):
    """chunk_summary, boundary_scan and chunk_output one by one (chunk 64:
    the tcgen05 phases; chunk 32: the mma.sync phases)."""
    H, W, heads = 10, 13, 2
    q, k, v, g = gpu_inputs(2, H, W, heads, dk, dv, seed=77)
    direction = 3
    ref_out, ref_dS, ref_gamma, ref_Se = oracle_mod.gla_chunked(
        q.cpu(), k.cpu(), v.cpu(), g.cpu(), H, W, direction, chunk)
    B, nc = 2, (H * W + chunk - 1) // chunk
    dS = torch.empty((B, heads, nc, dk, dv), device="cuda", dtype=torch.float32)
    gamma = torch.empty((B, heads, nc, dk), device="cuda", dtype=torch.float32)
    gtr_gla.check(gtr_gla.gtr_gla_chunk_summary(k, v, g, B, heads, H, W, dk, dv, direction, chunk,
                                                dS, gamma))
    torch.cuda.synchronize()
    # fp16 tensor-core operands: the summary carries fp16 rounding of k*decay
    compare(dS, ref_dS, tol=2e-3)
    compare(gamma, ref_gamma, tol=1e-5)
    Se = torch.empty_like(dS)
    gtr_gla.check(gtr_gla.gtr_gla_boundary_scan(dS, gamma, B, heads, nc, dk, dv, Se))
    torch.cuda.synchronize()
    compare(Se, ref_Se, tol=2e-3)
    # in place
    dS2 = dS.clone()
    gtr_gla.check(gtr_gla.gtr_gla_boundary_scan(dS2, gamma, B, heads, nc, dk, dv, dS2))
    torch.cuda.synchronize()
    assert torch.equal(dS2, Se)
    # output from the oracle's own boundary states
    out = torch.empty_like(v)
    Se_ref = torch.from_numpy(ref_Se).float().cuda()
    gtr_gla.check(gtr_gla.gtr_gla_chunk_output(q, k, v, g, Se_ref, B, heads, H, W, dk, dv,
                                               direction, chunk, out))
    torch.cuda.synchronize()
    compare(out, ref_out)


def _rot(x):
    return x.flip(1).contiguous()


def _tr(x, H, W):
    B, N, h, d = x.shape
    return x.reshape(B, H, W, h, d).transpose(1, 2).reshape(B, N, h, d).contiguous()


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("shape", [(40, 40), (7, 19)])
def test_direction_maps_bit_exact(schedule, shape):
    """T->B equals L->R on the transposed grid, R->L equals L->R on the
    rotated grid, B->T equals T->B on the rotated grid: bit for bit."""
    H, W = shape
    q, k, v, g = gpu_inputs(2, H, W, 3, 64, 64, seed=5)
    X = (q, k, v, g)
    f = lambda d, Y, h, w: run_forward(*Y, h, w, d, 64, schedule)
    assert torch.equal(f(1, X, H, W), _rot(f(0, tuple(_rot(a) for a in X), H, W)))
    assert torch.equal(f(2, X, H, W), _tr(f(0, tuple(_tr(a, H, W) for a in X), W, H), W, H))
    assert torch.equal(f(3, X, H, W), _rot(f(2, tuple(_rot(a) for a in X), H, W)))


def _sampled_check(oracle_mod, w, q, k, v, g, out, direction, n_slices, seed):
    errs = []
    for (b, h) in sample_slices(w.B, w.heads, n_slices, seed):
        ref = oracle_mod.gla_serial(slice_of(q, b, h), slice_of(k, b, h), slice_of(v, b, h),
                                    slice_of(g, b, h), w.grid_h, w.grid_w, direction)
        errs.append(compare(out[b:b + 1, :, h:h + 1, :], ref)[0])
    return max(errs)


@pytest.mark.parametrize("direction", [0, 2])
def test_batched_full_size_sampled(oracle_mod, direction):
    w = WORKLOADS["batched"]
    q, k, v, g = make_workload_inputs(w, seed=direction, device="cuda")
    out = run_forward(q, k, v, g, w.grid_h, w.grid_w, direction, w.chunk)
    assert torch.isfinite(out).all()
    _sampled_check(oracle_mod, w, q, k, v, g, out, direction, 24, seed=direction)


def test_highres_twelve_block_stack_sampled(oracle_mod):
    """Twelve consecutive calls cycling L->R, R->L, T->B, B->T, each call with
    fresh inputs from the same recipe."""
    w = WORKLOADS["highres_1280"]
    for i in range(12):
        direction = i % 4
        q, k, v, g = make_workload_inputs(w, seed=1000 + i, device="cuda")
        out = run_forward(q, k, v, g, w.grid_h, w.grid_w, direction, w.chunk)
        _sampled_check(oracle_mod, w, q, k, v, g, out, direction, 2, seed=i)


@pytest.mark.parametrize("grid", [32, 64, 128, 256])
@pytest.mark.parametrize("batch", [1, 8])
@pytest.mark.parametrize("gate", ["mild", "strong"])
def test_resolution_sweep_sampled(oracle_mod, grid, batch, gate):
    w = WORKLOADS[f"sweep_b{batch}_{grid}_{gate}"]
    q, k, v, g = make_workload_inputs(w, seed=grid + batch, device="cuda")
    for direction in range(4):
        out = run_forward(q, k, v, g, w.grid_h, w.grid_w, direction, w.chunk)
        n = 2 if grid >= 128 else 3
        _sampled_check(oracle_mod, w, q, k, v, g, out, direction, n, seed=direction)
        del out
    torch.cuda.empty_cache()


def test_host_entry_point_matches_device_call(oracle_mod):
    H, W, heads, dk, dv = 20, 20, 2, 64, 64
    q, k, v, g = make_inputs(1, H, W, heads, dk, dv, seed=3)
    pin = lambda x: x.pin_memory()
    qh, kh, vh, gh = (pin(x) for x in (q, k, v, g))
    out_h = torch.empty((1, H * W, heads, dv), dtype=torch.float16).pin_memory()
    gtr_gla.check(gtr_gla.gtr_gla_forward_host(qh, kh, vh, gh, 1, heads, H, W, dk, dv, 2, 64, out_h))
    out_d = run_forward(q.cuda(), k.cuda(), v.cuda(), g.cuda(), H, W, 2, 64)
    assert torch.equal(out_h, out_d.cpu())
    compare(out_h, oracle_mod.gla_serial(q, k, v, g, H, W, 2))


@pytest.mark.parametrize("pinned", [True, False])
def test_host_entry_point_pipelined_slices(oracle_mod, pinned):
    """Enough traffic to cut the batch into slices (8 batch items over 6
    slices with page-locked buffers, 3 items with pageable ones): every
    slice's output lands in place and matches the oracle and the device call."""
    B, H, W, heads, dk, dv = (8, 32, 32, 8, 64, 64) if pinned else (3, 40, 40, 8, 64, 64)
    q, k, v, g = make_inputs(B, H, W, heads, dk, dv, seed=21)
    host = [x.pin_memory() if pinned else x.clone() for x in (q, k, v, g)]
    out_h = torch.full((B, H * W, heads, dv), float("nan"), dtype=torch.float16)
    if pinned:
        out_h = out_h.pin_memory()
    gtr_gla.check(gtr_gla.gtr_gla_forward_host(*host, B, heads, H, W, dk, dv, 1, 64, out_h))
    assert torch.isfinite(out_h).all()
    compare(out_h, oracle_mod.gla_serial(q, k, v, g, H, W, 1))
    out_d = run_forward(q.cuda(), k.cuda(), v.cuda(), g.cuda(), H, W, 1, 64)
    assert ((out_h.float() - out_d.cpu().float()).abs().max() / out_d.float().abs().max()).item() < 2e-3


def test_empty_and_streams():
    q, k, v, g = gpu_inputs(1, 4, 4, 1, 16, 16, seed=1)
    out = torch.zeros_like(v)
    before = gtr_gla.gtr_gla_launch_count()
    assert gtr_gla.gtr_gla_forward(q, k, v, g, 0, 1, 4, 4, 16, 16, 0, 16, out) == 0
    assert gtr_gla.gtr_gla_launch_count() == before
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o1 = gtr_gla.forward(q, k, v, g, 4, 4, chunk=16)
    s.synchronize()
    o2 = run_forward(q, k, v, g, 4, 4, 0, 16)
    assert torch.equal(o1, o2)
    assert gtr_gla.gtr_gla_get_last_device_status() == 0


def test_fused_repeated_calls_reset_control_words(oracle_mod):
    """The fused kernel's ticket and flags start from zero on every call:
    back-to-back calls, interleaved with the three-phase schedule on the same
    stream, all stay correct."""
    H, W, heads = 24, 24, 4
    for i in range(4):
        q, k, v, g = gpu_inputs(2, H, W, heads, 64, 64, seed=300 + i)
        out = run_forward(q, k, v, g, H, W, i % 4, 64, "fused")
        compare(out, oracle_full(oracle_mod, q, k, v, g, H, W, i % 4))
        run_forward(q, k, v, g, H, W, i % 4, 64, "three_phase")
    assert gtr_gla.gtr_gla_get_last_device_status() == 0


@pytest.mark.parametrize("schedule,d,chunk,H,W", [("fused", 64, 16, 8, 8), ("fused_tcgen05", 64, 64, 16, 16)])
def test_fused_bounded_wait_times_out_cleanly(oracle_mod, schedule, d, chunk, H, W):
    """A tile that never publishes its state: the successor's wait gives up
    after the spin limit, the status word reports GTR_ERR_TIMEOUT, the
    kernel finishes, and the next call is correct again.  Run on the mma.sync
    kernel and on the tcgen05 kernel (per-warp waits)."""
    heads = 2
    q, k, v, g = gpu_inputs(1, H, W, heads, d, d, seed=9)
    out = torch.zeros_like(v)
    st = gtr_gla.gtr_gla_debug_forward_fused(q, k, v, g, 1, heads, H, W, d, d, 0, chunk, schedule,
                                             1, 1, 2000, out)
    assert st == 0
    assert gtr_gla.gtr_gla_get_last_device_status() == 6  # GTR_ERR_TIMEOUT
    assert gtr_gla.gtr_gla_get_last_device_status() == 0  # cleared by the read
    out2 = run_forward(q, k, v, g, H, W, 0, chunk, schedule)
    compare(out2, oracle_full(oracle_mod, q, k, v, g, H, W, 0))
    # the hook with no hold changes nothing
    out3 = torch.zeros_like(v)
    assert gtr_gla.gtr_gla_debug_forward_fused(q, k, v, g, 1, heads, H, W, d, d, 0, chunk, schedule,
                                               -1, -1, 1 << 22, out3) == 0
    torch.cuda.synchronize()
    assert torch.equal(out3, out2)
    assert gtr_gla.gtr_gla_get_last_device_status() == 0


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_special_gates_d64(oracle_mod, schedule):
    """d_k = d_v = 64, chunk 64: the shape of the tcgen05 path, whose exact
    score path takes over when the decay over a chunk is strong."""
    H, W = 10, 13
    q, k, v, g = gpu_inputs(2, H, W, 2, 64, 64, seed=17)
    cases = {
        "mild": g,
        "open": torch.zeros_like(g),
        "closed": torch.full_like(g, -1.0e4),
        "strong": gpu_inputs(2, H, W, 2, 64, 64, seed=17, gate="strong")[3],
        "mixed": torch.where(torch.rand_like(g) < 0.97, g, g * 60.0),
    }
    for name, gg in cases.items():
        for direction in range(4):
            out = run_forward(q, k, v, gg, H, W, direction, 64, schedule)
            compare(out, oracle_full(oracle_mod, q, k, v, gg, H, W, direction))
    # |q~| above 16 in a few tokens with mild gates: the tcgen05 kernel
    # rewrites those chunks' query operand without the 1/gamma_c factor
    gen = torch.Generator(device="cuda").manual_seed(5)
    big = torch.rand(q.shape[:3], device="cuda", generator=gen) < 0.05
    qb = torch.where(big[..., None], q.float() * 300.0, q.float()).half()
    for direction in (0, 2):
        out = run_forward(qb, k, v, g, H, W, direction, 64, schedule)
        compare(out, oracle_full(oracle_mod, qb, k, v, g, H, W, direction))


@pytest.mark.parametrize("direction", [0, 2])
def test_batched_full_size_tcgen05_sampled(oracle_mod, direction):
    w = WORKLOADS["batched"]
    q, k, v, g = make_workload_inputs(w, seed=10 + direction, device="cuda")
    out = run_forward(q, k, v, g, w.grid_h, w.grid_w, direction, w.chunk, "fused_tcgen05")
    assert torch.isfinite(out).all()
    _sampled_check(oracle_mod, w, q, k, v, g, out, direction, 24, seed=direction)
    ref = run_forward(q, k, v, g, w.grid_h, w.grid_w, direction, w.chunk, "fused")
    assert ((out.float() - ref.float()).abs().max() / ref.float().abs().max()).item() < 2e-3


@pytest.mark.parametrize("B,heads", [(1, 6), (4, 40)])
def test_cuda_graph_twelve_call_stack(B, heads):
    """A stack of 12 forward calls cycling the four directions (the high-res
    block stack), captured once into a CUDA graph and replayed: every replay
    gives the outputs of the eager calls bit for bit.  (1, 6) runs the
    mma.sync kernel with two chunks per tile, (4, 40) the tcgen05 kernel."""
    H = W = 24
    xs = [gpu_inputs(B, H, W, heads, 64, 64, seed=400 + i) for i in range(12)]
    outs = [torch.empty_like(x[2]) for x in xs]

    def stack():
        st = torch.cuda.current_stream()
        for i, (q, k, v, g) in enumerate(xs):
            gtr_gla.forward(q, k, v, g, H, W, direction=i % 4, chunk=64, out=outs[i], stream=st)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        stack()  # eager: allocates the workspaces before the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):  # the stream whose workspace exists
        stack()
    for rep in range(3):
        for o in outs:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for o, e in zip(outs, eager):
            assert torch.equal(o, e), rep
    assert gtr_gla.gtr_gla_get_last_device_status() == 0
    del graph


@pytest.mark.parametrize("dk,dv", WALK_SHAPES)
@pytest.mark.parametrize("schedule", ["walk_tcgen05", "three_phase", "three_phase_mma"])
def test_walk_shapes_all_directions(oracle_mod, dk, dv, schedule):
    """Every shape of the tcgen05 walk kernel and of the tcgen05 phases, all
    four directions, on a ragged grid (7 x 19 = 133 tokens: two full chunks
    and a tail of 5) and a grid of several full chunks, B = 2, 3 heads."""
    for (H, W) in [(7, 19), (16, 24)]:
        q, k, v, g = gpu_inputs(2, H, W, 3, dk, dv, seed=dk * 7 + dv + H)
        for direction in range(4):
            out = run_forward(q, k, v, g, H, W, direction, 64, schedule)
            compare(out, oracle_full(oracle_mod, q, k, v, g, H, W, direction))


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (32, 64)])
def test_walk_special_gates(oracle_mod, dk, dv):
    """Open, closed, strong and mixed gates, and a few |q~| > 16 tokens,
    through the walk kernel: the whole-chunk form and the exact score path."""
    H, W = 10, 13
    q, k, v, g = gpu_inputs(2, H, W, 2, dk, dv, seed=31 + dk)
    cases = {
        "open": torch.zeros_like(g),
        "closed": torch.full_like(g, -1.0e4),
        "strong": gpu_inputs(2, H, W, 2, dk, dv, seed=31 + dk, gate="strong")[3],
        "mixed": torch.where(torch.rand_like(g) < 0.97, g, g * 60.0),
    }
    for name, gg in cases.items():
        for direction in (0, 3):
            out = run_forward(q, k, v, gg, H, W, direction, 64, "walk_tcgen05")
            compare(out, oracle_full(oracle_mod, q, k, v, gg, H, W, direction))
    gen = torch.Generator(device="cuda").manual_seed(6)
    big = torch.rand(q.shape[:3], device="cuda", generator=gen) < 0.05
    qb = torch.where(big[..., None], q.float() * 300.0, q.float()).half()
    out = run_forward(qb, k, v, g, H, W, 1, 64, "walk_tcgen05")
    compare(out, oracle_full(oracle_mod, qb, k, v, g, H, W, 1))


def test_chained_tcgen05_control_block_resets_itself(oracle_mod):
    """The chained tcgen05 kernel's ticket and flags are never cleared by the
    host: each launch leaves them ready for the next.  Launches of different
    grid sizes (different sequences and chunk counts) on one stream, each
    checked against the oracle, then the first shape again; a large problem
    (400 sequences), a small one and the large one again, so that the small
    problem's ring would overwrite the large problem's flags if the two
    shared a buffer."""
    shapes = [(2, 24, 24, 4), (3, 16, 40, 5), (1, 7, 9, 3), (2, 24, 24, 4), (40, 16, 16, 10), (1, 16, 16, 2),
              (40, 16, 16, 10)]
    for i, (B, H, W, heads) in enumerate(shapes):
        q, k, v, g = gpu_inputs(B, H, W, heads, 64, 64, seed=600 + i)
        for direction in (i % 4, (i + 1) % 4):
            out = run_forward(q, k, v, g, H, W, direction, 64, "fused_tcgen05")
            compare(out, oracle_full(oracle_mod, q, k, v, g, H, W, direction))
    assert gtr_gla.gtr_gla_get_last_device_status() == 0
