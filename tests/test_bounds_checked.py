"""Bounds-checked debug build on the GPU: every schedule, head size and
direction on tiny and odd shapes (7 x 9 grid, one or three heads) through
libgtr_gla_checked.so, where every global index computed at run time is
tested against its buffer before the access.  The outputs must match the
oracle and the build must report no skipped access.  This stands in for a
run under a memory-checking tool."""
import ctypes

import pytest
import torch

from recurrent_vision_backbone_key_b200 import build as libbuild
from recurrent_vision_backbone_key_b200 import gtr_gla
from recurrent_vision_backbone_key_b200.synthetic import make_inputs
from gpu_util import compare

pytestmark = pytest.mark.gpu

SCHEDULES = {"auto": 0, "fused": 1, "three_phase": 2, "three_phase_simt": 3, "fused_tcgen05": 4,
             "walk_tcgen05": 5, "three_phase_mma": 6}


@pytest.fixture(scope="module")
def clib():
    libbuild.build(checked=True)
    lib = gtr_gla.load_checked()
    assert lib.gtr_gla_bounds_checked() == 1
    gtr_gla.bounds_report(lib, clear=True)
    return lib


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def run_checked(lib, q, k, v, g, H, W, direction, chunk, schedule):
    B, N, heads, dv = v.shape
    dk = q.shape[-1]
    out = torch.full_like(v, float("nan"))
    st = lib.gtr_gla_forward_ex(_p(q), _p(k), _p(v), _p(g), B, heads, H, W, dk, dv, direction, chunk,
                                SCHEDULES[schedule], _p(out), None)
    assert st == 0, gtr_gla.STATUS_NAMES.get(st, st)
    torch.cuda.synchronize()
    return out


def assert_no_skips(lib):
    cnt, site, idx, lim = gtr_gla.bounds_report(lib, clear=True)
    assert cnt == 0, f"{cnt} accesses out of bounds; first at site {site}: index {idx} >= {lim}"


@pytest.mark.parametrize("schedule", list(SCHEDULES))
@pytest.mark.parametrize("dk,dv,chunk", [(16, 16, 16), (32, 64, 32), (64, 64, 64), (128, 128, 64), (32, 64, 64),
                                         (64, 128, 64)])
def test_checked_build_odd_shapes(clib, oracle_mod, schedule, dk, dv, chunk):
    for B, H, W, heads in ((1, 7, 9, 1), (2, 7, 9, 3)):
        q, k, v, g = make_inputs(B, H, W, heads, dk, dv, seed=dk + chunk + B)
        dq, dk_, dvv, dg = (x.cuda() for x in (q, k, v, g))
        for direction in range(4):
            out = run_checked(clib, dq, dk_, dvv, dg, H, W, direction, chunk, schedule)
            assert_no_skips(clib)
            compare(out.cpu(), oracle_mod.gla_serial(q, k, v, g, H, W, direction))


@pytest.mark.parametrize("schedule", ["auto", "fused", "fused_tcgen05"])
@pytest.mark.parametrize("gates", ["strong", "deep"])
def test_checked_build_exact_paths(clib, oracle_mod, schedule, gates):
    """Strong gates and large queries send the kernels down the paths that
    read the raw operands again: the mma.sync kernel's tf32 diagonal form
    (strong) and its per-pair exponentials (deep: a few gates of -150 nats,
    beyond fp32 factors), the tcgen05 kernels' exact score path (both)."""
    H, W, heads = 9, 15, 2
    q, k, v, g = make_inputs(1, H, W, heads, 64, 64, seed=31, gate="strong")
    q = torch.where(torch.rand(q.shape[:3])[..., None] < 0.05, q.float() * 300.0, q.float()).half()
    if gates == "deep":
        g = torch.where(torch.rand(g.shape) < 0.1, torch.full_like(g, -150.0), g)
    dq, dk_, dvv, dg = (x.cuda() for x in (q, k, v, g))
    for direction in range(4):
        out = run_checked(clib, dq, dk_, dvv, dg, H, W, direction, 64, schedule)
        assert_no_skips(clib)
        compare(out.cpu(), oracle_mod.gla_serial(q, k, v, g, H, W, direction))


@pytest.mark.parametrize("gates", ["strong", "deep"])
def test_checked_build_tf32_diagonal_d128(clib, oracle_mod, gates):
    """d_k = d_v = 128 on the fused mma.sync kernel: its tf32 diagonal form
    reads the raw q, k kept in shared memory beside the prepared operands."""
    H, W, heads = 9, 15, 2
    q, k, v, g = make_inputs(1, H, W, heads, 128, 128, seed=53, gate="strong")
    if gates == "deep":
        g = torch.where(torch.rand(g.shape) < 0.1, torch.full_like(g, -150.0), g)
    dq, dk_, dvv, dg = (x.cuda() for x in (q, k, v, g))
    for direction in range(4):
        out = run_checked(clib, dq, dk_, dvv, dg, H, W, direction, 64, "fused")
        assert_no_skips(clib)
        compare(out.cpu(), oracle_mod.gla_serial(q, k, v, g, H, W, direction))


@pytest.mark.parametrize("gates", ["mild", "strong"])
def test_checked_build_chained_tcgen05_d128(clib, oracle_mod, gates):
    """d_k = d_v = 128 on the chained tcgen05 kernel: two value-half CTAs
    per chunk, each chaining its 128 x 64 state slice through the ring over
    three chunks (the last one short); strong gates take the exact score
    path, which reads the raw rows again."""
    H, W, heads = 13, 11, 3
    q, k, v, g = make_inputs(2, H, W, heads, 128, 128, seed=59, gate=gates)
    dq, dk_, dvv, dg = (x.cuda() for x in (q, k, v, g))
    for direction in range(4):
        out = run_checked(clib, dq, dk_, dvv, dg, H, W, direction, 64, "fused_tcgen05")
        assert_no_skips(clib)
        compare(out.cpu(), oracle_mod.gla_serial(q, k, v, g, H, W, direction))


def test_checked_build_other_entry_points(clib, oracle_mod):
    """The host-buffer entry point and the no-allocation entry point."""
    B, H, W, heads = 2, 7, 9, 3
    q, k, v, g = make_inputs(B, H, W, heads, 32, 64, seed=41)
    ref = oracle_mod.gla_serial(q, k, v, g, H, W, 3)
    out_h = torch.full((B, H * W, heads, 64), float("nan"), dtype=torch.float16)
    st = clib.gtr_gla_forward_host(_p(q), _p(k), _p(v), _p(g), B, heads, H, W, 32, 64, 3, 32, _p(out_h), None)
    assert st == 0
    assert_no_skips(clib)
    compare(out_h, ref)
    dq, dk_, dvv, dg = (x.cuda() for x in (q, k, v, g))
    out = torch.full_like(dvv, float("nan"))
    st = clib.gtr_gla_forward_noalloc(_p(dq), _p(dk_), _p(dvv), _p(dg), B, heads, H, W, 32, 64, 3, 32, _p(out), None)
    assert st == 0
    torch.cuda.synchronize()
    assert_no_skips(clib)
    compare(out.cpu(), ref)
