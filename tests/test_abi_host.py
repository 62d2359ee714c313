"""Host-side checks of the C ABI that need no GPU: the library loads, it
exports every function include/gtr_gla.h declares, and argument validation
returns the documented status before any CUDA call is made."""
import ctypes
import os
import re

import pytest

from recurrent_vision_backbone_key_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    from recurrent_vision_backbone_key_b200 import gtr_gla
    return gtr_gla


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(gtr_\w+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    cdll = lib.load()
    for n in sorted(names):
        assert hasattr(cdll, n), n
    assert names <= set(lib.SIGNATURES), names - set(lib.SIGNATURES)


def test_bounds_checked_build_loads_and_exports(lib):
    """The bounds-checked debug build has the same C ABI; it says it is the
    checked one, and the normal build refuses the report call."""
    libbuild.build(checked=True)
    checked = lib.load_checked()
    for n in sorted(declared_functions()):
        assert hasattr(checked, n), n
    assert checked.gtr_gla_bounds_checked() == 1
    assert lib.load().gtr_gla_bounds_checked() == 0
    cnt, site = ctypes.c_ulonglong(7), ctypes.c_int(7)
    idx, lim = ctypes.c_longlong(7), ctypes.c_longlong(7)
    st = lib.load().gtr_gla_debug_bounds_report(ctypes.byref(cnt), ctypes.byref(site), ctypes.byref(idx),
                                                ctypes.byref(lim), 0)
    assert st == 1 and cnt.value == 0 and site.value == 0


def test_version_and_status_strings(lib):
    assert lib.gtr_gla_version() >= 100
    assert lib.gtr_gla_status_string(0) == "ok"
    assert lib.gtr_gla_status_string(6) == "device wait timed out"


A = 1 << 20  # fake, 16-byte aligned "device" addresses; never dereferenced


def fwd(lib, **kw):
    args = dict(q=A, k=2 * A, v=3 * A, g=4 * A, B=1, heads=2, grid_h=4, grid_w=4, d_k=16,
                d_v=16, direction=0, chunk=16, out=5 * A, stream=0)
    args.update(kw)
    return lib.gtr_gla_forward(**args)


def test_error_paths(lib):
    assert fwd(lib, q=None) == 1
    assert fwd(lib, out=None) == 1
    assert fwd(lib, direction=4) == 1
    assert fwd(lib, direction=-1) == 1
    assert fwd(lib, B=-1) == 1
    assert fwd(lib, d_k=48) == 2
    assert fwd(lib, d_v=256) == 2
    assert fwd(lib, chunk=128) == 2
    assert fwd(lib, chunk=0) == 2
    assert fwd(lib, q=A + 8) == 3
    assert fwd(lib, g=4 * A + 4) == 3
    # out overlapping q (q spans 1*16*2*16*2 = 1 KiB)
    assert fwd(lib, out=A + 512) == 4
    assert fwd(lib, out=4 * A) == 4
    assert "overlaps" in lib.last_error()


def test_empty_problems_launch_nothing(lib):
    before = lib.gtr_gla_launch_count()
    assert fwd(lib, B=0) == 0
    assert fwd(lib, grid_h=0) == 0
    assert fwd(lib, heads=0) == 0
    assert lib.gtr_gla_launch_count() == before


def test_phase_entry_points_validate(lib):
    assert lib.gtr_gla_chunk_summary(2 * A, 3 * A, 4 * A, 1, 1, 4, 4, 16, 16, 0, 16, None, 6 * A, 0) == 1
    assert lib.gtr_gla_chunk_summary(2 * A, 3 * A, 4 * A, 1, 1, 4, 4, 16, 16, 0, 16, 2 * A, 6 * A, 0) == 4
    assert lib.gtr_gla_boundary_scan(A, 2 * A, 1, 1, 3, 16, 24, 3 * A, 0) == 2
    assert lib.gtr_gla_boundary_scan(A, 2 * A, 1, 1, 0, 16, 16, 3 * A, 0) == 0
    # partial overlap of S_enter with dS is an error, exact in-place is fine
    assert lib.gtr_gla_boundary_scan(A, 2 * A, 1, 1, 2, 16, 16, A + 16, 0) == 4
    assert lib.gtr_gla_chunk_output(A, 2 * A, 3 * A, 4 * A, 6 * A, 1, 1, 4, 4, 16, 16, 5, 16, 5 * A, 0) == 1
    assert lib.gtr_gla_chunk_output(A, 2 * A, 3 * A, 4 * A, 6 * A, 1, 1, 4, 4, 16, 16, 0, 16, 6 * A, 0) == 4


def test_workspace_bytes(lib):
    # three-phase: dS (nseq*nc*dk*dv fp32) + gamma (nseq*nc*dk fp32), 256-byte aligned
    n = lib.gtr_gla_workspace_bytes_ex(2, 3, 10, 10, 32, 64, 16, "three_phase")
    nc = (100 + 15) // 16
    assert n >= 6 * nc * 32 * 64 * 4 + 6 * nc * 32 * 4
    assert lib.gtr_gla_workspace_bytes_ex(1, 1, 4, 4, 24, 16, 16, "three_phase") == 0
    # the seven-argument form is the bound over the schedules AUTO may take
    n7 = lib.gtr_gla_workspace_bytes(2, 3, 10, 10, 32, 64, 16)
    assert n7 >= n and n7 >= lib.gtr_gla_workspace_bytes_ex(2, 3, 10, 10, 32, 64, 16, "fused")
    assert lib.gtr_gla_workspace_bytes(0, 3, 10, 10, 32, 64, 16) == 0
    assert lib.gtr_gla_workspace_bytes(1, 1, 4, 4, 24, 16, 16) == 0
    # the chained kernels' workspace: control words (ticket, unused, four
    # flags per (sequence, 64 value columns)) padded to 256 bytes, a two-slot
    # fp32 ring of d_k x d_v states per sequence, the stream's status word
    a256 = lambda x: (x + 255) // 256 * 256
    for (B, heads, d) in ((2, 3, 64), (2, 3, 128), (5, 7, 128)):
        nseq = B * heads
        want = a256((nseq * 4 * (d // 64) + 2) * 4) + nseq * 2 * d * d * 4 + 256
        assert lib.gtr_gla_workspace_bytes_ex(B, heads, 10, 10, d, d, 64, "fused_tcgen05") == want


def test_dispatch_plan(lib):
    """The kernels each schedule launches (host-only decision, 148 SMs)."""
    plan = lambda B, heads, H, W, dk, dv, C, sched: lib.gtr_gla_plan(B, heads, H, W, dk, dv, C, sched, 148)
    # batched: 384 sequences at d = 64 (2.6 per SM) -> the tcgen05 walk kernel
    assert plan(32, 12, 40, 40, 64, 64, 64, "auto") == 5
    assert plan(25, 12, 8, 8, 64, 64, 64, "auto") == 5     # 300 items
    assert plan(64, 12, 40, 40, 64, 64, 64, "auto") == 4   # 768: more than one wave -> chained
    assert plan(32, 12, 40, 40, 32, 64, 64, "auto") == 5   # the deployment shape, batched
    assert plan(16, 12, 40, 40, 64, 128, 64, "auto") == 5  # 192 sequences x 2 value slices
    # latency configs and the B1 sweep: at most 24 sequences -> three phases (mma.sync phases)
    assert plan(1, 6, 40, 40, 64, 64, 64, "auto") == 6
    assert plan(1, 6, 80, 80, 64, 64, 64, "auto") == 6
    assert plan(1, 8, 256, 256, 128, 128, 64, "auto") == 6
    assert plan(2, 12, 40, 40, 64, 64, 64, "auto") == 6   # 24 sequences
    assert plan(5, 5, 40, 40, 64, 64, 64, "auto") == 3    # 25: the two-chunk mma.sync kernel
    # B8 sweep: 64 sequences, d_v = 128 -> mma.sync, one chunk per tile
    assert plan(8, 8, 256, 256, 128, 128, 64, "auto") == 2
    # 64 sequences at d = 64: fewer than 2 per SM -> mma.sync with two chunks per tile
    assert plan(8, 8, 64, 64, 64, 64, 64, "auto") == 3
    assert plan(32, 12, 40, 40, 64, 64, 32, "auto") == 2   # chunk 32: not the tcgen05 shape
    # explicit schedules
    assert plan(8, 8, 64, 64, 64, 64, 64, "fused_tcgen05") == 4
    assert plan(8, 8, 64, 64, 32, 64, 64, "fused_tcgen05") == 3  # not its shape
    assert plan(8, 8, 64, 64, 128, 128, 64, "fused_tcgen05") == 4  # d_k = d_v = 128: value-half tiles
    assert plan(8, 8, 64, 64, 128, 64, 64, "fused_tcgen05") == 3  # d_k != d_v: not its shape
    assert plan(64, 8, 64, 64, 128, 128, 64, "auto") == 2  # AUTO keeps d=128 on mma.sync
    # d = 128 doubles the chained kernel's tiles (two value halves per chunk):
    # 2^30 chunk tiles give 2^31, past its 32-bit tile index
    assert plan(16384, 64, 256, 256, 128, 128, 64, "fused_tcgen05") == 2
    assert plan(8192, 64, 256, 256, 128, 128, 64, "fused_tcgen05") == 4
    assert plan(16384, 64, 256, 256, 64, 64, 64, "fused_tcgen05") == 4
    assert plan(32, 12, 40, 40, 64, 64, 64, "fused") == 2
    assert plan(8, 8, 256, 256, 128, 128, 64, "walk_tcgen05") == 5
    assert plan(8, 8, 64, 64, 32, 64, 64, "walk_tcgen05") == 5
    assert plan(8, 8, 64, 64, 64, 32, 64, "walk_tcgen05") == 3  # d_v = 32: not a walk shape
    assert plan(1, 1, 8, 8, 16, 16, 16, "three_phase") == 0
    assert plan(1, 1, 8, 8, 16, 16, 16, "three_phase_mma") == 6
    assert plan(1, 1, 8, 8, 16, 16, 16, "three_phase_simt") == 1
    # invalid arguments
    assert lib.gtr_gla_plan(1, 1, 8, 8, 16, 16, 16, 9, 148) == -1
    assert lib.gtr_gla_plan(1, 1, 8, 8, 24, 16, 16, 0, 148) == -1
    assert lib.gtr_gla_plan(1, 1, 8, 8, 16, 16, 16, 0, 0) == -1


def test_debug_hook_validates_spin_limit(lib):
    """The test hook's spin limit bounds only the wait for a predecessor's
    boundary state and must be positive; waits for a CTA's own tensor-core
    work have a fixed bound the caller cannot lower."""
    cdll = lib.load()
    args = [A, 2 * A, 3 * A, 4 * A, 1, 2, 16, 16, 64, 64, 0, 64, 4, 1, 1]
    for bad in (0, -1):
        assert cdll.gtr_gla_debug_forward_fused(*args, bad, 5 * A, 0) == 1
        assert "spin_limit" in lib.last_error()
    assert cdll.gtr_gla_debug_forward_fused(*args[:12], 2, 1, 1, 100, 5 * A, 0) == 1  # schedule


def test_noalloc_error_paths_set_text(lib):
    """Every refusal of the no-allocation entry point names its reason."""
    cases = [
        (dict(q=None), 1, "null"),
        (dict(direction=7), 1, "direction"),
        (dict(B=-1), 1, "negative"),
        (dict(d_k=48), 2, "d_k"),
        (dict(chunk=128), 2, "chunk"),
        (dict(q=A + 8), 3, "aligned"),
        (dict(out=A + 512), 4, "overlaps"),
        (dict(B=64, heads=64, grid_h=64, grid_w=64, d_k=128, d_v=128, out=1 << 40), 2, "16 MiB"),
    ]
    for kw, want, text in cases:
        args = dict(q=A, k=2 * A, v=3 * A, g=4 * A, B=1, heads=2, grid_h=4, grid_w=4, d_k=16,
                    d_v=16, direction=0, chunk=16, out=5 * A, stream=0)
        args.update(kw)
        assert lib.gtr_gla_forward_noalloc(**args) == want, kw
        assert text in lib.last_error(), (kw, lib.last_error())


def test_host_entry_alias_check(lib):
    """The host-buffer entry point refuses an output that overlaps an input
    before it touches the device."""
    import torch
    q = torch.zeros((1, 16, 2, 16), dtype=torch.float16)
    g = torch.zeros((1, 16, 2, 16), dtype=torch.float32)
    st = lib.gtr_gla_forward_host(q, q, q, g, 1, 2, 4, 4, 16, 16, 0, 16, q, 0)
    assert st == 4 and "overlaps" in lib.last_error()


def test_state_and_gated_entry_points_validate(lib):
    """Argument checks of the state-carrying and the gated forward, before
    any device work (fake, aligned addresses)."""
    base = dict(q=A, k=2 * A, v=3 * A, g=4 * A, B=1, heads=2, grid_h=4, grid_w=4, d_k=64, d_v=64,
                direction=0, chunk=64, out=5 * A, stream=0)

    def state(**kw):
        a = dict(base, S0=6 * A, SN=7 * A)
        a.update(kw)
        return lib.gtr_gla_forward_state(**a)

    assert state(d_k=16) == 2 and "chunk 64" in lib.last_error()
    assert state(chunk=32) == 2
    assert state(d_v=32) == 2
    assert state(q=None) == 1
    assert state(S0=6 * A + 4) == 3
    assert state(SN=7 * A + 8) == 3
    assert state(SN=A) == 4            # SN over q
    assert state(SN=6 * A + 256) == 4  # SN partly over S0
    assert state(S0=5 * A) == 4        # out over S0

    def gated(**kw):
        a = dict(base, gate=6 * A, norm_weight=7 * A, norm_eps=1e-5)
        a.update(kw)
        return lib.gtr_gla_forward_gated(**a)

    assert gated(d_v=128) == 2 and "d_v = 64" in lib.last_error()
    assert gated(gate=None) == 1
    assert gated(norm_weight=None) == 1
    assert gated(norm_eps=-1.0) == 1
    assert gated(norm_eps=float("nan")) == 1
    assert gated(gate=6 * A + 2) == 3
    assert gated(out=6 * A) == 4


def test_sswiglu_entry_point_validates(lib):
    args = dict(a=A, v=2 * A, w=3 * A, bias=4 * A, B=1, grid_h=4, grid_w=4, C=64, out=5 * A, stream=0)

    def call(**kw):
        a = dict(args)
        a.update(kw)
        return lib.gtr_sswiglu_forward(**a)

    assert call(C=12) == 2 and "multiple of 8" in lib.last_error()
    assert call(B=-1) == 1
    assert call(a=None) == 1
    assert call(w=None) == 1
    assert call(a=A + 8) == 3
    assert call(w=3 * A + 2) == 3
    assert call(out=A + 64) == 4
    assert call(out=3 * A) == 4
    # grid limits of the launch: B along z, 32-channel groups along y
    assert call(B=65536) == 2 and "too large" in lib.last_error()
    assert call(C=65536 * 32 + 8) == 2
    before = lib.gtr_gla_launch_count()
    assert call(B=0) == 0 and call(grid_h=0) == 0 and call(C=0) == 0
    assert lib.gtr_gla_launch_count() == before
