"""C-ABI checks that need no GPU: the library builds and loads, exports every
function include/muon.h declares, validates arguments on the host before any
CUDA call, and sizes its workspace as documented."""

import ctypes

import pytest

import __graft_entry__
import muon_newton_schulz_02_b200 as muon

INVALID, SHAPE = -1, -2


@pytest.fixture(scope="module")
def L():
    __graft_entry__.build()
    return muon.lib()


def test_exports_every_declared_function(L):
    names = muon.header_functions()
    assert {"muon_step", "muon_step_ex", "muon_orthogonalize", "muon_step_host", "muon_workspace_size",
            "muon_sync_status", "muon_last_error", "muon_release", "muon_profile_enable",
            "muon_profile_read", "muon_launch_count", "muon_debug_set"} <= set(names)
    for f in names:
        assert hasattr(L, f), f


def test_bounds_checking_build_exports_the_same_functions():
    # the twin library with device bounds checks (MUON_DEBUG_BOUNDS) loads on a
    # host without a GPU and exports every declared function too
    D = ctypes.CDLL(muon.DEBUG_LIB_PATH)
    for f in muon.header_functions():
        assert hasattr(D, f), f
    assert "muon_guard_check" in muon.header_functions()


def test_guard_check_is_refused_without_guard_bands(L):
    # guard bands are chosen at load time (MUON_GUARD_BANDS=1); without them the
    # hook refuses before touching any device
    assert L.muon_guard_check(None) == -7                # MUON_ERR_UNSUPPORTED


def _arr(n, v=1):
    return (ctypes.c_void_p * n)(*[ctypes.c_void_p(v)] * n)


def _shapes(*dims):
    return (ctypes.c_int64 * len(dims))(*dims)


def test_argument_errors_are_reported_before_any_launch(L):
    p = _arr(1)
    sh = _shapes(4, 8)
    assert L.muon_step(p, p, p, None, 1, 0.02, 0.95, 5, None) == INVALID
    assert "shapes" in muon.last_error()
    assert L.muon_step(p, p, p, sh, 0, 0.02, 0.95, 5, None) == INVALID
    assert L.muon_step(p, p, p, sh, 1, 0.02, 0.95, -1, None) == INVALID
    assert L.muon_step(p, p, p, _shapes(0, 8), 1, 0.02, 0.95, 5, None) == SHAPE
    assert L.muon_step(p, p, p, _shapes(4, -3), 1, 0.02, 0.95, 5, None) == SHAPE
    assert L.muon_step(None, p, p, sh, 1, 0.02, 0.95, 5, None) == INVALID
    assert L.muon_step(p, p, _arr(1, 0), sh, 1, 0.02, 0.95, 5, None) == INVALID
    assert "momentum_bufs[0]" in muon.last_error()
    assert L.muon_step_ex(p, p, p, sh, 1, 0.02, 0.95, 5, 3.4445, -4.775, 2.0315, 1e-7, 2, None) == INVALID
    assert L.muon_step_ex(p, p, p, sh, 1, 0.02, 0.95, 5, 3.4445, -4.775, 2.0315, -1.0, 1, None) == INVALID
    assert L.muon_orthogonalize(p, _arr(1, 0), sh, 1, 5, None) == INVALID
    assert L.muon_step_host(p, None, p, sh, 1, 0.02, 0.95, 5, None) == INVALID
    for bad_iters in (-1, 3):
        assert L.muon_step_fp8(p, p, p, sh, 1, 0.02, 0.95, 5, 3.4445, -4.775, 2.0315, 1e-7, 1, bad_iters, None) == INVALID
        assert "fp8_iters" in muon.last_error()
    assert L.muon_step_fp8(p, p, p, sh, 1, 0.02, 0.95, 5, 3.4445, -4.775, 2.0315, 1e-7, 2, 1, None) == INVALID


def _ws(shapes):
    flat = [v for s in shapes for v in s]
    return muon.lib().muon_workspace_size((ctypes.c_int64 * len(flat))(*flat), len(shapes))


def _expect_ws(shapes):
    """Layout documented in the C source: a fixed 4 KiB region of norm
    arrival counters, then per shape class (padded short side kp, long side
    lp, both multiples of 128) two bf16 iterates [B][kp][lp] and two bf16
    [B][kp][kp] matrices, then per-tile norm partials (64x128 tiles),
    per-matrix scales and per-matrix completion counters (of the chained
    launch), each region rounded to 1 KiB.  Matrices that a fused
    kernel runs whole (short side <= 128 and long side <= 512 on one CTA, or
    short side <= 256 and long side <= 256 on a CTA pair) take none."""
    up = lambda v, a: (v + a - 1) // a * a
    classes = {}
    for r, c in shapes:
        k, l = min(r, c), max(r, c)
        if (k <= 128 and up(l, 64) <= 512) or (k <= 256 and l <= 256):
            continue                      # fused single-CTA or CTA-pair kernel: no workspace
        classes.setdefault((up(k, 128), up(l, 128)), []).append((r, c))
    if not classes:
        return 4096
    off = 4096
    tiles = 0
    for (kp, lp), mats in classes.items():
        b = len(mats)
        off = up(off + b * kp * lp * 2, 1024)
        off = up(off + b * kp * lp * 2, 1024)
        off = up(off + b * kp * kp * 2, 1024)
        off = up(off + b * kp * kp * 2, 1024)
        tiles += b * (kp // 64) * (lp // 128)
    n = sum(len(v) for v in classes.values())
    off = up(off + tiles * 4, 1024)
    off = up(off + n * 4, 1024)
    off = up(off + n * 4, 1024)
    return off


@pytest.mark.parametrize("shapes", [
    [(128, 512)],
    [(768, 768)] * 4 + [(768, 3072), (3072, 768)],
    [(1, 1), (127, 129), (129, 127), (1000, 300)],
    [(128, 640), (129, 512), (256, 256), (64, 64)],
    [(256, 256), (200, 256), (257, 256), (256, 257)],
])
def test_workspace_size_matches_layout(L, shapes):
    assert _ws(shapes) == _expect_ws(shapes)


def test_guard_bands_add_one_band_after_every_region():
    # MUON_GUARD_BANDS=1 (read when the library loads, so in a child process):
    # 4 KiB after the counter region and after each of the four buffers per shape
    # class, the norm partials, the scales and the completion counters
    import json
    import os
    import subprocess
    import sys
    sets = [[(768, 768)] * 4 + [(768, 3072), (3072, 768)], [(1, 1), (127, 129), (129, 127), (1000, 300)]]
    code = f"""
import ctypes, json, sys
sys.path.insert(0, {muon.HERE + '/..'!r})
import muon_newton_schulz_02_b200 as muon
out = []
for shapes in {sets!r}:
    flat = [v for s in shapes for v in s]
    out.append(muon.lib().muon_workspace_size((ctypes.c_int64 * len(flat))(*flat), len(shapes)))
print(json.dumps(out))
"""
    env = dict(os.environ, MUON_GUARD_BANDS="1")
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr[-2000:]
    got = json.loads(res.stdout.strip().splitlines()[-1])
    up = lambda v, a: (v + a - 1) // a * a
    for shapes, ws in zip(sets, got):
        classes = {(up(min(r, c), 128), up(max(r, c), 128)) for r, c in shapes
                   if not ((min(r, c) <= 128 and up(max(r, c), 64) <= 512) or (min(r, c) <= 256 and max(r, c) <= 256))}
        bands = 1 + 4 * len(classes) + 3
        assert ws == _expect_ws(shapes) + bands * 4096, (shapes, ws)


def test_workspace_size_rejects_bad_input(L):
    assert _ws([(0, 4)]) == 0
    assert muon.lib().muon_workspace_size(None, 1) == 0


def test_many_matrices_split_into_groups(L):
    # more matrices than one launch holds: groups share the data region
    shapes = [(192, 192)] * 700
    one_group = _expect_ws([(192, 192)] * 320)
    got = _ws(shapes)
    assert got == one_group


def test_launch_count_and_debug_hooks_run_without_gpu(L):
    assert muon.launch_count() == 0
    muon.debug_set(0, 0)


def test_binding_marshals_pointers_and_shapes_in_one_pass():
    import torch
    P = [torch.zeros(3, 5), torch.zeros(7, 2)]
    G = [torch.ones(3, 5), torch.ones(7, 2)]
    B = [torch.full((3, 5), 2.0), torch.full((7, 2), 2.0)]
    pp, gp, bp, sh, n = muon._marshal_step(P, G, B, device_kind="cpu")
    assert n == 2 and list(sh) == [3, 5, 7, 2]
    assert [pp[i] for i in range(2)] == [t.data_ptr() for t in P]
    assert [gp[i] for i in range(2)] == [t.data_ptr() for t in G]
    assert [bp[i] for i in range(2)] == [t.data_ptr() for t in B]


@pytest.mark.parametrize("bad,msg", [
    (lambda torch: torch.zeros(3), "2-D"),
    (lambda torch: torch.zeros(3, 4, dtype=torch.float64), "contiguous float32"),
    (lambda torch: torch.zeros(4, 3).t(), "contiguous float32"),
])
def test_binding_rejects_bad_tensors_before_any_call(bad, msg):
    import torch
    t = bad(torch)
    with pytest.raises(ValueError, match=msg):
        muon._marshal_step([t], [t], [t], device_kind="cpu")
    with pytest.raises(ValueError, match="live on cuda"):
        muon._marshal_step([torch.zeros(3, 4)], [torch.zeros(3, 4)], [torch.zeros(3, 4)])
    with pytest.raises(ValueError, match="shapes differ"):
        muon._marshal_step([torch.zeros(3, 4)], [torch.zeros(4, 3)], [torch.zeros(3, 4)], device_kind="cpu")
    with pytest.raises(ValueError, match="equally long"):
        muon._marshal_step([torch.zeros(3, 4)], [], [torch.zeros(3, 4)], device_kind="cpu")
    with pytest.raises(ValueError, match="live on cuda"):
        muon.PreparedStep([torch.zeros(3, 4)], [torch.zeros(3, 4)], lr=0.02, mu=0.95)
