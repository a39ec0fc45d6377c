"""GPU tests of the debugging aids: guard bands after every workspace region
(MUON_GUARD_BANDS=1) and the bounds-checking build (libmuon_b200_debug.so,
device checks of every tile a GEMM role takes).  Both are chosen when the
library is loaded, so each runs in a child process; its results are compared
bitwise with the ordinary library's in this process, and the bounds checks are
made to fire by a host-side injection (tile indices past the end of a grid),
which they stop before any memory access."""

import json
import os
import subprocess
import sys

import pytest

import muon_newton_schulz_02_b200 as muon

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, shapes, ns_steps, entry point): the chained launch, one launch per phase
# (short side above 1024), ragged shapes next to the fused kernels, no iteration,
# and NS5 alone
CASES = [
    ("chain", [(768, 768), (768, 3072), (3072, 768)], 5, "step"),
    ("per_phase", [(1100, 1100), (1100, 2000)], 5, "step"),
    ("ragged", [(300, 700), (1000, 300), (260, 1030), (129, 127), (90, 400)], 5, "step"),
    ("no_iteration", [(512, 768), (640, 384)], 0, "step"),
    ("orthogonalize", [(384, 1024), (1024, 640)], 5, "orthogonalize"),
]

# Runs CASES with the library already chosen; returns {name: [sha1 of results, guard bytes changed]}.
RUN = r'''
import hashlib, torch
def run_cases(muon, cases, guards):
    dev = torch.device("cuda:0")
    out = {}
    for name, shapes, ns, entry in cases:
        gen = torch.Generator().manual_seed(len(name) * 1000 + len(shapes))
        W = [(torch.randn(*s, generator=gen) * 0.02).to(dev) for s in shapes]
        g = [torch.randn(*s, generator=gen).to(dev) for s in shapes]
        b = [(torch.randn(*s, generator=gen) * 0.1).to(dev) for s in shapes]
        if entry == "step":
            muon.step(W, g, b, lr=0.02, mu=0.95, ns_steps=ns)
            res = W + b
        else:
            res = muon.orthogonalize(g, ns_steps=ns)
        torch.cuda.synchronize()
        assert muon.sync_status() == 0, muon.last_error()
        h = hashlib.sha1()
        for t in res:
            h.update(t.cpu().numpy().tobytes())
        out[name] = [h.hexdigest(), muon.guard_check() if guards else 0]
    return out
'''


def _reference():
    ns = {}
    exec(RUN, ns)
    return ns["run_cases"](muon, CASES, False)


def _child(code, env_extra):
    env = dict(os.environ, **env_extra)
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


def test_guard_bands_stay_intact_and_results_do_not_change():
    code = RUN + f'''
import json, sys
sys.path.insert(0, {ROOT!r})
import muon_newton_schulz_02_b200 as muon
print(json.dumps(run_cases(muon, {CASES!r}, True)))
'''
    got = _child(code, {"MUON_GUARD_BANDS": "1"})
    ref = _reference()
    for name, _, _, _ in CASES:
        digest, changed = got[name]
        assert changed == 0, f"{name}: {changed} guard-band bytes were overwritten"
        assert digest == ref[name][0], f"{name}: results differ with guard bands"


def test_bounds_checking_build_gives_the_same_results_and_stops_out_of_range_tiles():
    code = RUN + f'''
import json, sys, torch
sys.path.insert(0, {ROOT!r})
import muon_newton_schulz_02_b200 as muon
muon.LIB_PATH = muon.DEBUG_LIB_PATH
res = run_cases(muon, {CASES!r}, False)
# injection: the next GEMM launch of one phase gets a tile index past the end
# of its grid for every cluster; the checks stop it before any memory access
dev = torch.device("cuda:0")
W = [torch.zeros(1100, 1100, device=dev)]
g = [torch.ones(1100, 1100, device=dev)]
b = [torch.zeros(1100, 1100, device=dev)]
muon.debug_set(32, 20_000_000)
try:
    muon.step(W, g, b, lr=0.02, mu=0.95)
    res["injected"] = [muon.sync_status(), muon.last_error()]
finally:
    muon.debug_set(0, 0)
# the context is still usable, and the next calls give the same results again
again = run_cases(muon, {CASES[:2]!r}, False)
res["again"] = [again[n][0] for n in sorted(again)]
res["loaded"] = [l.split()[-1] for l in open("/proc/self/maps") if "libmuon_b200" in l]
print(json.dumps(res))
'''
    got = _child(code, {})
    ref = _reference()
    for name, _, _, _ in CASES:
        assert got[name][0] == ref[name][0], f"{name}: the bounds-checking build gives other results"
    status, msg = got["injected"]
    assert status == -6 and "bounds" in msg, (status, msg)      # MUON_ERR_DEVICE
    assert got["again"] == [ref[n][0] for n in sorted(["chain", "per_phase"])]
    assert any(p.endswith("libmuon_b200_debug.so") for p in got["loaded"])
