"""The checking build (libgla_debug.so, -DGLA_DEBUG_BOUNDS).

CPU part (no GPU): the checking build compiles from the same sources, loads,
reports its build flag (the normal build reports none), exports every
function include/gla.h declares, and rejects bad arguments on the host with
the same status codes as the normal build (fake pointers, never
dereferenced: validation fails first).

GPU part: a child process with GLA_DEBUG_BOUNDS=1 (so the package loads the
checking build, and only it) runs small in-bounds cases through the public
API -- the status word stays 0 and the results match the fp64 oracle -- and
then inputs that violate a stated precondition (a log-decay a_t > 0, a
non-finite q, a NaN decay in a decode step): each call completes without a
fault, GLA_ERR_INVALID_ARG is recorded, and the context keeps working.
"""
import ctypes
import os
import subprocess
import sys

import pytest

import linear_attention_simple_b200 as gla
from test_boundary import declared_functions

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, MISALIGNED = range(4)
P = ctypes.c_void_p


@pytest.fixture(scope="module")
def libs():
    from linear_attention_simple_b200 import build
    build.build()
    build.build(debug=True)
    return gla.declare(ctypes.CDLL(gla.LIB_PATH)), gla.declare(ctypes.CDLL(gla.LIB_DEBUG_PATH))


def test_build_flags(libs):
    normal, debug = libs
    assert normal.gla_build_flags() == 0
    assert debug.gla_build_flags() == gla.GLA_BUILD_DEBUG_BOUNDS


def test_checking_build_exports_every_declared_symbol(libs):
    _, debug = libs
    for name in declared_functions():
        assert hasattr(debug, name), "libgla_debug.so does not export %s" % name


def test_checking_build_validates_like_the_normal_build(libs):
    def fwd(L, q=0x1000, a=0x4000, o=0x5000, B=1, T=128, H=1, dk=96, scale=96 ** -0.5):
        return L.gla_chunk_fwd(P(q), P(0x2000), P(0x3000), P(a), None, P(o), None, None, 0, B, T, H, dk, 192,
                               0, scale, 0, None)

    def dec(L, ns=4, N=4, state=0x1000):
        return L.gla_decode_step(P(state), None, ns, P(0x2000), P(0x3000), P(0x4000), P(0x5000), P(0x6000), N, 16,
                                 96, 192, 96 ** -0.5, None)

    for L in libs:
        assert fwd(L, q=None) == INVALID
        assert fwd(L, dk=64) == UNSUPPORTED
        assert fwd(L, a=0x4002) == MISALIGNED
        assert fwd(L, scale=-1.0) == INVALID
        assert fwd(L, B=0) == OK
        assert dec(L, ns=3) == INVALID
        assert dec(L, state=None) == INVALID


_CHILD = r'''
import numpy as np, torch
import linear_attention_simple_b200 as gla
from linear_attention_simple_b200 import inputs
from oracle import recurrent
assert gla.gla_build_flags() == gla.GLA_BUILD_DEBUG_BOUNDS, "the checking build is not the one loaded"
f = lambda t: t.detach().float().cpu().numpy().astype(np.float64)
rel = lambda x, r: float(np.linalg.norm(x - r) / max(np.linalg.norm(r), 1e-300))

# in bounds, preconditions met: nothing recorded, results as the oracle's
d = inputs.chunk_inputs(2, 300, 3, seed=71, device="cuda", s0_std=0.1, with_dO=True)
o, sf = gla.gla_chunk_fwd(d["q"], d["k"], d["v"], d["a"], s0=d["s0"])
g = gla.gla_chunk_bwd(d["q"], d["k"], d["v"], d["a"], d["dO"], s0=d["s0"])
assert gla.gla_get_device_status() == 0
ro, rs = recurrent.fwd(f(d["q"]), f(d["k"]), f(d["v"]), f(d["a"]), f(d["s0"]))
assert rel(f(o), ro) <= 1e-2 and rel(f(sf), rs) <= 5e-3
rg = recurrent.bwd(f(d["q"]), f(d["k"]), f(d["v"]), f(d["a"]), f(d["dO"]), f(d["s0"]))
for got, ref in zip(g, rg):
    assert rel(f(got), ref) <= 1e-2
dec = inputs.decode_inputs(8, 2, seed=72, device="cuda")[0]
st0 = f(dec["state"])
od = gla.gla_decode_step(dec["state"], dec["q"], dec["k"], dec["v"], dec["a"])
assert gla.gla_get_device_status() == 0
rst, rod = recurrent.decode(st0, f(dec["q"]), f(dec["k"]), f(dec["v"]), f(dec["a"]))
assert rel(f(dec["state"]), rst) <= 1e-5 and rel(f(od), rod) <= 1e-5
fr = inputs.front_inputs(1, 40, 256, seed=73, device="cuda")
y = gla.conv1d_silu_causal(fr["x"], fr["w"])
assert gla.gla_get_device_status() == 0

# a_t > 0 somewhere: reported, no fault
bad = d["a"].clone()
bad[1, 17, 2] = 0.25
gla.gla_chunk_fwd(d["q"], d["k"], d["v"], bad, s0=d["s0"])
assert gla.gla_get_device_status() == 1, "a > 0 not reported (forward)"
gla.gla_chunk_bwd(d["q"], d["k"], d["v"], bad, d["dO"], s0=d["s0"])
assert gla.gla_get_device_status() == 1, "a > 0 not reported (backward)"
# a non-finite q: reported
qn = d["q"].clone()
qn[0, 5, 1, 7] = float("inf")
gla.gla_chunk_fwd(qn, d["k"], d["v"], d["a"], s0=d["s0"])
assert gla.gla_get_device_status() == 1, "inf in q not reported"
# a NaN decay in a decode step: reported
an = dec["a"].clone()
an[3, 1] = float("nan")
gla.gla_decode_step(dec["state"], dec["q"], dec["k"], dec["v"], an)
assert gla.gla_get_device_status() == 1, "NaN decay not reported (decode)"

# the context is still usable and clean afterwards
o2, _ = gla.gla_chunk_fwd(d["q"], d["k"], d["v"], d["a"], s0=d["s0"])
assert gla.gla_get_device_status() == 0
assert torch.equal(o2, o)
print("checking build ok")
'''


@pytest.mark.gpu
def test_checking_build_on_the_gpu():
    from linear_attention_simple_b200 import build
    build.build(debug=True)
    env = dict(os.environ, GLA_DEBUG_BOUNDS="1", PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    r = subprocess.run([sys.executable, "-c", _CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    print(r.stdout[-2000:], r.stderr[-4000:])
    assert r.returncode == 0, r.stderr[-4000:]
    assert "checking build ok" in r.stdout
