"""gla_chunk_fwd_noalloc: the chunked forward for callers that cannot allocate
device memory (a runtime that owns all device memory in its own pool, a
plugin host that forbids cudaMalloc, a path that cannot take the implicit
synchronisation of an allocation).  It uses libgla's built-in scratch array
instead of a caller workspace.

The new entry point is called through the C ABI (ctypes, raw pointers) twice
in a row on different inputs, and each result is compared with the existing
gla_chunk_fwd given a PyTorch-allocated workspace, and with the fp64 oracle
on sampled heads, within the same tolerances as the other forward tests.
The shapes use the segmented path, so the scratch array is really used; the
second call reuses what the first left in it.  This file is named to be
collected last and needs no state from other tests, so it passes alone in a
fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_simple_b200 as gla
from linear_attention_simple_b200 import inputs
from oracle import recurrent
from tolerances import REL_BF16, REL_STATE, assert_bf16_close, rel_l2

pytestmark = pytest.mark.gpu

UNSUPPORTED = 2


@pytest.fixture(scope="module")
def L():
    from linear_attention_simple_b200 import build
    build.build()
    return gla.lib()


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _noalloc_call(L, d, o, sf):
    B, T, H, dk = d["q"].shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.gla_chunk_fwd_noalloc(_p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["a"]), _p(d["s0"]),
                                   _p(o), _p(sf), B, T, H, dk, 192, 0, dk ** -0.5, 0, stream)


def test_noalloc_matches_workspace_forward_on_two_calls(L):
    B, T, H = 1, 3000, 4                       # 24 chunks, 4 units -> 24 segments
    assert 0 < gla.gla_chunk_workspace_bytes(B, T, H) <= gla_scratch_bytes()
    for seed in (401, 402):                     # two calls in a row, different inputs
        d = inputs.chunk_inputs(B, T, H, seed=seed, device="cuda", s0_std=0.1)
        o = torch.full((B, T, H, 192), float("nan"), dtype=torch.bfloat16, device="cuda")
        sf = torch.full((B, H, 96, 192), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_call(L, d, o, sf) == 0
        ro, rs = gla.gla_chunk_fwd(d["q"], d["k"], d["v"], d["a"], s0=d["s0"])
        torch.cuda.synchronize()
        f = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
        assert rel_l2(f(o), f(ro)) <= REL_BF16
        assert rel_l2(f(sf), f(rs)) <= REL_STATE
        assert gla.gla_get_device_status() == 0
        # and against the oracle on two sampled heads
        hs = [0, H - 1]
        sl = lambda x: f(x[:, :, hs])  # noqa: E731
        o_ref, s_ref = recurrent.fwd(sl(d["q"]), sl(d["k"]), sl(d["v"]), f(d["a"][:, :, hs]), f(d["s0"][:, hs]))
        r = assert_bf16_close(sl(o), o_ref, "o (no-alloc) vs oracle")
        es = rel_l2(f(sf[:, hs]), s_ref)
        assert es <= REL_STATE, "S_T rel L2 %.3g" % es
        print("no-alloc vs oracle: o rel %.3g raw-max %.3g beyond-rounding %.3g, S_T rel %.3g" % (r + (es,)))


def test_noalloc_rejects_shapes_beyond_the_scratch_size(L):
    B, T, H = 1, 65536, 16                      # needs about 10.6 MB of scratch
    assert gla.gla_chunk_workspace_bytes(B, T, H) > gla_scratch_bytes()
    # No tensor pointers at all: the size check comes first, so the call is
    # rejected before anything could be launched (a regression would stop at
    # the null-pointer check, never at a kernel).
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = L.gla_chunk_fwd_noalloc(None, None, None, None, None, None, None, B, T, H, 96, 192, 0,
                                 96 ** -0.5, 0, stream)
    assert st == UNSUPPORTED


def gla_scratch_bytes():
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "include", "gla.h")).read()
    m = re.search(r"#define GLA_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", hdr)
    return int(m.group(1)) << int(m.group(2))
