"""GPU parity of the front end's backward (LayerNorm -> causal conv -> SiLU)
against the fp64 oracle's backward (itself pinned by finite differences and
torch float64 autograd on the CPU).

Tolerances: dx is stored in bf16, so it takes the bf16 bound (rel L2 <= 1e-2,
max-abs <= 5e-2 beyond bf16 storage rounding; tests/tolerances.py).  dw,
dbias, dln_gamma, dln_beta and dconv_state_in are fp32 sums of fp32 terms
(inputs are the exact bf16 values), so their bound is rel L2 <= 1e-4.
"""
import numpy as np
import pytest
import torch

import linear_attention_simple_b200 as gla
from linear_attention_simple_b200 import inputs
from oracle import recurrent
from tolerances import assert_bf16_close, rel_l2

pytestmark = pytest.mark.gpu
REL_SUM = 1e-4


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.fixture(scope="module", autouse=True)
def _build():
    from linear_attention_simple_b200 import build
    build.build()
    gla.lib()


def _case(B, T, D, affine, hist, seed):
    d = inputs.front_inputs(B, T, D, seed=seed, device="cuda", with_state=hist)
    d["dy"] = inputs.randn((B, T, D), seed + 5, "cuda", dtype=torch.bfloat16)
    d["g"] = d["b"] = d["bias"] = None
    if affine:
        d["g"] = inputs.randn((D,), seed + 6, "cuda", std=0.5) + 1.0
        d["b"] = inputs.randn((D,), seed + 7, "cuda", std=0.5)
        d["bias"] = inputs.randn((D,), seed + 8, "cuda", std=0.5)
    return d


def _check(d, ln, want_hist=True):
    got = gla.conv1d_silu_causal_bwd(d["x"], d["w"], d["dy"], apply_ln=ln, ln_gamma=d["g"], ln_beta=d["b"],
                                     bias=d["bias"], conv_state_in=d["conv_state"])
    opt = lambda t: None if t is None else _np(t)  # noqa: E731
    ref = recurrent.ln_conv_silu_bwd(_np(d["x"]), _np(d["w"]), _np(d["dy"]), ln=ln, ln_gamma=opt(d["g"]),
                                     ln_beta=opt(d["b"]), bias=opt(d["bias"]), conv_state=opt(d["conv_state"]))
    rdx, rdw, rdb, rdg, rdbe, rdcs = ref
    assert_bf16_close(_np(got["dx"]), rdx, "dx")
    assert rel_l2(_np(got["dw"]), rdw) <= REL_SUM
    assert rel_l2(_np(got["dbias"]), rdb) <= REL_SUM
    if ln:
        assert rel_l2(_np(got["dln_gamma"]), rdg) <= REL_SUM
        assert rel_l2(_np(got["dln_beta"]), rdbe) <= REL_SUM
    else:
        assert float(np.abs(_np(got["dln_gamma"])).max()) == 0.0
    if want_hist:
        assert rel_l2(_np(got["dconv_state_in"]), rdcs) <= REL_SUM
    return got


@pytest.mark.parametrize("B,T,D,ln,affine,hist", [
    (1, 1, 8, True, False, False),
    (1, 2, 64, True, True, True),
    (2, 37, 256, True, True, True),
    (1, 300, 3072, True, True, True),
    (3, 129, 64, False, False, True),
    (2, 5, 512, True, False, True),
    (1, 130, 4096, True, True, True),
    (2, 200, 2056, True, True, True),
    (1, 700, 2048, True, False, True),
    (1, 7, 3072, False, True, True),
    (2, 160, 2560, True, False, False),
    (1, 90, 3064, True, True, False),
])
def test_front_bwd_parity(B, T, D, ln, affine, hist):
    """Up to D = 2,048 and above D = 3,072 a worker owns 4 channels; in
    between 8, in clusters of 2 CTAs (2,056 and 3,064: the channel units do
    not split evenly over the cluster; 2,560 and 3,072: they do)."""
    _check(_case(B, T, D, affine, hist, seed=70 + T + D), ln)


def test_front_bwd_full_size():
    """B = 1, T = 65,536, D = 3,072 (the long-context front end), every output
    against the full fp64 oracle."""
    _check(_case(1, 65536, 3072, False, False, seed=1007), True, want_hist=True)


def test_front_bwd_empty_and_workspace():
    D = 64
    x = torch.zeros((2, 0, D), dtype=torch.bfloat16, device="cuda")
    w = inputs.randn((D, 4), 80, "cuda")
    got = gla.conv1d_silu_causal_bwd(x, w, x)
    torch.cuda.synchronize()
    assert float(got["dw"].abs().max()) == 0.0 and float(got["dconv_state_in"].abs().max()) == 0.0
    d = _case(1, 300, D, False, False, seed=81)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(gla.GlaError):
        gla.conv1d_silu_causal_bwd(d["x"], d["w"], d["dy"], ws=small)
