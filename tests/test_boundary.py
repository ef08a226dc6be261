"""C-ABI boundary tests that need no GPU.

The library must load on a host without a GPU, export every function that
include/gla.h declares, and reject bad arguments on the host with the
documented status codes before any device work (fake pointers are used: they
are never dereferenced because validation fails first).
"""
import ctypes
import os
import re

import pytest

import linear_attention_simple_b200 as gla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, MISALIGNED, CUDA, TIMEOUT = range(6)


@pytest.fixture(scope="module")
def L():
    from linear_attention_simple_b200 import build
    build.build()
    return gla.lib()


def declared_functions():
    txt = open(os.path.join(ROOT, "include", "gla.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", txt)) - {"sizeof"})


def test_header_declares_the_four_hot_path_calls():
    names = declared_functions()
    for n in ("gla_chunk_fwd", "gla_chunk_bwd", "gla_decode_step", "conv1d_silu_causal"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), "libgla.so does not export %s" % name
    assert set(gla.EXPORTED_SYMBOLS) <= set(declared_functions())


def test_status_strings(L):
    for code, name in gla.STATUS.items():
        assert gla.gla_status_string(code) == name
    assert gla.gla_status_string(99) == "GLA_ERR_UNKNOWN"


def test_workspace_query(L):
    assert gla.gla_chunk_workspace_bytes(8, 2048, 16) >= 0
    assert gla.gla_chunk_workspace_bytes(8, 2048, 16, 64, 192) == 0      # unsupported dk
    assert gla.gla_chunk_workspace_bytes(0, 2048, 16) == 0
    small = gla.gla_chunk_workspace_bytes(1, 256, 1, for_bwd=True)
    big = gla.gla_chunk_workspace_bytes(1, 65536, 16, for_bwd=True)
    assert big >= small


P = ctypes.c_void_p


def _fwd(L, q=0x1000, k=0x2000, v=0x3000, a=0x4000, s0=None, o=0x5000, sf=None, ws=None,
         wsb=0, B=1, T=128, H=1, dk=96, dv=192, ld=0, scale=96 ** -0.5, dt=0):
    return L.gla_chunk_fwd(P(q), P(k), P(v), P(a), P(s0), P(o), P(sf), P(ws), wsb, B, T, H, dk,
                           dv, ld, scale, dt, None)


def test_chunk_fwd_validation(L):
    assert _fwd(L, q=None) == INVALID
    assert _fwd(L, a=None) == INVALID
    assert _fwd(L, dk=64) == UNSUPPORTED
    assert _fwd(L, dv=128) == UNSUPPORTED
    assert _fwd(L, dk=0) == INVALID
    assert _fwd(L, scale=0.0) == INVALID
    assert _fwd(L, scale=-1.0) == INVALID
    assert _fwd(L, scale=float("nan")) == INVALID
    assert _fwd(L, dt=7) == INVALID
    assert _fwd(L, T=-1) == INVALID
    assert _fwd(L, q=0x1001) == MISALIGNED
    assert _fwd(L, v=0x3008) == MISALIGNED
    assert _fwd(L, ld=100) == INVALID          # below the packed stride
    assert _fwd(L, ld=196) == MISALIGNED       # 392 bytes, not a multiple of 16
    assert _fwd(L, o=None) == INVALID
    assert _fwd(L, s0=0x6004) == MISALIGNED
    assert _fwd(L, B=0) == OK                  # nothing to do
    assert _fwd(L, H=0) == OK


def test_chunk_bwd_validation(L):
    def bwd(**kw):
        d = dict(q=0x1000, k=0x2000, v=0x3000, a=0x4000, s0=None, dO=0x5000, dsT=None,
                 gq=0x6000, gk=0x7000, gv=0x8000, ga=0x9000, gs0=None, ws=None, wsb=0, B=1,
                 T=128, H=1, dk=96, dv=192, ld=0, scale=96 ** -0.5, dt=0)
        d.update(kw)
        return L.gla_chunk_bwd(P(d["q"]), P(d["k"]), P(d["v"]), P(d["a"]), P(d["s0"]),
                               P(d["dO"]), P(d["dsT"]), P(d["gq"]), P(d["gk"]), P(d["gv"]),
                               P(d["ga"]), P(d["gs0"]), P(d["ws"]), d["wsb"], d["B"], d["T"],
                               d["H"], d["dk"], d["dv"], d["ld"], d["scale"], d["dt"], None)
    assert bwd(dO=None) == INVALID
    assert bwd(ga=None) == INVALID
    assert bwd(dt=1) == UNSUPPORTED            # fp32 backward is not provided
    assert bwd(dk=128) == UNSUPPORTED
    assert bwd(gq=0x6002) == MISALIGNED
    need = gla.gla_chunk_workspace_bytes(1, 128, 1, for_bwd=True)
    if need > 0:
        assert bwd(ws=None, wsb=0) == INVALID   # workspace missing
        assert bwd(ws=0xA000, wsb=need - 16) == INVALID
    assert bwd(B=0) == OK


def test_decode_validation(L):
    def dec(state=0x1000, slot=None, q=0x2000, k=0x3000, v=0x4000, a=0x5000, o=0x6000, N=4,
            H=16, dk=96, dv=192, scale=96 ** -0.5):
        return L.gla_decode_step(P(state), P(slot), P(q), P(k), P(v), P(a), P(o), N, H, dk, dv,
                                 scale, None)
    assert dec(state=None) == INVALID
    assert dec(o=None) == INVALID
    assert dec(dk=64) == UNSUPPORTED
    assert dec(N=-1) == INVALID
    assert dec(scale=0.0) == INVALID
    assert dec(state=0x1004) == MISALIGNED
    assert dec(slot=0x7002) == MISALIGNED
    assert dec(N=0) == OK


def test_conv_validation(L):
    def conv(x=0x1000, ln=1, g=None, b=None, eps=1e-5, w=0x2000, bias=None, csi=None, cso=None,
             y=0x3000, B=1, T=16, D=3072, W=4):
        return L.conv1d_silu_causal(P(x), ln, P(g), P(b), eps, P(w), P(bias), P(csi), P(cso),
                                    P(y), B, T, D, W, None)
    assert conv(x=None) == INVALID
    assert conv(w=None) == INVALID
    assert conv(W=3) == UNSUPPORTED
    assert conv(D=3070) == UNSUPPORTED
    assert conv(D=8192) == UNSUPPORTED
    assert conv(eps=0.0) == INVALID
    assert conv(ln=0, eps=0.0) != INVALID      # eps only matters with LayerNorm
    assert conv(csi=0x4000, cso=0x4000) == INVALID
    assert conv(y=0x3002) == MISALIGNED
    assert conv(B=0) == OK


def test_wait_limit_setter(L):
    assert L.gla_set_wait_limit_ns(5_000_000) == OK
    assert L.gla_set_wait_limit_ns(0) == OK


def test_no_gpu_reports_cuda_error_not_a_crash(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    out = ctypes.c_int(0)
    assert L.gla_get_device_status(None, ctypes.byref(out)) == CUDA
    assert L.gla_last_cuda_error() != 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(gla, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(gla, "_LIB", None)
    with pytest.raises(gla.GlaLibraryMissing):
        gla.lib()


def test_product_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "linear_attention_simple_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "gla_oracle" not in src, f
