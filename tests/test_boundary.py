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


def test_training_pair_validation(L):
    saved = gla.gla_chunk_saved_state_bytes(1, 300, 2)
    assert saved == 2 * 3 * 2 * 96 * 192 * 2
    assert gla.gla_chunk_saved_state_bytes(1, 300, 2, dk=64) == 0
    assert 0 < gla.gla_chunk_workspace_bytes(8, 2048, 16, for_bwd=True, from_saved=True) < \
        gla.gla_chunk_workspace_bytes(8, 2048, 16, for_bwd=True)

    def fwd(q=0x1000, o=0x5000, sv=0x9000, svb=saved, dt=0, T=300):
        return L.gla_chunk_fwd_train(P(q), P(0x2000), P(0x3000), P(0x4000), None, P(o), None, P(sv), svb, None, 0,
                                     1, T, 2, 96, 192, 0, 96 ** -0.5, dt, None)
    assert fwd(sv=None) == INVALID
    assert fwd(svb=saved - 16) == INVALID
    assert fwd(sv=0x9008) == MISALIGNED
    assert fwd(dt=1) == UNSUPPORTED
    assert fwd(q=None) == INVALID

    def bwd(sv=0x9000, svb=saved, sf=None, dsT=None, dO=0x6000, ws=0xA000, wsb=1 << 30):
        return L.gla_chunk_bwd_saved(P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(sv), svb, P(sf), P(dO), P(dsT),
                                     P(0x7000), P(0x7100), P(0x7200), P(0x7300), None, P(ws), wsb, 1, 300, 2, 96, 192,
                                     0, 96 ** -0.5, 0, None)
    assert bwd(sv=None) == INVALID
    assert bwd(svb=saved - 1) == INVALID
    assert bwd(dsT=0xB000) == INVALID               # dS_T given without the final state
    assert bwd(dO=None) == INVALID
    assert bwd(ws=None, wsb=0) == INVALID
    assert bwd(sf=0xB004, dsT=0xB000) == MISALIGNED


def test_decode_validation(L):
    def dec(state=0x1000, slot=None, ns=4, q=0x2000, k=0x3000, v=0x4000, a=0x5000, o=0x6000, N=4,
            H=16, dk=96, dv=192, scale=96 ** -0.5):
        return L.gla_decode_step(P(state), P(slot), ns, P(q), P(k), P(v), P(a), P(o), N, H, dk, dv,
                                 scale, None)
    assert dec(state=None) == INVALID
    assert dec(o=None) == INVALID
    assert dec(dk=64) == UNSUPPORTED
    assert dec(N=-1) == INVALID
    assert dec(scale=0.0) == INVALID
    assert dec(state=0x1004) == MISALIGNED
    assert dec(slot=0x7002) == MISALIGNED
    assert dec(ns=-1) == INVALID
    assert dec(ns=3) == INVALID                 # identity slots need N_slots >= N
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
    # eps only matters with LayerNorm: without it the call gets past the eps
    # check to the (later) width check; nothing here reaches a launch
    assert conv(ln=0, eps=0.0, W=3) == UNSUPPORTED
    assert conv(ln=1, eps=0.0, W=3) == INVALID
    assert conv(csi=0x4000, cso=0x4000) == INVALID
    assert conv(y=0x3002) == MISALIGNED
    assert conv(B=0) == OK


def test_varlen_validation(L):
    def varlen(q=0x1000, k=0x2000, v=0x3000, a=0x4000, cu=0x5000, N=2, s0=None, o=0x6000, sf=None,
               ws=None, wsb=0, total=256, H=2, dk=96, dv=192, ld=0, scale=96 ** -0.5, dt=0):
        return L.gla_chunk_fwd_varlen(P(q), P(k), P(v), P(a), P(cu), N, P(s0), P(o), P(sf), P(ws), wsb, total,
                                      H, dk, dv, ld, scale, dt, None)
    assert varlen(N=-1) == INVALID
    assert varlen(N=70000) == UNSUPPORTED
    assert varlen(dt=1) == UNSUPPORTED           # bf16 only
    assert varlen(cu=None) == INVALID
    assert varlen(o=None) == INVALID
    assert varlen(q=None) == INVALID
    assert varlen(dk=64) == UNSUPPORTED
    assert varlen(s0=0x7008) == MISALIGNED
    assert varlen(ws=0x7004, wsb=4096) == MISALIGNED
    assert varlen(N=0) == OK
    # the segment scratch: none for a short total, grows with the tokens
    assert gla.gla_chunk_varlen_workspace_bytes(8, 256, 16) == 0
    small = gla.gla_chunk_varlen_workspace_bytes(8, 16384, 16)
    assert small > 0 and gla.gla_chunk_varlen_workspace_bytes(8, 65536, 16) >= small
    assert gla.gla_chunk_varlen_workspace_bytes(8, 16384, 16, dk=64) == 0


def test_conv_decode_and_backward_validation(L):
    def dec(x=0x1000, slot=None, ns=4, ln=1, g=None, b=None, eps=1e-5, w=0x2000, bias=None, cs=0x3000, y=0x4000,
            N=4, D=3072, W=4):
        return L.conv1d_silu_decode_step(P(x), P(slot), ns, ln, P(g), P(b), eps, P(w), P(bias), P(cs), P(y), N, D,
                                         W, None)
    assert dec(x=None) == INVALID
    assert dec(cs=None) == INVALID
    assert dec(W=3) == UNSUPPORTED
    assert dec(D=12) == UNSUPPORTED
    assert dec(eps=-1.0) == INVALID
    assert dec(cs=0x3004) == MISALIGNED
    assert dec(ns=2) == INVALID                 # identity slots need N_slots >= N
    assert dec(N=0) == OK

    need = gla.conv1d_silu_causal_bwd_workspace_bytes(1, 64, 3072)
    assert need > 0
    assert gla.conv1d_silu_causal_bwd_workspace_bytes(1, 64, 3072, 3) == 0

    def bwd(x=0x1000, ln=1, g=None, b=None, eps=1e-5, w=0x2000, bias=None, csi=None, dy=0x3000, dx=0x4000,
            dw=0x5000, dbias=None, dg=None, db=None, dcs=None, ws=0x6000, wsb=need, B=1, T=64, D=3072, W=4):
        return L.conv1d_silu_causal_bwd(P(x), ln, P(g), P(b), eps, P(w), P(bias), P(csi), P(dy), P(dx), P(dw),
                                        P(dbias), P(dg), P(db), P(dcs), P(ws), wsb, B, T, D, W, None)
    assert bwd(dw=None) == INVALID
    assert bwd(dy=None) == INVALID
    assert bwd(B=70000) == UNSUPPORTED
    assert bwd(W=5) == UNSUPPORTED
    assert bwd(ws=None) == INVALID
    assert bwd(wsb=need - 16) == INVALID
    assert bwd(dx=0x4008) == MISALIGNED
    assert bwd(dcs=0x7004) == MISALIGNED


def test_segment_calls_validation(L):
    """gla_segment_state_fwd / _bwd, gla_state_fold, gla_segment_workspace_bytes:
    every case below is rejected on the host before any device work."""
    need = gla.gla_segment_workspace_bytes(1, 1000, 2)
    assert need > 0
    assert gla.gla_segment_workspace_bytes(1, 1000, 2, 64, 192) == 0
    assert gla.gla_segment_workspace_bytes(0, 1000, 2) == 0
    # more (batch, head) pairs or a shorter sequence never need more scratch per token
    assert gla.gla_segment_workspace_bytes(1, 8192, 16) >= gla.gla_segment_workspace_bytes(1, 4096, 16)

    def seg(fn, u=0x1000, y=0x2000, a=0x3000, s=0x4000, g=0x5000, ws=0x6000, wsb=need, B=1, T=1000, H=2,
            dk=96, dv=192, ld=0, scale=96 ** -0.5, dt=0):
        if fn == "fwd":
            return L.gla_segment_state_fwd(P(u), P(y), P(a), P(s), P(g), P(ws), wsb, B, T, H, dk, dv, ld, dt,
                                           None)
        return L.gla_segment_state_bwd(P(u), P(y), P(a), P(s), P(g), P(ws), wsb, B, T, H, dk, dv, ld, scale,
                                       dt, None)
    for fn in ("fwd", "bwd"):
        assert seg(fn, u=None) == INVALID
        assert seg(fn, a=None) == INVALID
        assert seg(fn, s=None) == INVALID         # the segment state is required
        assert seg(fn, ws=None) == INVALID
        assert seg(fn, wsb=need - 16) == INVALID
        assert seg(fn, dk=64) == UNSUPPORTED
        assert seg(fn, dt=1) == UNSUPPORTED       # bf16 only
        assert seg(fn, T=-1) == INVALID
        assert seg(fn, s=0x4004) == MISALIGNED
        assert seg(fn, g=0x5008) == MISALIGNED
        assert seg(fn, y=0x2002) == MISALIGNED
        assert seg(fn, B=0) == OK
    assert seg("bwd", scale=0.0) == INVALID

    def fold(s=0x1000, g=0x2000, n=3, rev=0, s_in=None, out=0x3000, units=4, dk=96, dv=192):
        return L.gla_state_fold(P(s), P(g), n, rev, P(s_in), P(out), units, dk, dv, None)
    assert fold(n=-1) == INVALID
    assert fold(units=-1) == INVALID
    assert fold(out=None) == INVALID
    assert fold(s=None) == INVALID
    assert fold(g=None) == INVALID
    assert fold(dk=64) == UNSUPPORTED
    assert fold(s=0x1008) == MISALIGNED
    assert fold(g=0x2002) == MISALIGNED           # g needs 4-byte alignment only
    assert fold(s_in=0x4004) == MISALIGNED
    assert fold(units=0) == OK


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


def test_bindings_reject_host_tensors(L):
    """Every binding refuses CPU tensors before any call into the library:
    there is no host fallback for any step."""
    import torch
    bf = lambda *s: torch.zeros(s, dtype=torch.bfloat16)  # noqa: E731
    f32 = lambda *s: torch.zeros(s, dtype=torch.float32)  # noqa: E731
    B, T, H = 1, 4, 2
    q, k, v, a = bf(B, T, H, 96), bf(B, T, H, 96), bf(B, T, H, 192), f32(B, T, H)
    calls = [
        lambda: gla.gla_chunk_fwd(q, k, v, a),
        lambda: gla.gla_chunk_bwd(q, k, v, a, bf(B, T, H, 192)),
        lambda: gla.gla_decode_step(f32(2, H, 96, 192), bf(2, H, 96), bf(2, H, 96), bf(2, H, 192), f32(2, H)),
        lambda: gla.conv1d_silu_causal(bf(1, T, 64), f32(64, 4)),
        lambda: gla.conv1d_silu_decode_step(bf(2, 64), f32(64, 4), f32(2, 3, 64)),
        lambda: gla.conv1d_silu_causal_bwd(bf(1, T, 64), f32(64, 4), bf(1, T, 64)),
        lambda: gla.gla_chunk_fwd_varlen(bf(T, H, 96), bf(T, H, 96), bf(T, H, 192), f32(T, H),
                                         torch.tensor([0, T], dtype=torch.int32)),
        lambda: gla.gla_segment_state_fwd(k, v, a),
        lambda: gla.gla_segment_state_bwd(q, bf(B, T, H, 192), a),
        lambda: gla.gla_state_fold(f32(2, B, H, 96, 192), f32(2, B, H)),
        lambda: gla.gla_chunk_fwd_noalloc(q, k, v, a),
    ]
    for call in calls:
        # rejected by the binding itself, not by the library (a GlaError would
        # mean host pointers reached libgla)
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()
