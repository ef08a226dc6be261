"""libgla -- Simple Gated Linear Attention mixer for B200 (sm_100a).

Thin Python binding over the C ABI in ``include/gla.h``: the functions below
have the same names as the exported C entry points and only marshal
arguments (check dtypes/devices/strides, allocate outputs with PyTorch when
the caller passes none, pass raw pointers and the current CUDA stream).
Every step of the computation runs in the kernels of ``libgla.so``; there is
no CPU or PyTorch fallback.  Importing this package does not load the
library; the first call does, and raises ``GlaLibraryMissing`` when
``libgla.so`` has not been built (``python -m linear_attention_simple_b200.build``).
With ``GLA_DEBUG_BOUNDS=1`` in the environment the first call loads the
checking build ``libgla_debug.so`` instead (same ABI; input scans and index
checks that record GLA_ERR_INVALID_ARG in the device status word; built by
``python -m linear_attention_simple_b200.build --debug``).
"""
import ctypes
import os

import torch

__all__ = [
    "GlaError", "GlaLibraryMissing", "lib", "gla_status_string", "gla_launch_count",
    "gla_chunk_workspace_bytes", "gla_chunk_fwd", "gla_chunk_bwd", "gla_decode_step",
    "conv1d_silu_causal", "gla_get_device_status", "gla_set_wait_limit_ns",
    "gla_selftest_wait_timeout", "gla_trace_enable", "gla_trace_summary",
    "gla_chunk_fwd_noalloc", "conv1d_silu_decode_step", "conv1d_silu_causal_bwd",
    "conv1d_silu_causal_bwd_workspace_bytes", "gla_chunk_fwd_varlen", "gla_segment_workspace_bytes",
    "gla_segment_state_fwd", "gla_segment_state_bwd", "gla_state_fold", "gla_build_flags",
    "gla_chunk_varlen_workspace_bytes", "gla_chunk_saved_state_bytes", "gla_chunk_fwd_train",
    "gla_chunk_bwd_saved", "EXPORTED_SYMBOLS",
    "LIB_PATH", "LIB_DEBUG_PATH", "GLA_BUILD_DEBUG_BOUNDS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgla.so")
LIB_DEBUG_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgla_debug.so")
GLA_BUILD_DEBUG_BOUNDS = 1

EXPORTED_SYMBOLS = (
    "gla_status_string", "gla_last_cuda_error", "gla_launch_count",
    "gla_chunk_workspace_bytes", "gla_chunk_fwd", "gla_chunk_bwd", "gla_decode_step",
    "conv1d_silu_causal", "gla_get_device_status", "gla_set_wait_limit_ns",
    "gla_selftest_wait_timeout", "gla_trace_enable", "gla_trace_summary",
    "gla_chunk_fwd_noalloc", "conv1d_silu_decode_step", "conv1d_silu_causal_bwd",
    "conv1d_silu_causal_bwd_workspace_bytes", "gla_chunk_fwd_varlen", "gla_segment_workspace_bytes",
    "gla_segment_state_fwd", "gla_segment_state_bwd", "gla_state_fold", "gla_build_flags",
    "gla_chunk_varlen_workspace_bytes", "gla_chunk_saved_state_bytes", "gla_chunk_fwd_train",
    "gla_chunk_bwd_saved",
)

GLA_BF16, GLA_F32 = 0, 1
STATUS = {0: "GLA_OK", 1: "GLA_ERR_INVALID_ARG", 2: "GLA_ERR_UNSUPPORTED",
          3: "GLA_ERR_MISALIGNED", 4: "GLA_ERR_CUDA", 5: "GLA_ERR_TIMEOUT"}


class GlaLibraryMissing(RuntimeError):
    pass


class GlaError(RuntimeError):
    def __init__(self, fn, status, cuda_err=0):
        self.status = status
        self.cuda_error = cuda_err
        msg = "%s failed: %s" % (fn, STATUS.get(status, str(status)))
        if status == 4:
            msg += " (cudaError %d)" % cuda_err
        super().__init__(msg)


_LIB = None
_vp = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float


def lib():
    """Load libgla.so (once; libgla_debug.so when GLA_DEBUG_BOUNDS=1).
    Raises GlaLibraryMissing if it is not built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    debug = os.environ.get("GLA_DEBUG_BOUNDS", "0") not in ("", "0")
    path = LIB_DEBUG_PATH if debug else LIB_PATH
    if not os.path.exists(path):
        raise GlaLibraryMissing("%s not found; build it with `python -m linear_attention_simple_b200.build%s`"
                                % (path, " --debug" if debug else ""))
    _LIB = declare(ctypes.CDLL(path))
    return _LIB


def declare(L):
    """Set the ctypes signatures of every exported entry point on a loaded
    copy of the library (the normal or the checking build); returns L."""
    L.gla_status_string.restype = ctypes.c_char_p
    L.gla_status_string.argtypes = [_i]
    L.gla_last_cuda_error.restype = _i
    L.gla_launch_count.restype = ctypes.c_ulonglong
    L.gla_chunk_workspace_bytes.restype = ctypes.c_size_t
    L.gla_chunk_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i]
    L.gla_chunk_fwd.restype = _i
    L.gla_chunk_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                _i, _i, _i, _i, _i, _i64, _f, _i, _vp]
    L.gla_chunk_bwd.restype = _i
    L.gla_chunk_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _vp, ctypes.c_size_t, _i, _i, _i, _i, _i, _i64, _f, _i, _vp]
    L.gla_chunk_saved_state_bytes.restype = ctypes.c_size_t
    L.gla_chunk_saved_state_bytes.argtypes = [_i, _i, _i, _i, _i]
    L.gla_chunk_fwd_train.restype = _i
    L.gla_chunk_fwd_train.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp,
                                      ctypes.c_size_t, _i, _i, _i, _i, _i, _i64, _f, _i, _vp]
    L.gla_chunk_bwd_saved.restype = _i
    L.gla_chunk_bwd_saved.argtypes = [_vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp, _vp, _vp, _vp, _vp, _vp,
                                      _vp, _vp, _vp, ctypes.c_size_t, _i, _i, _i, _i, _i, _i64, _f, _i, _vp]
    L.gla_decode_step.restype = _i
    L.gla_decode_step.argtypes = [_vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp]
    L.conv1d_silu_causal.restype = _i
    L.conv1d_silu_causal.argtypes = [_vp, _i, _vp, _vp, _f, _vp, _vp, _vp, _vp, _vp,
                                     _i, _i, _i, _i, _vp]
    L.conv1d_silu_causal_bwd_workspace_bytes.restype = ctypes.c_size_t
    L.conv1d_silu_causal_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i]
    L.conv1d_silu_causal_bwd.restype = _i
    L.conv1d_silu_causal_bwd.argtypes = [_vp, _i, _vp, _vp, _f, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                         _vp, _vp, ctypes.c_size_t, _i, _i, _i, _i, _vp]
    L.gla_chunk_fwd_varlen.restype = _i
    L.gla_chunk_fwd_varlen.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, ctypes.c_size_t, _i,
                                       _i, _i, _i, ctypes.c_longlong, _f, _i, _vp]
    L.gla_chunk_varlen_workspace_bytes.restype = ctypes.c_size_t
    L.gla_chunk_varlen_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
    L.gla_segment_workspace_bytes.restype = ctypes.c_size_t
    L.gla_segment_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
    L.gla_segment_state_fwd.restype = _i
    L.gla_segment_state_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _i, _i, _i, _i, _i,
                                        _i64, _i, _vp]
    L.gla_segment_state_bwd.restype = _i
    L.gla_segment_state_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _i, _i, _i, _i, _i,
                                        _i64, _f, _i, _vp]
    L.gla_state_fold.restype = _i
    L.gla_state_fold.argtypes = [_vp, _vp, _i, _i, _vp, _vp, _i, _i, _i, _vp]
    L.conv1d_silu_decode_step.restype = _i
    L.conv1d_silu_decode_step.argtypes = [_vp, _vp, _i, _i, _vp, _vp, _f, _vp, _vp, _vp, _vp, _i, _i, _i, _vp]
    L.gla_get_device_status.restype = _i
    L.gla_get_device_status.argtypes = [_vp, ctypes.POINTER(_i)]
    L.gla_set_wait_limit_ns.restype = _i
    L.gla_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    L.gla_selftest_wait_timeout.restype = _i
    L.gla_selftest_wait_timeout.argtypes = [_vp]
    L.gla_chunk_fwd_noalloc.restype = _i
    L.gla_chunk_fwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                        _i64, _f, _i, _vp]
    L.gla_trace_enable.restype = _i
    L.gla_trace_enable.argtypes = [_i]
    L.gla_trace_summary.restype = _i
    L.gla_trace_summary.argtypes = [ctypes.POINTER(ctypes.c_char_p),
                                    ctypes.POINTER(ctypes.c_ulonglong),
                                    ctypes.POINTER(ctypes.c_double), _i]
    L.gla_build_flags.restype = _i
    L.gla_build_flags.argtypes = []
    return L


def _check(fn, status):
    if status != 0:
        raise GlaError(fn, status, lib().gla_last_cuda_error())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t):
    if t.dtype == torch.bfloat16:
        return GLA_BF16
    if t.dtype == torch.float32:
        return GLA_F32
    raise TypeError("q/k/v must be bfloat16 or float32, got %s" % t.dtype)


def _token_stride(x, B, T, H, d):
    """Token stride (elements) of a [B,T,H,d] view whose head and feature
    dims are packed; raises if the view is not of that form."""
    if x.shape != (B, T, H, d):
        raise ValueError("expected shape %s, got %s" % ((B, T, H, d), tuple(x.shape)))
    s = x.stride()
    if s[3] != 1 or s[2] != d:
        raise ValueError("head and feature dims must be packed (strides %s)" % (s,))
    if B > 1 and T > 0 and s[0] != T * s[1]:
        raise ValueError("batch stride must be T * token stride (strides %s)" % (s,))
    return s[1]


def _need(x, name, dtype, shape=None, contiguous=True):
    if x is None:
        return
    if not x.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if x.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, x.dtype))
    if shape is not None and tuple(x.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(x.shape)))
    if contiguous and not x.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def gla_status_string(status):
    return lib().gla_status_string(int(status)).decode()


def gla_launch_count():
    return int(lib().gla_launch_count())


def gla_build_flags():
    """Bit mask of how the loaded library was built (GLA_BUILD_DEBUG_BOUNDS
    for the checking build)."""
    return int(lib().gla_build_flags())


def gla_chunk_workspace_bytes(B, T, H, dk=96, dv=192, for_bwd=False, from_saved=False):
    """Workspace bytes of gla_chunk_fwd (default), gla_chunk_bwd (for_bwd) or
    gla_chunk_bwd_saved (for_bwd and from_saved)."""
    mode = (2 if from_saved else 1) if for_bwd else 0
    return int(lib().gla_chunk_workspace_bytes(B, T, H, dk, dv, mode))


def gla_chunk_saved_state_bytes(B, T, H, dk=96, dv=192):
    return int(lib().gla_chunk_saved_state_bytes(B, T, H, dk, dv))


def _qkv_strides(q, k, v):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    lq = _token_stride(q, B, T, H, dk)
    lk = _token_stride(k, B, T, H, dk)
    lv = _token_stride(v, B, T, H, dv)
    if lq == H * dk and lk == H * dk and lv == H * dv:
        return 0
    if not (lq == lk == lv):
        raise ValueError("q, k and v must share one token stride when not packed "
                         "(got %d, %d, %d)" % (lq, lk, lv))
    return lq


def gla_chunk_fwd(q, k, v, a, s0=None, o=None, s_final=None, ws=None, scale=None,
                  want_final_state=True, stream=None):
    """Chunked forward.  q, k [B,T,H,dk]; v [B,T,H,dv] (bf16 or fp32, may be
    views into one fused projection buffer); a [B,T,H] fp32; s0 [B,H,dk,dv]
    fp32 or None.  Returns (o, s_final)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    for name, x in (("k", k), ("v", v)):
        if x.dtype != q.dtype:
            raise TypeError("%s must have the dtype of q" % name)
    ld = _qkv_strides(q, k, v)
    _need(a, "a", torch.float32, (B, T, H))
    _need(s0, "s0", torch.float32, (B, H, dk, dv))
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype, (B, T, H, dv))
    if s_final is None and want_final_state:
        s_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(s_final, "s_final", torch.float32, (B, H, dk, dv))
    need = gla_chunk_workspace_bytes(B, T, H, dk, dv, False) if dt == GLA_BF16 else 0
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    if scale is None:
        scale = dk ** -0.5
    st = lib().gla_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(s0), _ptr(o),
                             _ptr(s_final), _ptr(ws), 0 if ws is None else ws.numel(),
                             B, T, H, dk, dv, ld, float(scale), dt, _stream(stream))
    _check("gla_chunk_fwd", st)
    return o, s_final


def gla_chunk_bwd(q, k, v, a, dO, s0=None, ds_final=None, grads=None, ws=None, scale=None,
                  want_grad_s0=True, stream=None):
    """Chunked backward.  Returns (dq, dk, dv, da, ds0)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    ld = _qkv_strides(q, k, v)
    _need(a, "a", torch.float32, (B, T, H))
    _need(dO, "dO", q.dtype, (B, T, H, dv))
    _need(s0, "s0", torch.float32, (B, H, dk, dv))
    _need(ds_final, "ds_final", torch.float32, (B, H, dk, dv))
    dev = q.device
    if grads is None:
        grads = (torch.empty((B, T, H, dk), dtype=q.dtype, device=dev),
                 torch.empty((B, T, H, dk), dtype=q.dtype, device=dev),
                 torch.empty((B, T, H, dv), dtype=q.dtype, device=dev),
                 torch.empty((B, T, H), dtype=torch.float32, device=dev),
                 torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
                 if want_grad_s0 else None)
    gq, gk, gv, ga, gs0 = grads
    _need(gq, "grad_q", q.dtype, (B, T, H, dk))
    _need(gk, "grad_k", q.dtype, (B, T, H, dk))
    _need(gv, "grad_v", q.dtype, (B, T, H, dv))
    _need(ga, "grad_a", torch.float32, (B, T, H))
    _need(gs0, "grad_s0", torch.float32, (B, H, dk, dv))
    need = gla_chunk_workspace_bytes(B, T, H, dk, dv, True)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    if scale is None:
        scale = dk ** -0.5
    st = lib().gla_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(s0), _ptr(dO),
                             _ptr(ds_final), _ptr(gq), _ptr(gk), _ptr(gv), _ptr(ga), _ptr(gs0),
                             _ptr(ws), 0 if ws is None else ws.numel(), B, T, H, dk, dv, ld,
                             float(scale), dt, _stream(stream))
    _check("gla_chunk_bwd", st)
    return gq, gk, gv, ga, gs0


def gla_chunk_fwd_train(q, k, v, a, s0=None, o=None, s_final=None, saved=None, ws=None, scale=None,
                        stream=None):
    """gla_chunk_fwd that also keeps the state entering every chunk (bf16 hi
    and lo planes) for gla_chunk_bwd_saved.  Returns (o, s_final, saved);
    saved is a uint8 tensor of gla_chunk_saved_state_bytes bytes."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype != torch.bfloat16:
        raise TypeError("gla_chunk_fwd_train takes bf16 q, k, v")
    ld = _qkv_strides(q, k, v)
    _need(a, "a", torch.float32, (B, T, H))
    _need(s0, "s0", torch.float32, (B, H, dk, dv))
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype, (B, T, H, dv))
    if s_final is None:
        s_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(s_final, "s_final", torch.float32, (B, H, dk, dv))
    nsv = gla_chunk_saved_state_bytes(B, T, H, dk, dv)
    if saved is None:
        saved = torch.empty(max(nsv, 16), dtype=torch.uint8, device=q.device)
    _need(saved, "saved", torch.uint8)
    need = gla_chunk_workspace_bytes(B, T, H, dk, dv)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    sc = dk ** -0.5 if scale is None else scale
    st = lib().gla_chunk_fwd_train(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(s0), _ptr(o), _ptr(s_final),
                                   _ptr(saved), saved.numel(), _ptr(ws), 0 if ws is None else ws.numel(),
                                   B, T, H, dk, dv, ld, float(sc), GLA_BF16, _stream(stream))
    _check("gla_chunk_fwd_train", st)
    return o, s_final, saved


def gla_chunk_bwd_saved(q, k, v, a, saved, dO, s_final=None, ds_final=None, grads=None, ws=None, scale=None,
                        want_grad_s0=True, stream=None):
    """gla_chunk_bwd from the states gla_chunk_fwd_train kept (s_final is
    needed only with ds_final).  Returns (dq, dk, dv, da, ds0)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype != torch.bfloat16:
        raise TypeError("gla_chunk_bwd_saved takes bf16 q, k, v")
    ld = _qkv_strides(q, k, v)
    _need(a, "a", torch.float32, (B, T, H))
    _need(dO, "dO", q.dtype, (B, T, H, dv))
    _need(saved, "saved", torch.uint8)
    _need(s_final, "s_final", torch.float32, (B, H, dk, dv))
    _need(ds_final, "ds_final", torch.float32, (B, H, dk, dv))
    dev = q.device
    if grads is None:
        grads = (torch.empty((B, T, H, dk), dtype=q.dtype, device=dev),
                 torch.empty((B, T, H, dk), dtype=q.dtype, device=dev),
                 torch.empty((B, T, H, dv), dtype=q.dtype, device=dev),
                 torch.empty((B, T, H), dtype=torch.float32, device=dev),
                 torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if want_grad_s0 else None)
    gq, gk, gv, ga, gs0 = grads
    _need(gq, "grad_q", q.dtype, (B, T, H, dk))
    _need(gk, "grad_k", q.dtype, (B, T, H, dk))
    _need(gv, "grad_v", q.dtype, (B, T, H, dv))
    _need(ga, "grad_a", torch.float32, (B, T, H))
    _need(gs0, "grad_s0", torch.float32, (B, H, dk, dv))
    need = gla_chunk_workspace_bytes(B, T, H, dk, dv, for_bwd=True, from_saved=True)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    sc = dk ** -0.5 if scale is None else scale
    st = lib().gla_chunk_bwd_saved(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(saved), saved.numel(), _ptr(s_final),
                                   _ptr(dO), _ptr(ds_final), _ptr(gq), _ptr(gk), _ptr(gv), _ptr(ga), _ptr(gs0),
                                   _ptr(ws), 0 if ws is None else ws.numel(), B, T, H, dk, dv, ld, float(sc),
                                   GLA_BF16, _stream(stream))
    _check("gla_chunk_bwd_saved", st)
    return gq, gk, gv, ga, gs0


def gla_decode_step(state, q, k, v, a, o=None, slot_idx=None, scale=None, stream=None):
    """In-place decode step.  state [N_slots,H,dk,dv] fp32; q, k [N,H,dk] and
    v [N,H,dv] bf16; a [N,H] fp32; slot_idx [N] int32 or None (a slot outside
    the pool is skipped and recorded in the device status word).  Returns o."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    _need(state, "state", torch.float32)
    if state.dim() != 4 or tuple(state.shape[1:]) != (H, dk, dv):
        raise ValueError("state must be [N_slots, %d, %d, %d]" % (H, dk, dv))
    _need(q, "q", torch.bfloat16, (N, H, dk))
    _need(k, "k", torch.bfloat16, (N, H, dk))
    _need(v, "v", torch.bfloat16, (N, H, dv))
    _need(a, "a", torch.float32, (N, H))
    _need(slot_idx, "slot_idx", torch.int32, (N,))
    if slot_idx is None and state.shape[0] != N:
        raise ValueError("without slot_idx the state must have N slots")
    if o is None:
        o = torch.empty((N, H, dv), dtype=torch.float32, device=q.device)
    _need(o, "o", torch.float32, (N, H, dv))
    if scale is None:
        scale = dk ** -0.5
    st = lib().gla_decode_step(_ptr(state), _ptr(slot_idx), state.shape[0], _ptr(q), _ptr(k), _ptr(v), _ptr(a),
                               _ptr(o), N, H, dk, dv, float(scale), _stream(stream))
    _check("gla_decode_step", st)
    return o


def conv1d_silu_causal(x, w, apply_ln=True, ln_gamma=None, ln_beta=None, ln_eps=1e-5,
                       bias=None, conv_state_in=None, conv_state_out=None, y=None,
                       stream=None):
    """LayerNorm -> causal depthwise conv -> SiLU.  x [B,T,D] bf16; w [D,W]
    fp32.  Returns y (and fills conv_state_out [B,W-1,D] fp32 if given)."""
    B, T, D = x.shape
    W = w.shape[1]
    _need(x, "x", torch.bfloat16, (B, T, D))
    _need(w, "w", torch.float32, (D, W))
    _need(ln_gamma, "ln_gamma", torch.float32, (D,))
    _need(ln_beta, "ln_beta", torch.float32, (D,))
    _need(bias, "bias", torch.float32, (D,))
    _need(conv_state_in, "conv_state_in", torch.float32, (B, W - 1, D))
    _need(conv_state_out, "conv_state_out", torch.float32, (B, W - 1, D))
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", torch.bfloat16, (B, T, D))
    st = lib().conv1d_silu_causal(_ptr(x), 1 if apply_ln else 0, _ptr(ln_gamma), _ptr(ln_beta),
                                  float(ln_eps), _ptr(w), _ptr(bias), _ptr(conv_state_in),
                                  _ptr(conv_state_out), _ptr(y), B, T, D, W, _stream(stream))
    _check("conv1d_silu_causal", st)
    return y


def gla_chunk_varlen_workspace_bytes(N, total_T, H, dk=96, dv=192):
    return int(lib().gla_chunk_varlen_workspace_bytes(N, total_T, H, dk, dv))


def gla_chunk_fwd_varlen(q, k, v, a, cu_seqlens, s0=None, o=None, s_final=None, scale=None,
                         want_final_state=True, ws=None, segmented=True, stream=None):
    """Chunked forward over packed sequences: q, k [total,H,96], v [total,H,192]
    bf16, a [total,H] fp32, cu_seqlens [N+1] int32 on the device.  With
    segmented (the default) a workspace is allocated when the caller passes
    none, so long sequences are cut into parallel segments.  Returns
    (o [total,H,192] bf16, s_final [N,H,96,192] fp32 or None)."""
    total, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype != torch.bfloat16:
        raise TypeError("gla_chunk_fwd_varlen takes bf16 q, k, v")
    _need(k, "k", torch.bfloat16, (total, H, dk))
    _need(v, "v", torch.bfloat16, (total, H, dv))
    _need(q, "q", torch.bfloat16, (total, H, dk))
    _need(a, "a", torch.float32, (total, H))
    N = cu_seqlens.numel() - 1
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,))
    _need(s0, "s0", torch.float32, (N, H, dk, dv))
    if o is None:
        o = torch.empty((total, H, dv), dtype=torch.bfloat16, device=q.device)
    _need(o, "o", torch.bfloat16, (total, H, dv))
    if s_final is None and want_final_state:
        s_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(s_final, "s_final", torch.float32, (N, H, dk, dv))
    sc = dk ** -0.5 if scale is None else scale
    if ws is None and segmented:
        need = gla_chunk_varlen_workspace_bytes(N, total, H, dk, dv)
        if need > 0:
            ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib().gla_chunk_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(cu_seqlens), N, _ptr(s0), _ptr(o),
                                    _ptr(s_final), _ptr(ws), 0 if ws is None else ws.numel(), total, H, dk, dv,
                                    0, float(sc), GLA_BF16, _stream(stream))
    _check("gla_chunk_fwd_varlen", st)
    return o, s_final


def gla_segment_workspace_bytes(B, T, H, dk=96, dv=192):
    return int(lib().gla_segment_workspace_bytes(B, T, H, dk, dv))


def _segment_outputs(B, H, dk, dv, dev, s_seg, g_seg, want_g):
    if s_seg is None:
        s_seg = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    _need(s_seg, "s_seg", torch.float32, (B, H, dk, dv))
    if g_seg is None and want_g:
        g_seg = torch.empty((B, H), dtype=torch.float32, device=dev)
    _need(g_seg, "g_seg", torch.float32, (B, H))
    return s_seg, g_seg


def _segment_ws(ws, B, T, H, dk, dv, dev):
    need = gla_segment_workspace_bytes(B, T, H, dk, dv)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    return ws


def gla_segment_state_fwd(k, v, a, s_seg=None, g_seg=None, ws=None, want_decay=True, stream=None):
    """State a segment of tokens leaves from a zero start, and its total
    log-decay.  k [B,T,H,96], v [B,T,H,192] bf16; a [B,T,H] fp32.  Returns
    (s_seg [B,H,96,192] fp32, g_seg [B,H] fp32 or None)."""
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    if k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("gla_segment_state_fwd takes bf16 k and v")
    lk = _token_stride(k, B, T, H, dk)
    lv = _token_stride(v, B, T, H, dv)
    if lk == H * dk and lv == H * dv:
        ld = 0
    elif lk == lv:
        ld = lk
    else:
        raise ValueError("k and v must share one token stride when not packed (got %d, %d)" % (lk, lv))
    _need(a, "a", torch.float32, (B, T, H))
    s_seg, g_seg = _segment_outputs(B, H, dk, dv, k.device, s_seg, g_seg, want_decay)
    ws = _segment_ws(ws, B, T, H, dk, dv, k.device)
    st = lib().gla_segment_state_fwd(_ptr(k), _ptr(v), _ptr(a), _ptr(s_seg), _ptr(g_seg), _ptr(ws),
                                     0 if ws is None else ws.numel(), B, T, H, dk, dv, ld, GLA_BF16,
                                     _stream(stream))
    _check("gla_segment_state_fwd", st)
    return s_seg, g_seg


def gla_segment_state_bwd(q, dO, a, ds_seg=None, g_seg=None, ws=None, scale=None, want_decay=False,
                          stream=None):
    """Gradient of the state entering a segment from the segment's own
    outputs (zero gradient at its end), and optionally its total log-decay.
    q [B,T,H,96] bf16 (packed heads; any token stride), dO [B,T,H,192] bf16
    contiguous; a [B,T,H] fp32.  Returns (ds_seg [B,H,96,192], g_seg or None)."""
    B, T, H, dk = q.shape
    dv = dO.shape[-1]
    if q.dtype != torch.bfloat16:
        raise TypeError("gla_segment_state_bwd takes bf16 q and dO")
    lq = _token_stride(q, B, T, H, dk)
    if lq != H * dk and lq < H * dv:
        raise ValueError("an unpacked q needs a token stride >= H*dv (got %d)" % lq)
    _need(dO, "dO", torch.bfloat16, (B, T, H, dv))
    _need(a, "a", torch.float32, (B, T, H))
    ds_seg, g_seg = _segment_outputs(B, H, dk, dv, q.device, ds_seg, g_seg, want_decay)
    ws = _segment_ws(ws, B, T, H, dk, dv, q.device)
    sc = dk ** -0.5 if scale is None else scale
    st = lib().gla_segment_state_bwd(_ptr(q), _ptr(dO), _ptr(a), _ptr(ds_seg), _ptr(g_seg), _ptr(ws),
                                     0 if ws is None else ws.numel(), B, T, H, dk, dv,
                                     0 if lq == H * dk else lq, float(sc), GLA_BF16, _stream(stream))
    _check("gla_segment_state_bwd", st)
    return ds_seg, g_seg


def gla_state_fold(s, g, reverse=False, s_in=None, out=None, stream=None):
    """x <- exp(g[j]) x + s[j] over j = 0..n-1 (n-1..0 if reverse) from
    x = s_in (zeros if None).  s [n, *U, 96, 192] fp32, g [n, *U] fp32 with U
    the unit dims (e.g. B, H); s_in / out [*U, 96, 192].  Returns out."""
    n = s.shape[0]
    unit_shape = tuple(s.shape[1:-2])
    dk, dv = s.shape[-2], s.shape[-1]
    units = 1
    for x in unit_shape:
        units *= x
    _need(s, "s", torch.float32)
    _need(g, "g", torch.float32, (n,) + unit_shape)
    _need(s_in, "s_in", torch.float32, unit_shape + (dk, dv))
    if out is None:
        out = torch.empty(unit_shape + (dk, dv), dtype=torch.float32, device=s.device)
    _need(out, "out", torch.float32, unit_shape + (dk, dv))
    st = lib().gla_state_fold(_ptr(s), _ptr(g), n, 1 if reverse else 0, _ptr(s_in), _ptr(out), units, dk, dv,
                              _stream(stream))
    _check("gla_state_fold", st)
    return out


def conv1d_silu_causal_bwd_workspace_bytes(B, T, D, W=4):
    return int(lib().conv1d_silu_causal_bwd_workspace_bytes(B, T, D, W))


def conv1d_silu_causal_bwd(x, w, dy, apply_ln=True, ln_gamma=None, ln_beta=None, ln_eps=1e-5, bias=None,
                           conv_state_in=None, want=("dx", "dw", "dbias", "dln_gamma", "dln_beta", "dconv_state_in"),
                           ws=None, stream=None):
    """Backward of conv1d_silu_causal.  Returns a dict with the gradients in
    `want` (dx [B,T,D] bf16; dw [D,W], dbias, dln_gamma, dln_beta [D],
    dconv_state_in [B,W-1,D] fp32)."""
    B, T, D = x.shape
    W = w.shape[1]
    _need(x, "x", torch.bfloat16, (B, T, D))
    _need(dy, "dy", torch.bfloat16, (B, T, D))
    _need(w, "w", torch.float32, (D, W))
    _need(ln_gamma, "ln_gamma", torch.float32, (D,))
    _need(ln_beta, "ln_beta", torch.float32, (D,))
    _need(bias, "bias", torch.float32, (D,))
    _need(conv_state_in, "conv_state_in", torch.float32, (B, W - 1, D))
    dev = x.device
    out = {"dx": torch.empty_like(x), "dw": torch.empty((D, W), dtype=torch.float32, device=dev)}
    for name, shape in (("dbias", (D,)), ("dln_gamma", (D,)), ("dln_beta", (D,)),
                        ("dconv_state_in", (B, W - 1, D))):
        out[name] = torch.empty(shape, dtype=torch.float32, device=dev) if name in want else None
    need = conv1d_silu_causal_bwd_workspace_bytes(B, T, D, W)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    st = lib().conv1d_silu_causal_bwd(_ptr(x), 1 if apply_ln else 0, _ptr(ln_gamma), _ptr(ln_beta), float(ln_eps),
                                      _ptr(w), _ptr(bias), _ptr(conv_state_in), _ptr(dy), _ptr(out["dx"]),
                                      _ptr(out["dw"]), _ptr(out["dbias"]), _ptr(out["dln_gamma"]),
                                      _ptr(out["dln_beta"]), _ptr(out["dconv_state_in"]), _ptr(ws),
                                      ws.numel() * ws.element_size(), B, T, D, W, _stream(stream))
    _check("conv1d_silu_causal_bwd", st)
    return {k: v for k, v in out.items() if k in want or k in ("dx", "dw")}


def conv1d_silu_decode_step(x, w, conv_state, slot_idx=None, apply_ln=True, ln_gamma=None,
                            ln_beta=None, ln_eps=1e-5, bias=None, y=None, stream=None):
    """Front end at decode time: one token per sequence.  x [N,D] bf16;
    conv_state [N_slots,W-1,D] fp32 (oldest first), updated in place;
    slot_idx [N] int32 or None.  Returns y [N,D] bf16."""
    N, D = x.shape
    W = w.shape[1]
    _need(x, "x", torch.bfloat16, (N, D))
    _need(w, "w", torch.float32, (D, W))
    _need(ln_gamma, "ln_gamma", torch.float32, (D,))
    _need(ln_beta, "ln_beta", torch.float32, (D,))
    _need(bias, "bias", torch.float32, (D,))
    n_slots = conv_state.shape[0] if conv_state is not None else N
    _need(conv_state, "conv_state", torch.float32, (n_slots, W - 1, D))
    if slot_idx is not None:
        _need(slot_idx, "slot_idx", torch.int32, (N,))
    elif n_slots != N:
        raise ValueError("conv_state has %d slots for %d sequences and no slot_idx" % (n_slots, N))
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", torch.bfloat16, (N, D))
    st = lib().conv1d_silu_decode_step(_ptr(x), _ptr(slot_idx), n_slots, 1 if apply_ln else 0, _ptr(ln_gamma),
                                       _ptr(ln_beta), float(ln_eps), _ptr(w), _ptr(bias), _ptr(conv_state),
                                       _ptr(y), N, D, W, _stream(stream))
    _check("conv1d_silu_decode_step", st)
    return y


def gla_get_device_status(stream=None):
    """Synchronise the stream and return (and clear) the device status word."""
    out = ctypes.c_int(0)
    _check("gla_get_device_status", lib().gla_get_device_status(_stream(stream),
                                                                ctypes.byref(out)))
    return out.value


def gla_set_wait_limit_ns(ns):
    _check("gla_set_wait_limit_ns", lib().gla_set_wait_limit_ns(int(ns)))


def gla_selftest_wait_timeout(stream=None):
    _check("gla_selftest_wait_timeout", lib().gla_selftest_wait_timeout(_stream(stream)))


def gla_trace_enable(enable=True):
    """Start (clearing earlier records) or stop per-launch event tracing."""
    _check("gla_trace_enable", lib().gla_trace_enable(1 if enable else 0))


def gla_trace_summary(max_entries=64):
    """Synchronise on the traced launches and return
    [(kernel_name, launches, total_ms), ...] in first-launch order."""
    names = (ctypes.c_char_p * max_entries)()
    counts = (ctypes.c_ulonglong * max_entries)()
    totals = (ctypes.c_double * max_entries)()
    n = lib().gla_trace_summary(names, counts, totals, max_entries)
    return [(names[i].decode(), int(counts[i]), float(totals[i])) for i in range(n)]


def gla_chunk_fwd_noalloc(q, k, v, a, s0=None, o=None, s_final=None, scale=None,
                          want_final_state=True, stream=None):
    """gla_chunk_fwd without a workspace, for callers that cannot allocate
    device memory: libgla uses its built-in scratch array (shared by all
    calls on a GPU; calls that overlap on the GPU race).  Shapes that need
    more scratch than the array holds raise GlaError(GLA_ERR_UNSUPPORTED)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    ld = _qkv_strides(q, k, v)
    _need(a, "a", torch.float32, (B, T, H))
    _need(s0, "s0", torch.float32, (B, H, dk, dv))
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype, (B, T, H, dv))
    if s_final is None and want_final_state:
        s_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(s_final, "s_final", torch.float32, (B, H, dk, dv))
    if scale is None:
        scale = dk ** -0.5
    st = lib().gla_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(s0), _ptr(o),
                                     _ptr(s_final), B, T, H, dk, dv, ld, float(scale), dt,
                                     _stream(stream))
    _check("gla_chunk_fwd_noalloc", st)
    return o, s_final
