"""ctypes front end to the fp64 C oracle (``gla_oracle.c``).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Every function takes NumPy arrays (any float dtype; they are widened to
float64, which is exact for bf16 and fp32 inputs) and returns float64 arrays.

Pins (tests/test_oracle_pins.py):
  fwd     -- quadratic closed form; a == 0 causal linear attention; chunk-size
             independence; state carry across a split; T == 1 by hand.
  bwd     -- central finite differences of fwd; the two independent da
             formulas agree.
  decode  -- T decode steps equal the token recurrence's final state/outputs.
  front   -- LayerNorm moments; one-hot tap reduces to SiLU(LN(x));
             per-channel numpy.convolve.
"""
import ctypes
import numpy as np

from . import build as _build

_LIB = None
_dp = ctypes.POINTER(ctypes.c_double)


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lib.gla_oracle_fwd.restype = None
        lib.gla_oracle_bwd.restype = None
        lib.gla_oracle_decode.restype = None
        lib.gla_oracle_ln_conv_silu.restype = None
        lib.gla_oracle_ln_conv_silu_bwd.restype = None
        lib.gla_oracle_set_fault.argtypes = [ctypes.c_int]
        lib.gla_oracle_get_fault.restype = ctypes.c_int
        lib.gla_oracle_max_threads.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def _in(x):
    if x is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    return arr, arr.ctypes.data_as(_dp)


def _ptr(arr):
    return None if arr is None else arr.ctypes.data_as(_dp)


def set_fault(code: int) -> None:
    """Plant a known mistake (tests of the pins only); 0 clears it."""
    _lib().gla_oracle_set_fault(int(code))


def max_threads() -> int:
    return int(_lib().gla_oracle_max_threads())


FAULTS = {
    "bwd_silu_sigmoid": 9,
    "bwd_ln_no_mean": 10,
    "no_decay": 1,
    "exclusive_state": 2,
    "double_scale": 3,
    "decay_index": 4,
    "bwd_da_no_exp": 5,
    "bwd_dk_sign": 6,
    "ln_no_center": 7,
    "conv_tap_flip": 8,
}


def fwd(q, k, v, a, s0=None, scale=None):
    """Token recurrence.  q,k [B,T,H,dk]; v [B,T,H,dv]; a [B,T,H]; s0 [B,H,dk,dv].
    Returns (o [B,T,H,dv], s_final [B,H,dk,dv])."""
    q, qp = _in(q)
    k, kp = _in(k)
    v, vp = _in(v)
    a, ap = _in(a)
    s0, sp = _in(s0)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if scale is None:
        scale = dk ** -0.5
    o = np.zeros((B, T, H, dv), np.float64)
    sf = np.zeros((B, H, dk, dv), np.float64)
    _lib().gla_oracle_fwd(qp, kp, vp, ap, sp, _ptr(o), _ptr(sf), B, T, H, dk, dv,
                          ctypes.c_double(scale))
    return o, sf


def bwd(q, k, v, a, dO, s0=None, dsT=None, scale=None):
    """Reverse recurrence.  Returns (dq, dk, dv, da, ds0)."""
    q, qp = _in(q)
    k, kp = _in(k)
    v, vp = _in(v)
    a, ap = _in(a)
    dO, gp = _in(dO)
    s0, sp = _in(s0)
    dsT, tp = _in(dsT)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if scale is None:
        scale = dk ** -0.5
    dq = np.zeros_like(q)
    dk_ = np.zeros_like(k)
    dv_ = np.zeros_like(v)
    da = np.zeros_like(a)
    ds0 = np.zeros((B, H, dk, dv), np.float64)
    _lib().gla_oracle_bwd(qp, kp, vp, ap, sp, gp, tp, _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(da),
                          _ptr(ds0), B, T, H, dk, dv, ctypes.c_double(scale))
    return dq, dk_, dv_, da, ds0


def decode(state, q, k, v, a, slot_idx=None, scale=None):
    """One decode step.  state [N_slots,H,dk,dv] (a new array is returned,
    the input is not modified); q,k [N,H,dk]; v [N,H,dv]; a [N,H].
    Returns (new_state, o [N,H,dv])."""
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    q, qp = _in(q)
    k, kp = _in(k)
    v, vp = _in(v)
    a, ap = _in(a)
    N, H, dk = q.shape
    dv = v.shape[-1]
    if scale is None:
        scale = dk ** -0.5
    o = np.zeros((N, H, dv), np.float64)
    sl = None
    slp = None
    if slot_idx is not None:
        sl = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.int64))
        slp = sl.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong))
    _lib().gla_oracle_decode(_ptr(st), slp, qp, kp, vp, ap, _ptr(o), N, H, dk, dv,
                             ctypes.c_double(scale))
    return st, o


def ln_conv_silu(x, w, ln=True, ln_gamma=None, ln_beta=None, ln_eps=1e-5, bias=None,
                 conv_state=None, silu=True):
    """LayerNorm -> causal depthwise conv -> SiLU.  x [B,T,D]; w [D,W];
    conv_state [B,W-1,D] (history of conv inputs, oldest first).
    Returns (y [B,T,D], conv_state_out [B,W-1,D])."""
    x, xp = _in(x)
    w, wp = _in(w)
    g, gp = _in(ln_gamma)
    be, bp = _in(ln_beta)
    bi, bip = _in(bias)
    cs, csp = _in(conv_state)
    B, T, D = x.shape
    W = w.shape[1]
    y = np.zeros_like(x)
    cso = np.zeros((B, W - 1, D), np.float64)
    _lib().gla_oracle_ln_conv_silu(xp, gp, bp, ctypes.c_double(ln_eps), 1 if ln else 0, wp, bip,
                                   csp, _ptr(cso), _ptr(y), B, T, D, W, 1 if silu else 0)
    return y, cso


def ln_conv_silu_bwd(x, w, dy, ln=True, ln_gamma=None, ln_beta=None, ln_eps=1e-5, bias=None,
                     conv_state=None):
    """Backward of ln_conv_silu for the gradient dy of y.  Returns
    (dx [B,T,D], dw [D,W], dbias [D], dgamma [D], dbeta [D], dconv_state [B,W-1,D])."""
    x, xp = _in(x)
    w, wp = _in(w)
    dy, dyp = _in(dy)
    g, gp = _in(ln_gamma)
    be, bp = _in(ln_beta)
    bi, bip = _in(bias)
    cs, csp = _in(conv_state)
    B, T, D = x.shape
    W = w.shape[1]
    dx = np.zeros_like(x)
    dw = np.zeros((D, W), np.float64)
    dbias = np.zeros(D, np.float64)
    dgamma = np.zeros(D, np.float64)
    dbeta = np.zeros(D, np.float64)
    dcs = np.zeros((B, W - 1, D), np.float64)
    _lib().gla_oracle_ln_conv_silu_bwd(xp, gp, bp, ctypes.c_double(ln_eps), 1 if ln else 0, wp, bip, csp,
                                       dyp, _ptr(dx), _ptr(dw), _ptr(dbias), _ptr(dgamma), _ptr(dbeta),
                                       _ptr(dcs), B, T, D, W)
    return dx, dw, dbias, dgamma, dbeta, dcs
