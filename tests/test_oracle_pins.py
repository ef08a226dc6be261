"""Pins for the fp64 CPU oracle (no GPU).

The oracle (oracle/gla_oracle.c) is checked against things other than itself:
an independently written quadratic closed form, the textbook a == 0 special
case, an independently written chunked evaluation at several chunk sizes,
state carry across a split, a hand-worked two-token example, central finite
differences for the backward, two independent formulas for da, decode steps
against the recurrence, LayerNorm moments, numpy.convolve and scipy's
logistic function for the front end, and the pages' sizing identities.
Each planted mistake (oracle.recurrent.FAULTS) must be caught by at least one
of these pins; test_planted_mistakes_are_caught checks that.
"""
import json
import os

import numpy as np
import pytest
import scipy.special

from oracle import chunked, closed_form, recurrent
from linear_attention_simple_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np(t):
    return None if t is None else t.float().numpy().astype(np.float64)


def _small(B=2, T=48, H=2, dk=5, dv=3, seed=0, s0_std=0.3, a_mean=3.0):
    d = inputs.chunk_inputs(B, T, H, dk, dv, dtype=__import__("torch").float32, seed=seed,
                            s0_std=s0_std)
    a = _np(d["a"])
    if a_mean != 3.0:
        a = _np(inputs.log_decay((B, T, H), seed + 99, mean=a_mean))
    return _np(d["q"]), _np(d["k"]), _np(d["v"]), a, _np(d["s0"])


def _rel(x, ref):
    return np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300)


# ---------------------------------------------------------------- forward pins

def check_closed_form():
    errs = []
    for seed, a_mean in ((0, 3.0), (1, -1.0)):
        q, k, v, a, s0 = _small(seed=seed, a_mean=a_mean)
        o, sT = recurrent.fwd(q, k, v, a, s0)
        o2, sT2 = closed_form.quadratic(q, k, v, a, s0)
        errs += [_rel(o, o2), _rel(sT, sT2)]
    return max(errs)


def test_fwd_matches_quadratic_closed_form():
    assert check_closed_form() < 1e-12


def check_a_zero():
    q, k, v, _, _ = _small(T=40, seed=3)
    a = np.zeros(q.shape[:3])
    o, _ = recurrent.fwd(q, k, v, a, None)
    return _rel(o, closed_form.causal_linear_attention(q, k, v))


def test_a_zero_reduces_to_causal_linear_attention():
    assert check_a_zero() < 1e-12


@pytest.mark.parametrize("C", [1, 7, 16, 64, 128])
def test_chunk_size_independence(C):
    q, k, v, a, s0 = _small(B=1, T=300, H=2, dk=4, dv=3, seed=5)
    o, sT = recurrent.fwd(q, k, v, a, s0)
    oc, sTc = chunked.chunked(q, k, v, a, s0, C=C)
    assert _rel(oc, o) < 1e-12
    assert _rel(sTc, sT) < 1e-12


@pytest.mark.parametrize("split", [1, 77, 128, 199])
def test_state_carry_matches_unsplit(split):
    q, k, v, a, s0 = _small(B=2, T=200, H=2, dk=4, dv=3, seed=6)
    o, sT = recurrent.fwd(q, k, v, a, s0)
    o1, s1 = recurrent.fwd(q[:, :split], k[:, :split], v[:, :split], a[:, :split], s0)
    o2, s2 = recurrent.fwd(q[:, split:], k[:, split:], v[:, split:], a[:, split:], s1)
    assert _rel(np.concatenate([o1, o2], axis=1), o) < 1e-13
    assert _rel(s2, sT) < 1e-13


def check_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_T2_dk1_dv1.json")))
    sh = (1, 2, 1, 1)
    o, sT = recurrent.fwd(np.reshape(g["q"], sh), np.reshape(g["k"], sh),
                          np.reshape(g["v"], sh), np.reshape(g["a"], (1, 2, 1)), None,
                          scale=g["scale"])
    return max(np.max(np.abs(o.ravel() - np.array(g["o"]))), abs(sT.item() - g["s_final"]))


def test_hand_worked_two_token_example():
    assert check_hand_example() < 1e-12


def test_decay_only_state():
    """k = v = 0: the state only decays, S_T = exp(sum a) S_0, and o = 0 iff q = 0."""
    q, k, v, a, s0 = _small(B=1, T=30, H=2, seed=8)
    o, sT = recurrent.fwd(q, np.zeros_like(k), np.zeros_like(v), a, s0)
    expect = np.exp(a.sum(axis=1))[:, :, None, None] * s0
    assert _rel(sT, expect) < 1e-13


# --------------------------------------------------------------- backward pins

def _loss(q, k, v, a, s0, dO, dsT):
    o, sT = recurrent.fwd(q, k, v, a, s0)
    return float(np.sum(o * dO) + np.sum(sT * dsT))


def check_finite_differences(seed=11):
    rng = np.random.default_rng(seed)
    q, k, v, a, s0 = _small(B=1, T=12, H=2, dk=3, dv=2, seed=seed)
    dO = rng.standard_normal((1, 12, 2, 2))
    dsT = rng.standard_normal((1, 2, 3, 2))
    dq, dk, dv, da, ds0 = recurrent.bwd(q, k, v, a, dO, s0, dsT)
    args = [q, k, v, a, s0]
    grads = [dq, dk, dv, da, ds0]
    h = 1e-6
    worst = 0.0
    for idx, (x, g) in enumerate(zip(args, grads)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            mi = it.multi_index
            xp = [y.copy() for y in args]
            xm = [y.copy() for y in args]
            xp[idx][mi] += h
            xm[idx][mi] -= h
            fd[mi] = (_loss(*xp, dO, dsT) - _loss(*xm, dO, dsT)) / (2 * h)
        worst = max(worst, _rel(g, fd))
    return worst


def test_bwd_matches_central_finite_differences():
    assert check_finite_differences() < 1e-6


def check_da_two_formulas(seed=12):
    rng = np.random.default_rng(seed)
    q, k, v, a, s0 = _small(B=2, T=70, H=2, dk=4, dv=3, seed=seed)
    dO = rng.standard_normal(v.shape)
    dsT = rng.standard_normal(s0.shape)
    o, sT = recurrent.fwd(q, k, v, a, s0)
    dq, dk, dv, da, ds0 = recurrent.bwd(q, k, v, a, dO, s0, dsT)
    # (ii) reverse cumulative sum of dO.o - k.dk plus <dS_T, S_T> (identity q.dq = dO.o)
    per_tok = np.sum(dO * o, axis=-1) - np.sum(k * dk, axis=-1)
    da2 = np.flip(np.cumsum(np.flip(per_tok, axis=1), axis=1), axis=1)
    da2 = da2 + np.sum(dsT * sT, axis=(2, 3))[:, None, :]
    ident = _rel(np.sum(q * dq, axis=-1), np.sum(dO * o, axis=-1))
    return max(_rel(da, da2), ident)


def test_da_two_independent_formulas_agree():
    assert check_da_two_formulas() < 1e-11


# ----------------------------------------------------------------- decode pins

def check_decode_equals_recurrence():
    q, k, v, a, s0 = _small(B=3, T=9, H=2, dk=4, dv=3, seed=13)
    o, sT = recurrent.fwd(q, k, v, a, s0)
    state = s0.copy()
    outs = []
    for t in range(q.shape[1]):
        state, ot = recurrent.decode(state, q[:, t], k[:, t], v[:, t], a[:, t])
        outs.append(ot)
    return max(_rel(np.stack(outs, axis=1), o), _rel(state, sT))


def test_decode_steps_equal_recurrence():
    assert check_decode_equals_recurrence() < 1e-13


def test_decode_slot_indirection():
    q, k, v, a, s0 = _small(B=4, T=1, H=2, dk=4, dv=3, seed=14)
    pool = np.concatenate([s0, 2 * s0], axis=0)          # 8 slots
    slots = np.array([5, 0, 7, 2])
    st, o = recurrent.decode(pool, q[:, 0], k[:, 0], v[:, 0], a[:, 0], slot_idx=slots)
    st2, o2 = recurrent.decode(pool[slots], q[:, 0], k[:, 0], v[:, 0], a[:, 0])
    assert _rel(o, o2) < 1e-15 and _rel(st[slots], st2) < 1e-15
    untouched = [i for i in range(8) if i not in slots]
    assert np.array_equal(st[untouched], pool[untouched])


# -------------------------------------------------------------- front-end pins

def _front(B=2, T=19, D=64, W=4, seed=15, shift=0.0):
    d = inputs.front_inputs(B, T, D, W, seed=seed, with_state=True)
    return _np(d["x"]) + shift, _np(d["w"]), _np(d["conv_state"])


def check_ln_moments():
    x, w, _ = _front(shift=3.0)        # nonzero mean so a missing centring shows
    onehot = np.zeros_like(w)
    onehot[:, -1] = 1.0
    y, _ = recurrent.ln_conv_silu(x, onehot, ln=True, silu=False)
    mean_err = np.max(np.abs(y.mean(axis=-1)))
    var_err = np.max(np.abs(y.var(axis=-1) - x.var(axis=-1) / (x.var(axis=-1) + 1e-5)))
    return max(mean_err, var_err)


def test_layernorm_moments():
    assert check_ln_moments() < 1e-12


def check_conv_vs_numpy():
    x, w, hist = _front()
    y, st_out = recurrent.ln_conv_silu(x, w, ln=False, silu=False, conv_state=hist)
    B, T, D = x.shape
    W = w.shape[1]
    ref = np.zeros_like(x)
    for b in range(B):
        full = np.concatenate([hist[b], x[b]], axis=0)       # [W-1+T, D]
        for c in range(D):
            # numpy.convolve flips its second argument: reverse the taps so that
            # w[c, W-1] multiplies the current token
            ref[b, :, c] = np.convolve(full[:, c], w[c, ::-1], mode="valid")
    st_ref = np.concatenate([hist, x], axis=1)[:, -(W - 1):]
    return max(_rel(y, ref), _rel(st_out, st_ref))


def test_conv_matches_numpy_convolve():
    assert check_conv_vs_numpy() < 1e-13


def test_silu_matches_scipy_expit():
    x, w, _ = _front(seed=16)
    onehot = np.zeros_like(w)
    onehot[:, -1] = 1.0
    y, _ = recurrent.ln_conv_silu(x, onehot, ln=False, silu=True)
    assert _rel(y, x * scipy.special.expit(x)) < 1e-14


def test_front_end_composes():
    """LN -> conv -> SiLU equals the three pinned stages run one after another."""
    x, w, hist = _front(seed=17)
    onehot = np.zeros_like(w)
    onehot[:, -1] = 1.0
    xn, _ = recurrent.ln_conv_silu(x, onehot, ln=True, silu=False)
    pre, _ = recurrent.ln_conv_silu(xn, w, ln=False, silu=False, conv_state=hist)
    y, _ = recurrent.ln_conv_silu(x, w, ln=True, silu=True, conv_state=hist)
    assert _rel(y, pre * scipy.special.expit(pre)) < 1e-13


# ------------------------------------------------ front-end backward pins

def _front_bwd_case(seed=18, T=6, D=8, ln=True):
    rng = np.random.default_rng(seed)
    B, W = 2, 4
    return dict(x=rng.standard_normal((B, T, D)) + 0.5, w=rng.standard_normal((D, W)) * 0.5,
                dy=rng.standard_normal((B, T, D)), g=1.0 + 0.5 * rng.standard_normal(D),
                be=0.5 * rng.standard_normal(D), bias=0.5 * rng.standard_normal(D),
                hist=rng.standard_normal((B, W - 1, D)), ln=ln)


def _front_loss(c, **over):
    v = dict(c)
    v.update(over)
    y, _ = recurrent.ln_conv_silu(v["x"], v["w"], ln=v["ln"], ln_gamma=v["g"] if v["ln"] else None,
                                  ln_beta=v["be"] if v["ln"] else None, bias=v["bias"], conv_state=v["hist"])
    return float(np.sum(y * c["dy"]))


def check_front_fd():
    """Central differences of sum(dy * y) through the pinned forward, every
    input element, against the oracle's backward; max relative error."""
    worst = 0.0
    for ln in (True, False):
        c = _front_bwd_case(ln=ln)
        dx, dw, dbias, dg, dbe, dcs = recurrent.ln_conv_silu_bwd(
            c["x"], c["w"], c["dy"], ln=ln, ln_gamma=c["g"] if ln else None, ln_beta=c["be"] if ln else None,
            bias=c["bias"], conv_state=c["hist"])
        pairs = [("x", dx), ("w", dw), ("bias", dbias), ("hist", dcs)] + ([("g", dg), ("be", dbe)] if ln else [])
        h = 1e-6
        for name, grad in pairs:
            num = np.zeros_like(grad)
            base = c[name]
            for idx in np.ndindex(base.shape):
                p_, m_ = base.copy(), base.copy()
                p_[idx] += h
                m_[idx] -= h
                num[idx] = (_front_loss(c, **{name: p_}) - _front_loss(c, **{name: m_})) / (2 * h)
            worst = max(worst, _rel(grad, num))
    return worst


def test_front_end_backward_finite_differences():
    assert check_front_fd() < 1e-6


def test_front_end_backward_matches_torch_autograd():
    """The oracle's hand-written backward against torch float64 autograd of an
    independently written forward (layer_norm, a causal conv1d over the history,
    silu)."""
    import torch
    c = _front_bwd_case(seed=19, T=9, D=16)
    t = {k: torch.tensor(c[k], dtype=torch.float64, requires_grad=True) for k in ("x", "w", "g", "be", "bias", "hist")}
    D = c["x"].shape[-1]
    xn = torch.nn.functional.layer_norm(t["x"], (D,), t["g"], t["be"], eps=1e-5)
    seq = torch.cat([t["hist"], xn], dim=1).transpose(1, 2)              # [B, D, W-1+T]
    u = torch.nn.functional.conv1d(seq, t["w"].unsqueeze(1), t["bias"], groups=D).transpose(1, 2)
    y = torch.nn.functional.silu(u)
    (y * torch.tensor(c["dy"])).sum().backward()
    dx, dw, dbias, dg, dbe, dcs = recurrent.ln_conv_silu_bwd(c["x"], c["w"], c["dy"], ln_gamma=c["g"],
                                                             ln_beta=c["be"], bias=c["bias"], conv_state=c["hist"])
    for ours, ref in ((dx, t["x"]), (dw, t["w"]), (dbias, t["bias"]), (dg, t["g"]), (dbe, t["be"]), (dcs, t["hist"])):
        assert _rel(ours, ref.grad.numpy()) < 1e-12


# ------------------------------------------------------------------ sizing pin

def test_sizing_identities_from_the_pages():
    g = json.load(open(os.path.join(GOLDEN, "sizing.json")))
    H, dk, dv, D, L, W = g["H"], g["dk"], g["dv"], g["D"], g["layers"], g["conv_width"]
    assert H * (2 * dk + 2 * dv) == g["fused_rows"]
    mixer = L * H * dk * dv * 4                      # fp32 matrix state, all layers
    conv = L * W * D * 4                             # fp32 conv window, all layers
    assert round((mixer + conv) / 1e6, 1) == g["state_mb_per_seq"]
    kv = L * 2 * D * 2 * g["kv_tokens"]              # bf16 K and V at 8,192 tokens
    assert round(kv / (mixer + conv)) == g["kv_ratio_at_8192"]


# ------------------------------------------------------- planted-mistake check

PIN_FOR_FAULT = {
    "no_decay": lambda: check_closed_form() < 1e-12,
    "exclusive_state": lambda: check_closed_form() < 1e-12,
    "double_scale": lambda: check_closed_form() < 1e-12,
    "decay_index": lambda: check_closed_form() < 1e-12,
    "bwd_da_no_exp": lambda: check_finite_differences() < 1e-6,
    "bwd_dk_sign": lambda: check_finite_differences() < 1e-6,
    "ln_no_center": lambda: check_ln_moments() < 1e-12,
    "conv_tap_flip": lambda: check_conv_vs_numpy() < 1e-13,
    "bwd_silu_sigmoid": lambda: check_front_fd() < 1e-6,
    "bwd_ln_no_mean": lambda: check_front_fd() < 1e-6,
}


@pytest.mark.parametrize("fault", sorted(recurrent.FAULTS))
def test_planted_mistakes_are_caught(fault):
    pin = PIN_FOR_FAULT[fault]
    assert pin(), "pin must pass on the unmodified oracle"
    recurrent.set_fault(recurrent.FAULTS[fault])
    try:
        assert not pin(), "planted mistake %r slipped through its pin" % fault
    finally:
        recurrent.set_fault(0)
