"""GPU parity of the sequence split across ranks.

The per-segment calls (gla_segment_state_fwd / _bwd) and the fold
(gla_state_fold) against the fp64 oracle; then the whole split with the
ranks emulated one after another on one device -- phase 1 of every rank,
the stacked phase-1 vectors in place of the all_gather, phase 3 of every
rank -- against the oracle run on the unsplit sequence.  Nothing here waits
on another rank: the phases are ordinary launches in sequence.

Tolerances (tests/tolerances.py): bf16 outputs and gradients rel L2 <= 1e-2
and max-abs <= 5e-2 beyond bf16 storage rounding; fp32 states rel L2 <=
5e-3; da rel L2 <= 1e-2, max-abs <= 5e-2 * max(1, max|da|), as the unsplit
backward's.  The fold is fp32 arithmetic on fp32 inputs: rel L2 <= 1e-6.
"""
import numpy as np
import pytest
import torch

import linear_attention_simple_b200 as gla
from linear_attention_simple_b200 import inputs, seqpar
from oracle import recurrent
from tolerances import ABS_BF16, REL_BF16, REL_STATE, assert_bf16_close, rel_l2

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.fixture(scope="module", autouse=True)
def _build():
    from linear_attention_simple_b200 import build
    build.build()
    gla.lib()


# B*H = 2 and 3 take the sub-segment path inside a rank (fewer units than
# half the SMs); B*H = 80 the single-segment one.
@pytest.mark.parametrize("B,T,H", [(1, 1, 2), (1, 1000, 2), (3, 4097, 1), (2, 300, 40)])
def test_segment_state_fwd_matches_oracle(B, T, H):
    d = inputs.chunk_inputs(B, T, H, seed=500 + T, device="cuda")
    s, g = gla.gla_segment_state_fwd(d["k"], d["v"], d["a"])
    assert gla.gla_get_device_status() == 0
    k, v, a = (_np(d[n]) for n in ("k", "v", "a"))
    _, ref = recurrent.fwd(np.zeros_like(k), k, v, a)
    assert rel_l2(_np(s), ref) <= REL_STATE, rel_l2(_np(s), ref)
    assert rel_l2(_np(g), a.sum(axis=1)) <= 1e-5


@pytest.mark.parametrize("B,T,H", [(1, 1, 2), (1, 1000, 2), (3, 4097, 1), (2, 300, 40)])
def test_segment_state_bwd_matches_oracle(B, T, H):
    d = inputs.chunk_inputs(B, T, H, seed=600 + T, device="cuda", with_dO=True)
    ds, g = gla.gla_segment_state_bwd(d["q"], d["dO"], d["a"], want_decay=True)
    assert gla.gla_get_device_status() == 0
    q, k, a, dO = (_np(d[n]) for n in ("q", "k", "a", "dO"))
    v0 = np.zeros(dO.shape)
    ref = recurrent.bwd(q, np.zeros_like(k), v0, a, dO)[4]      # dS_0 with zero dS_T
    assert rel_l2(_np(ds), ref) <= REL_STATE, rel_l2(_np(ds), ref)
    assert rel_l2(_np(g), a.sum(axis=1)) <= 1e-5


def test_segment_state_fused_projection_stride():
    """k, v (and q) as views of one [B, T, 9216] projection buffer."""
    d = inputs.chunk_inputs(2, 700, 16, seed=640, device="cuda", ld=9216, with_dO=True)
    s, _ = gla.gla_segment_state_fwd(d["k"], d["v"], d["a"])
    ds, _ = gla.gla_segment_state_bwd(d["q"], d["dO"], d["a"])
    assert gla.gla_get_device_status() == 0
    q, k, v, a, dO = (_np(d[n]) for n in ("q", "k", "v", "a", "dO"))
    assert rel_l2(_np(s), recurrent.fwd(np.zeros_like(k), k, v, a)[1]) <= REL_STATE
    assert rel_l2(_np(ds), recurrent.bwd(q, np.zeros_like(k), np.zeros_like(v), a, dO)[4]) <= REL_STATE


def _fold_ref(s, g, reverse, s_in):
    x = np.zeros(s.shape[1:]) if s_in is None else s_in.copy()
    order = range(s.shape[0] - 1, -1, -1) if reverse else range(s.shape[0])
    for j in order:
        x = np.exp(g[j])[..., None, None] * x + s[j]
    return x


@pytest.mark.parametrize("n,reverse,with_in", [(0, False, True), (0, True, False), (1, False, False),
                                               (5, False, True), (5, True, True), (7, True, False)])
def test_state_fold_matches_numpy(n, reverse, with_in):
    B, H = 2, 3
    s = inputs.randn((n, B, H, 96, 192), 700 + n, "cuda")
    g = -torch.rand((n, B, H), generator=torch.Generator("cuda").manual_seed(701), device="cuda") * 3.0
    s_in = inputs.randn((B, H, 96, 192), 702, "cuda") if with_in else None
    out = gla.gla_state_fold(s, g, reverse=reverse, s_in=s_in)
    ref = _fold_ref(_np(s), _np(g), reverse, None if s_in is None else _np(s_in))
    if n == 0 and not with_in:
        assert not out.abs().max().item()
    else:
        assert rel_l2(_np(out), ref) <= 1e-6


def test_state_fold_in_place_and_gathered_offsets():
    """out may be s_in; g may start at any entry (4-byte offsets)."""
    B, H, n = 1, 3, 6
    s = inputs.randn((n, B, H, 96, 192), 710, "cuda")
    g = -torch.rand((n, B, H), generator=torch.Generator("cuda").manual_seed(711), device="cuda")
    x = inputs.randn((B, H, 96, 192), 712, "cuda")
    ref = _fold_ref(_np(s[3:]), _np(g[3:]), True, _np(x))
    gla.gla_state_fold(s[3:], g[3:], reverse=True, s_in=x, out=x)
    assert rel_l2(_np(x), ref) <= 1e-6


def _split_inputs(d, lengths):
    bounds = np.concatenate([[0], np.cumsum(lengths)])
    parts = []
    for r in range(len(lengths)):
        lo, hi = int(bounds[r]), int(bounds[r + 1])
        parts.append({n: (d[n][:, lo:hi].contiguous() if d[n] is not None and n != "s0" else d[n])
                      for n in d})
    return parts


@pytest.mark.parametrize("lengths", [[300, 0, 517, 683], [128, 128, 128, 128], [1, 2, 3, 1000, 77]])
def test_seqpar_forward_emulated_ranks(lengths):
    B, H = 2, 3
    T = sum(lengths)
    d = inputs.chunk_inputs(B, T, H, seed=720 + len(lengths), device="cuda", s0_std=0.1)
    parts = _split_inputs(d, lengths)
    gathered = torch.stack([seqpar.fwd_local(p["k"], p["v"], p["a"]) for p in parts])
    outs = [seqpar.fwd_finish(p["q"], p["k"], p["v"], p["a"], gathered, r, s0=d["s0"])
            for r, p in enumerate(parts)]
    assert gla.gla_get_device_status() == 0
    o = torch.cat([x[0] for x in outs], dim=1)
    ro, rs = recurrent.fwd(*(_np(d[n]) for n in ("q", "k", "v", "a")), _np(d["s0"]))
    assert_bf16_close(_np(o), ro, "o")
    for _, s_final in outs:
        assert rel_l2(_np(s_final), rs) <= REL_STATE


def _check_grads(got, ref):
    for name, g, r in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        assert_bf16_close(g, r, name)
    e_da = rel_l2(got[3], ref[3])
    assert e_da <= REL_BF16, "da rel L2 %.3g" % e_da
    assert np.max(np.abs(got[3] - ref[3])) <= ABS_BF16 * max(1.0, float(np.max(np.abs(ref[3]))))


@pytest.mark.parametrize("lengths,with_dsT", [([300, 0, 517, 683], True), ([128, 128, 128, 128], False),
                                              ([1, 2, 3, 1000, 77], True)])
def test_seqpar_backward_emulated_ranks(lengths, with_dsT):
    B, H = 2, 3
    T = sum(lengths)
    d = inputs.chunk_inputs(B, T, H, seed=740 + len(lengths), device="cuda", s0_std=0.1, with_dO=True)
    dsT = inputs.randn((B, H, 96, 192), 749, "cuda", std=0.1) if with_dsT else None
    parts = _split_inputs(d, lengths)
    gathered = torch.stack([seqpar.bwd_local(p["q"], p["k"], p["v"], p["a"], p["dO"]) for p in parts])
    outs = [seqpar.bwd_finish(p["q"], p["k"], p["v"], p["a"], p["dO"], gathered, r, s0=d["s0"],
                              ds_final=dsT) for r, p in enumerate(parts)]
    assert gla.gla_get_device_status() == 0
    got = [_np(torch.cat([x[i] for x in outs], dim=1)) for i in range(4)]
    ref = recurrent.bwd(*(_np(d[n]) for n in ("q", "k", "v", "a", "dO")), _np(d["s0"]),
                        None if dsT is None else _np(dsT))
    _check_grads(got, ref)
    for x in outs:
        assert rel_l2(_np(x[4]), ref[4]) <= REL_STATE


def test_seqpar_long_prefill_eight_ranks_sampled():
    """T = 65,536 at B = 1, H = 16 (the long-prefill workload) cut into 8
    segments of 8,192: the split forward's o equals the unsplit gla_chunk_fwd's
    (both bf16 paths) to rel L2 <= 1e-3, and on two sampled heads o and the
    final state of both match the oracle run on the whole sequence.  (The
    final states of the two paths differ by more than o does: the unsplit
    path's last segment folds its state with a single bf16 copy of the
    decayed k, the split path's fold comes from the state-only pass, which
    keeps a hi + lo pair; both stay within the state bound.)"""
    B, T, H, R = 1, 65536, 16, 8
    d = inputs.chunk_inputs(B, T, H, seed=760, device="cuda", s0_std=0.1)
    parts = _split_inputs(d, [T // R] * R)
    gathered = torch.stack([seqpar.fwd_local(p["k"], p["v"], p["a"]) for p in parts])
    outs = [seqpar.fwd_finish(p["q"], p["k"], p["v"], p["a"], gathered, r, s0=d["s0"])
            for r, p in enumerate(parts)]
    o = torch.cat([x[0] for x in outs], dim=1)
    o_ref, s_ref = gla.gla_chunk_fwd(d["q"], d["k"], d["v"], d["a"], s0=d["s0"])
    assert gla.gla_get_device_status() == 0
    assert rel_l2(_np(o), _np(o_ref)) <= 1e-3
    assert rel_l2(_np(outs[-1][1]), _np(s_ref)) <= REL_STATE
    for h in (0, 13):
        sl = slice(h, h + 1)
        ro, rs = recurrent.fwd(*(_np(d[n][:, :, sl]) for n in ("q", "k", "v", "a")), _np(d["s0"][:, sl]))
        assert_bf16_close(_np(o[:, :, sl]), ro, "o head %d" % h)
        e_split, e_plain = rel_l2(_np(outs[0][1][:, sl]), rs), rel_l2(_np(s_ref[:, sl]), rs)
        print("head %d final state rel L2: split %.2e  unsplit %.2e" % (h, e_split, e_plain))
        assert e_split <= REL_STATE and e_plain <= REL_STATE
