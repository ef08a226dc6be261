"""GPU parity of the packed-sequence (varlen) chunked forward: every sequence
against the fp64 oracle run on that sequence alone, and against
gla_chunk_fwd called per sequence.  Tolerances as the dense forward's
(tests/tolerances.py): o bf16 bound, final states rel L2 <= 5e-3."""
import numpy as np
import pytest
import torch

import linear_attention_simple_b200 as gla
from linear_attention_simple_b200 import inputs
from oracle import recurrent
from tolerances import REL_STATE, assert_bf16_close, rel_l2

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.fixture(scope="module", autouse=True)
def _build():
    from linear_attention_simple_b200 import build
    build.build()
    gla.lib()


def _packed(lengths, H, seed, lead=0, trail=0, s0=True):
    total = lead + sum(lengths) + trail
    d = inputs.chunk_inputs(1, total, H, seed=seed, device="cuda", s0_std=None)
    q, k, v, a = (d[n][0].contiguous() for n in ("q", "k", "v", "a"))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]) + lead, dtype=torch.int32, device="cuda")
    st0 = inputs.randn((len(lengths), H, 96, 192), seed + 1, "cuda", std=0.1) if s0 else None
    return q, k, v, a, cu, st0


def test_varlen_parity_and_untouched_rows():
    lengths = [1, 127, 128, 129, 300, 0, 777]
    H = 3
    q, k, v, a, cu, s0 = _packed(lengths, H, seed=90, lead=5, trail=7)
    o = torch.full((q.shape[0], H, 192), float("nan"), dtype=torch.bfloat16, device="cuda")
    o, sf = gla.gla_chunk_fwd_varlen(q, k, v, a, cu, s0=s0, o=o)
    assert gla.gla_get_device_status() == 0
    c = cu.cpu().numpy()
    for n in range(len(lengths)):
        lo, hi = int(c[n]), int(c[n + 1])
        ro, rs = recurrent.fwd(_np(q[lo:hi])[None], _np(k[lo:hi])[None], _np(v[lo:hi])[None],
                               _np(a[lo:hi])[None], _np(s0[n])[None])
        if hi > lo:
            assert_bf16_close(_np(o[lo:hi]), ro[0], "o of sequence %d" % n)
        assert rel_l2(_np(sf[n]), rs[0]) <= REL_STATE
    # rows outside every sequence stay as they were
    assert torch.isnan(o[:5].float()).all() and torch.isnan(o[-7:].float()).all()


def test_varlen_equals_per_sequence_calls():
    lengths = [300, 128, 1000, 2]
    H = 4
    q, k, v, a, cu, s0 = _packed(lengths, H, seed=91)
    o, sf = gla.gla_chunk_fwd_varlen(q, k, v, a, cu, s0=s0)
    c = cu.cpu().numpy()
    for n in range(len(lengths)):
        lo, hi = int(c[n]), int(c[n + 1])
        od, sd = gla.gla_chunk_fwd(q[lo:hi][None].contiguous(), k[lo:hi][None].contiguous(),
                                   v[lo:hi][None].contiguous(), a[lo:hi][None].contiguous(),
                                   s0=s0[n][None].contiguous())
        # with few heads the dense call takes the segmented path (segment
        # states combined in fp32), so the two sum in different orders
        assert rel_l2(_np(o[lo:hi]), _np(od[0])) <= 1e-3
        assert rel_l2(_np(sf[n]), _np(sd[0])) <= 1e-3


def test_varlen_bad_offsets_are_reported_and_nothing_written():
    H = 2
    q, k, v, a, cu, _ = _packed([100, 50], H, seed=92, s0=False)
    bad = torch.tensor([0, 100, q.shape[0] + 10], dtype=torch.int32, device="cuda")
    o = torch.zeros((q.shape[0], H, 192), dtype=torch.bfloat16, device="cuda")
    gla.gla_chunk_fwd_varlen(q, k, v, a, bad, o=o)
    assert gla.gla_get_device_status() == 1            # GLA_ERR_INVALID_ARG, then cleared
    assert gla.gla_get_device_status() == 0
    assert float(o[100:].float().abs().max()) == 0.0   # the bad sequence wrote nothing


def test_varlen_prefill_size_sampled():
    """16,384 tokens in 8 sequences of mixed lengths, H = 16 (the prefill
    workload's tokens and heads), sampled (sequence, head) units."""
    lengths = [2048, 1000, 3000, 500, 4096, 1, 129, 5610]
    H = 16
    q, k, v, a, cu, s0 = _packed(lengths, H, seed=1008)
    o, sf = gla.gla_chunk_fwd_varlen(q, k, v, a, cu, s0=s0)
    c = cu.cpu().numpy()
    for n, h in ((0, 0), (2, 7), (4, 15), (7, 3), (6, 9)):
        lo, hi = int(c[n]), int(c[n + 1])
        ro, rs = recurrent.fwd(_np(q[lo:hi, h])[None, :, None], _np(k[lo:hi, h])[None, :, None],
                               _np(v[lo:hi, h])[None, :, None], _np(a[lo:hi, h])[None, :, None],
                               _np(s0[n, h])[None, None])
        assert_bf16_close(_np(o[lo:hi, h]), ro[0, :, 0], "o (%d, %d)" % (n, h))
        assert rel_l2(_np(sf[n, h]), rs[0, 0]) <= REL_STATE


def test_varlen_long_sequence_among_short_ones_is_segmented():
    """One 16,384-token sequence among short ones, with initial states: the
    long sequence is cut into segments (pre-pass, fold, output pass) and
    every sequence still matches the oracle run on it alone; the result also
    matches the unsegmented sweep (the fold only regroups the sums)."""
    lengths = [3, 16384, 128, 700, 1, 2000]
    H = 4
    q, k, v, a, cu, s0 = _packed(lengths, H, seed=93)
    total = q.shape[0]
    assert gla.gla_chunk_varlen_workspace_bytes(len(lengths), total, H) > 0
    o, sf = gla.gla_chunk_fwd_varlen(q, k, v, a, cu, s0=s0)
    assert gla.gla_get_device_status() == 0
    c = cu.cpu().numpy()
    for n in range(len(lengths)):
        lo, hi = int(c[n]), int(c[n + 1])
        ro, rs = recurrent.fwd(_np(q[lo:hi])[None], _np(k[lo:hi])[None], _np(v[lo:hi])[None],
                               _np(a[lo:hi])[None], _np(s0[n])[None])
        r = assert_bf16_close(_np(o[lo:hi]), ro[0], "o of sequence %d" % n)
        es = rel_l2(_np(sf[n]), rs[0])
        assert es <= REL_STATE, "S_T of sequence %d rel L2 %.3g" % (n, es)
        print("sequence %d (%d tokens): o rel %.3g raw-max %.3g beyond-rounding %.3g, S_T rel %.3g"
              % ((n, hi - lo) + r + (es,)))
    o1, sf1 = gla.gla_chunk_fwd_varlen(q, k, v, a, cu, s0=s0, segmented=False)
    assert rel_l2(_np(o), _np(o1)) <= 1e-3
    assert rel_l2(_np(sf), _np(sf1)) <= 1e-3


@pytest.mark.parametrize("name,lengths", [
    ("8 sequences of 1 to 5,610 tokens", [5610, 1, 3000, 2048, 777, 129, 4000, 819]),
    ("one 16,384-token sequence among 7 short ones", [16384, 500, 300, 1000, 200, 700, 100, 50]),
    ("8 equal sequences of 2,048 tokens", [2048] * 8),
])
def test_varlen_segmented_time(name, lengths):
    """Packed sequences at H = 16: the segmented and the one-sweep-per-sequence
    forward, timed with CUDA events (printed), and equal to each other.  With
    equal lengths the device plan does not split (both paths do the same
    work)."""
    H = 16
    q, k, v, a, cu, s0 = _packed(lengths, H, seed=94)
    ws = torch.empty(max(1, gla.gla_chunk_varlen_workspace_bytes(len(lengths), q.shape[0], H)),
                     dtype=torch.uint8, device="cuda")
    o = torch.empty((q.shape[0], H, 192), dtype=torch.bfloat16, device="cuda")
    sf = torch.empty((len(lengths), H, 96, 192), dtype=torch.float32, device="cuda")
    times = {}
    outs = {}
    for seg in (False, True):
        run = lambda: gla.gla_chunk_fwd_varlen(q, k, v, a, cu, s0=s0, o=o, s_final=sf,  # noqa: E731
                                               ws=ws if seg else None, segmented=seg)
        for _ in range(3):
            run()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            run()
        e1.record()
        e1.synchronize()
        times[seg] = e0.elapsed_time(e1) / 10 * 1e3
        outs[seg] = (o.clone(), sf.clone())
    assert gla.gla_get_device_status() == 0
    print("packed forward, %s (%d tokens), H = 16: one sweep per sequence %.1f us, segmented %.1f us"
          % (name, sum(lengths), times[False], times[True]))
    assert rel_l2(_np(outs[True][0]), _np(outs[False][0])) <= 1e-3
    assert rel_l2(_np(outs[True][1]), _np(outs[False][1])) <= 1e-3
