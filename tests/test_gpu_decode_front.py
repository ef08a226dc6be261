"""GPU parity: decode step, LayerNorm/conv/SiLU front end, fp32 forward, and
the bounded-wait failure path.  Every CUDA result is compared element by
element with the fp64 oracle on the same seeded inputs.

Tolerances (relative L2 = ||x - ref|| / ||ref||, ref = oracle):
  fp32 decode (state and o)      <= 1e-5
  fp32 forward (o and S_T)       <= 1e-5
  bf16 front end output y        <= 1e-2, max-abs <= 5e-2
"""
import numpy as np
import pytest
import torch

import linear_attention_simple_b200 as gla
from linear_attention_simple_b200 import inputs
from oracle import recurrent

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel(x, ref):
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


@pytest.fixture(scope="module", autouse=True)
def _build():
    from linear_attention_simple_b200 import build
    build.build()
    gla.lib()


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("N,H", [(1, 1), (37, 3), (256, 16)])
def test_decode_parity(N, H):
    d = inputs.decode_inputs(N, H, seed=20 + N, device="cuda")[0]
    st0 = _np(d["state"])
    o = gla.gla_decode_step(d["state"], d["q"], d["k"], d["v"], d["a"])
    ref_state, ref_o = recurrent.decode(st0, _np(d["q"]), _np(d["k"]), _np(d["v"]), _np(d["a"]))
    assert rel(_np(d["state"]), ref_state) <= 1e-5
    assert rel(_np(o), ref_o) <= 1e-5
    assert gla.gla_get_device_status() == 0


def test_decode_slot_indirection_leaves_other_slots_untouched():
    N, H, slots = 40, 4, 96
    d = inputs.decode_inputs(N, H, seed=31, device="cuda", n_slots=slots)[0]
    g = torch.Generator().manual_seed(5)
    idx = torch.randperm(slots, generator=g)[:N].to(torch.int32).cuda()
    before = d["state"].clone()
    o = gla.gla_decode_step(d["state"], d["q"], d["k"], d["v"], d["a"], slot_idx=idx)
    ref_state, ref_o = recurrent.decode(_np(before), _np(d["q"]), _np(d["k"]), _np(d["v"]),
                                        _np(d["a"]), slot_idx=idx.cpu().numpy())
    assert rel(_np(d["state"]), ref_state) <= 1e-5
    assert rel(_np(o), ref_o) <= 1e-5
    untouched = sorted(set(range(slots)) - set(idx.cpu().tolist()))
    assert torch.equal(d["state"][untouched], before[untouched])      # bit-exact


def test_decode_slot_outside_the_pool_is_skipped_and_reported():
    """A slot map entry outside [0, N_slots) (here N_slots and -1) touches no
    state and no output and records GLA_ERR_INVALID_ARG in the device status
    word; every other sequence is updated as usual.  The kernel checks the
    slot before any access, so the bad entries never address memory."""
    N, H, slots = 6, 2, 8
    d = inputs.decode_inputs(N, H, seed=32, device="cuda", n_slots=slots)[0]
    idx = torch.tensor([3, slots, 0, -1, 7, 5], dtype=torch.int32, device="cuda")
    good = [0, 2, 4, 5]
    before = d["state"].clone()
    o = torch.full((N, H, 192), 1234.5, dtype=torch.float32, device="cuda")
    gla.gla_decode_step(d["state"], d["q"], d["k"], d["v"], d["a"], o=o, slot_idx=idx)
    assert gla.gla_get_device_status() == 1                 # GLA_ERR_INVALID_ARG
    assert gla.gla_get_device_status() == 0                 # read clears it
    g = torch.tensor(good)
    ref_state, ref_o = recurrent.decode(_np(before), _np(d["q"][g]), _np(d["k"][g]), _np(d["v"][g]),
                                        _np(d["a"][g]), slot_idx=idx[g].cpu().numpy())
    assert rel(_np(d["state"]), ref_state) <= 1e-5
    assert rel(_np(o[g]), ref_o) <= 1e-5
    assert torch.all(o[[1, 3]] == 1234.5)                    # skipped rows not written
    untouched = sorted(set(range(slots)) - set(idx[g].cpu().tolist()))
    assert torch.equal(d["state"][untouched], before[untouched])


def test_decode_front_slot_outside_the_pool_is_skipped_and_reported():
    N, D, n_slots = 4, 256, 5
    x, w, pool, _ = _pool_inputs(N, D, n_slots, 66)
    idx = torch.tensor([1, n_slots, 4, -2], dtype=torch.int32, device="cuda")
    before = pool.clone()
    y = torch.full((N, D), 7.0, dtype=torch.bfloat16, device="cuda")
    gla.conv1d_silu_decode_step(x, w, pool, slot_idx=idx, y=y)
    assert gla.gla_get_device_status() == 1
    good = torch.tensor([0, 2])
    hist = _np(before[idx[good].long()])
    ref_y, ref_cs = recurrent.ln_conv_silu(_np(x[good])[:, None, :], _np(w), conv_state=hist)
    _front_check(_np(y[good]), ref_y[:, 0])
    assert rel(_np(pool[idx[good].long()]), ref_cs) <= 1e-5
    assert torch.all(y[[1, 3]] == 7.0)
    assert torch.equal(pool[[0, 2, 3]], before[[0, 2, 3]])


def test_decode_repeated_steps_match_recurrence():
    """T decode steps from S_0 equal the forward recurrence over T tokens."""
    N, H, T = 8, 2, 5
    d = inputs.chunk_inputs(N, T, H, seed=33, device="cuda", s0_std=0.1)
    state = d["s0"].clone()
    outs = []
    for t in range(T):
        outs.append(gla.gla_decode_step(state, d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                                        d["v"][:, t].contiguous(), d["a"][:, t].contiguous()))
    ref_o, ref_s = recurrent.fwd(_np(d["q"]), _np(d["k"]), _np(d["v"]), _np(d["a"]), _np(d["s0"]))
    assert rel(np.stack([_np(x) for x in outs], axis=1), ref_o) <= 1e-5
    assert rel(_np(state), ref_s) <= 1e-5


def test_decode_full_size_sampled():
    """1280 sequences x 16 heads (one layer of the 24-layer step, the launch the
    benchmark times), checked on 96 sampled (sequence, head) units."""
    N, H = 1280, 16
    d = inputs.decode_inputs(N, H, seed=1004, device="cuda")[0]
    g = torch.Generator().manual_seed(7)
    units = torch.randperm(N * H, generator=g)[:96]
    units = torch.cat([units, torch.tensor([0, N * H - 1])])
    n_idx, h_idx = units // H, units % H
    st0 = d["state"][n_idx, h_idx].clone()
    o = gla.gla_decode_step(d["state"], d["q"], d["k"], d["v"], d["a"])
    ref_state, ref_o = recurrent.decode(_np(st0)[:, None], _np(d["q"][n_idx, h_idx])[:, None],
                                        _np(d["k"][n_idx, h_idx])[:, None],
                                        _np(d["v"][n_idx, h_idx])[:, None],
                                        _np(d["a"][n_idx, h_idx])[:, None])
    assert rel(_np(d["state"][n_idx, h_idx]), ref_state[:, 0]) <= 1e-5
    assert rel(_np(o[n_idx, h_idx]), ref_o[:, 0]) <= 1e-5


# --------------------------------------------------------------- front end

def _front_check(y, ref):
    assert rel(y, ref) <= 1e-2
    assert float(np.max(np.abs(y - ref))) <= 5e-2


@pytest.mark.parametrize("B,T,D,hist,affine", [(1, 1, 256, False, False), (2, 37, 256, True, True), (3, 1000, 4096, True, True), (1, 200, 64, True, False),
                                               (3, 300, 3072, True, False), (1, 2, 64, True, True)])
def test_front_end_parity(B, T, D, hist, affine):
    d = inputs.front_inputs(B, T, D, seed=40 + T, device="cuda", with_state=hist)
    g = b = bias = None
    if affine:
        g = inputs.randn((D,), 41, "cuda", std=0.5) + 1.0
        b = inputs.randn((D,), 42, "cuda", std=0.5)
        bias = inputs.randn((D,), 43, "cuda", std=0.5)
    cs_out = torch.empty((B, 3, D), dtype=torch.float32, device="cuda")
    y = gla.conv1d_silu_causal(d["x"], d["w"], ln_gamma=g, ln_beta=b, bias=bias,
                               conv_state_in=d["conv_state"], conv_state_out=cs_out)
    ref_y, ref_cs = recurrent.ln_conv_silu(_np(d["x"]), _np(d["w"]), ln=True,
                                           ln_gamma=None if g is None else _np(g),
                                           ln_beta=None if b is None else _np(b),
                                           bias=None if bias is None else _np(bias),
                                           conv_state=None if d["conv_state"] is None
                                           else _np(d["conv_state"]))
    _front_check(_np(y), ref_y)
    assert rel(_np(cs_out), ref_cs) <= 1e-5


def test_front_end_without_layernorm():
    d = inputs.front_inputs(2, 50, 512, seed=44, device="cuda", with_state=True)
    y = gla.conv1d_silu_causal(d["x"], d["w"], apply_ln=False, conv_state_in=d["conv_state"])
    ref_y, _ = recurrent.ln_conv_silu(_np(d["x"]), _np(d["w"]), ln=False,
                                      conv_state=_np(d["conv_state"]))
    _front_check(_np(y), ref_y)


def test_front_end_chained_calls_equal_one_call():
    """Carrying conv_state_out into the next call reproduces the unsplit run."""
    B, T, D, split = 1, 90, 512, 41
    d = inputs.front_inputs(B, T, D, seed=45, device="cuda")
    y_full = gla.conv1d_silu_causal(d["x"], d["w"])
    cs = torch.empty((B, 3, D), dtype=torch.float32, device="cuda")
    y1 = gla.conv1d_silu_causal(d["x"][:, :split].contiguous(), d["w"], conv_state_out=cs)
    y2 = gla.conv1d_silu_causal(d["x"][:, split:].contiguous(), d["w"], conv_state_in=cs)
    y_split = torch.cat([y1, y2], dim=1)
    # bf16 outputs: the two runs do the same fp32 arithmetic per element
    assert rel(_np(y_split), _np(y_full)) <= 1e-6


def test_front_end_full_size_sampled():
    """T = 65536, D = 3072 (the long-context prefill front end, as benchmarked),
    checked on sampled tokens including CTA boundaries and both ends."""
    B, T, D = 1, 65536, 3072
    d = inputs.front_inputs(B, T, D, seed=1005, device="cuda")
    y = gla.conv1d_silu_causal(d["x"], d["w"])
    g = torch.Generator().manual_seed(9)
    toks = sorted(set(torch.randint(0, T, (40,), generator=g).tolist()) |
                  {0, 1, 2, 3, 221, 222, 223, 224, T - 1})
    x = _np(d["x"])
    w = _np(d["w"])
    ys = _np(y)
    got, ref = [], []
    for t in toks:
        lo = max(0, t - 3)
        r, _ = recurrent.ln_conv_silu(x[:, lo:t + 1], w)
        got.append(ys[:, t])
        ref.append(r[:, -1])
    _front_check(np.stack(got), np.stack(ref))


# ---------------------------------------------------- decode front end

def _pool_inputs(N, D, n_slots, seed):
    g = torch.Generator().manual_seed(seed)
    x = inputs.randn((N, D), seed, "cuda").to(torch.bfloat16)
    w = inputs.randn((D, 4), seed + 1, "cuda", std=0.5)
    pool = inputs.randn((n_slots, 3, D), seed + 2, "cuda")
    idx = torch.randperm(n_slots, generator=g)[:N].to(torch.int32).cuda()
    return x, w, pool, idx


@pytest.mark.parametrize("N,D,affine", [(1, 8, False), (37, 256, True), (64, 4096, True), (5, 3072, False)])
def test_decode_front_parity_with_slot_pool(N, D, affine):
    n_slots = 2 * N + 3
    x, w, pool, idx = _pool_inputs(N, D, n_slots, 60 + N)
    g = b = bias = None
    if affine:
        g = inputs.randn((D,), 61, "cuda", std=0.5) + 1.0
        b = inputs.randn((D,), 62, "cuda", std=0.5)
        bias = inputs.randn((D,), 63, "cuda", std=0.5)
    before = pool.clone()
    y = gla.conv1d_silu_decode_step(x, w, pool, slot_idx=idx, ln_gamma=g, ln_beta=b, bias=bias)
    hist = _np(before[idx.long()])                                  # [N, 3, D]
    ref_y, ref_cs = recurrent.ln_conv_silu(_np(x)[:, None, :], _np(w), ln=True,
                                           ln_gamma=None if g is None else _np(g),
                                           ln_beta=None if b is None else _np(b),
                                           bias=None if bias is None else _np(bias), conv_state=hist)
    _front_check(_np(y), ref_y[:, 0])
    after = pool[idx.long()]
    assert rel(_np(after), ref_cs) <= 1e-5
    # the two older rows move down unchanged (bit-exact); other slots untouched
    assert torch.equal(after[:, :2], before[idx.long()][:, 1:])
    untouched = sorted(set(range(n_slots)) - set(idx.cpu().tolist()))
    assert torch.equal(pool[untouched], before[untouched])


def test_decode_front_steps_equal_the_sequence_front_end():
    """T decode steps from a given history reproduce the oracle's front end over
    the T tokens, and leave the oracle's final history in the slots."""
    N, D, T = 6, 512, 9
    d = inputs.front_inputs(N, T, D, seed=64, device="cuda", with_state=True)
    pool = d["conv_state"].clone()
    ys = [gla.conv1d_silu_decode_step(d["x"][:, t].contiguous(), d["w"], pool) for t in range(T)]
    ref_y, ref_cs = recurrent.ln_conv_silu(_np(d["x"]), _np(d["w"]), conv_state=_np(d["conv_state"]))
    _front_check(np.stack([_np(y) for y in ys], axis=1), ref_y)
    assert rel(_np(pool), ref_cs) <= 1e-5


def test_decode_front_without_layernorm():
    N, D = 16, 1024
    x, w, pool, _ = _pool_inputs(N, D, N, 65)
    before = pool.clone()
    y = gla.conv1d_silu_decode_step(x, w, pool, apply_ln=False)
    ref_y, ref_cs = recurrent.ln_conv_silu(_np(x)[:, None, :], _np(w), ln=False, conv_state=_np(before))
    _front_check(_np(y), ref_y[:, 0])
    assert rel(_np(pool), ref_cs) <= 1e-6


def test_decode_front_full_size_sampled():
    """1,280 sequences x D = 3,072 (one layer of the decode step's front end),
    checked on sampled sequences."""
    N, D = 1280, 3072
    x, w, pool, idx = _pool_inputs(N, D, 2 * N, 1006)
    before = pool.clone()
    y = gla.conv1d_silu_decode_step(x, w, pool, slot_idx=idx)
    g = torch.Generator().manual_seed(11)
    pick = torch.cat([torch.randperm(N, generator=g)[:64], torch.tensor([0, N - 1])])
    hist = _np(before[idx[pick].long()])
    ref_y, ref_cs = recurrent.ln_conv_silu(_np(x[pick])[:, None, :], _np(w), conv_state=hist)
    _front_check(_np(y[pick]), ref_y[:, 0])
    assert rel(_np(pool[idx[pick].long()]), ref_cs) <= 1e-5


# -------------------------------------------------------------- fp32 path

@pytest.mark.parametrize("B,T,H,s0", [(1, 256, 1, False), (2, 77, 3, True), (1, 1, 1, True)])
def test_fwd_fp32_parity(B, T, H, s0):
    d = inputs.chunk_inputs(B, T, H, dtype=torch.float32, seed=50 + T, device="cuda",
                            s0_std=0.1 if s0 else None)
    o, sf = gla.gla_chunk_fwd(d["q"], d["k"], d["v"], d["a"], s0=d["s0"])
    ro, rs = recurrent.fwd(_np(d["q"]), _np(d["k"]), _np(d["v"]), _np(d["a"]),
                           None if d["s0"] is None else _np(d["s0"]))
    assert rel(_np(o), ro) <= 1e-5
    assert rel(_np(sf), rs) <= 1e-5


def test_fwd_empty_sequence_copies_state():
    d = inputs.chunk_inputs(2, 0, 3, seed=51, device="cuda", s0_std=0.1)
    o, sf = gla.gla_chunk_fwd(d["q"], d["k"], d["v"], d["a"], s0=d["s0"])
    torch.cuda.synchronize()
    assert o.numel() == 0
    assert torch.equal(sf, d["s0"])


# ------------------------------------------------------ failure detection

def test_bounded_wait_reports_timeout_and_context_survives():
    gla.gla_set_wait_limit_ns(5_000_000)          # 5 ms
    try:
        assert gla.gla_get_device_status() == 0
        gla.gla_selftest_wait_timeout()
        assert gla.gla_get_device_status() == 5     # GLA_ERR_TIMEOUT, then cleared
        assert gla.gla_get_device_status() == 0
    finally:
        gla.gla_set_wait_limit_ns(0)
    # the context is still usable
    d = inputs.decode_inputs(4, 2, seed=52, device="cuda")[0]
    st0 = _np(d["state"])
    o = gla.gla_decode_step(d["state"], d["q"], d["k"], d["v"], d["a"])
    ref_state, ref_o = recurrent.decode(st0, _np(d["q"]), _np(d["k"]), _np(d["v"]), _np(d["a"]))
    assert rel(_np(o), ref_o) <= 1e-5
