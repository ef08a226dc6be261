"""One long sequence split across the ranks of a process group.

Rank r of R holds tokens [t_r, t_{r+1}) of every (batch, head) sequence
(consecutive segments in rank order; lengths may differ, and may be 0).  The
chunked forward and backward are exact on each segment once the state
entering it (and, for the backward, the state gradient leaving it) is known,
and both follow from one exchange, because the state is linear in its inputs
(page "Como i14 llevo Laplace 3B a AWS Trainium2", section "Adaptaciones para
AWS Trainium2", item 1: the chunked form only regroups the recurrence; the
long-document use is the one of section "Por qué atención lineal importa"):

  1. local: each rank's segment state from zero L_r, its total log-decay
     G_r and (backward) the state gradient D_r its own outputs send back
     (gla_segment_state_fwd / gla_segment_state_bwd);
  2. exchange: one all_gather of B*H*(dk*dv + 1) floats per rank
     (B*H*(2*dk*dv + 1) for the backward);
  3. finish: S_in(r) = fold of (G_j, L_j), j < r, from S_0; dS_out(r) =
     fold of (G_j, D_j), j > r, right to left, from dS_T (gla_state_fold);
     then gla_chunk_fwd / gla_chunk_bwd on the rank's own tokens.

Every rank returns the global final state (forward) and the global dS_0
(backward), folded from the gathered entries.  The arithmetic runs in
libgla's kernels; this module only orders the calls and the exchange.  The
exchange uses torch.distributed (NCCL over NVLink on GPUs); it is a few MB at
most, once per call.

The two phases are separate functions (``fwd_local`` / ``fwd_finish``,
``bwd_local`` / ``bwd_finish``) so that callers can run the exchange
themselves, e.g. all ranks' phases one after another on one device.

``ops`` is the set of per-segment calls the phases make: ``LibglaOps``
(libgla's kernels) unless a caller passes another.  The package defines no
other set; the tests pass a host one to check the exchange on CPU ranks.
"""
import torch
import torch.distributed as dist

import linear_attention_simple_b200 as gla


class LibglaOps:
    """The libgla calls each phase makes (tensors on the current CUDA device)."""

    @staticmethod
    def segment_state_fwd(k, v, a):
        return gla.gla_segment_state_fwd(k, v, a)

    @staticmethod
    def segment_state_bwd(q, dO, a, scale):
        return gla.gla_segment_state_bwd(q, dO, a, scale=scale)[0]

    @staticmethod
    def state_fold(s, g, reverse, s_in):
        return gla.gla_state_fold(s, g, reverse=reverse, s_in=s_in)

    @staticmethod
    def chunk_fwd(q, k, v, a, s0, scale):
        return gla.gla_chunk_fwd(q, k, v, a, s0=s0, scale=scale, want_final_state=False)[0]

    @staticmethod
    def chunk_bwd(q, k, v, a, dO, s0, ds_final, scale):
        return gla.gla_chunk_bwd(q, k, v, a, dO, s0=s0, ds_final=ds_final, scale=scale,
                                 want_grad_s0=False)[:4]


def _dims(q, v):
    B, _, H, dk = q.shape
    return B, H, dk, v.shape[-1]


def _group_rank(group):
    return dist.get_world_size(group), dist.get_rank(group)


def exchange(flat, group=None):
    """All ranks' ``flat`` vectors, stacked in rank order: [R, n]."""
    R, _ = _group_rank(group)
    out = [torch.empty_like(flat) for _ in range(R)]
    dist.all_gather(out, flat.contiguous(), group=group)
    return torch.stack(out)


def _split(gathered, nstates, B, H, dk, dv):
    """[R, nstates*B*H*dk*dv + B*H] -> nstates arrays [R,B,H,dk,dv] and g [R,B,H]."""
    R = gathered.shape[0]
    ss = B * H * dk * dv
    states = [gathered[:, i * ss:(i + 1) * ss].contiguous().view(R, B, H, dk, dv) for i in range(nstates)]
    g = gathered[:, nstates * ss:].contiguous().view(R, B, H)
    return states, g


def fwd_local(k, v, a, ops=LibglaOps):
    """Phase 1 of the forward: [L_r, G_r] of this rank's segment, flat."""
    s, g = ops.segment_state_fwd(k, v, a)
    return torch.cat([s.reshape(-1), g.reshape(-1)])


def fwd_finish(q, k, v, a, gathered, rank, s0=None, scale=None, ops=LibglaOps):
    """Phase 3 of the forward for rank ``rank`` given every rank's phase-1
    vector ([R, n]).  Returns (o of this rank's tokens, global final state)."""
    B, H, dk, dv = _dims(q, v)
    sc = dk ** -0.5 if scale is None else scale
    (L,), g = _split(gathered, 1, B, H, dk, dv)
    s_in = ops.state_fold(L[:rank], g[:rank], False, s0) if rank > 0 else s0
    o = ops.chunk_fwd(q, k, v, a, s_in, sc)
    return o, ops.state_fold(L, g, False, s0)


def chunk_fwd_seqpar(q, k, v, a, s0=None, scale=None, group=None, ops=LibglaOps):
    """Forward of a sequence split across ``group``: this rank's segment of
    q, k [B,T_r,H,dk], v [B,T_r,H,dv], a [B,T_r,H]; s0 [B,H,dk,dv] the state
    before the whole sequence (the same on every rank, or None).  Returns
    (o [B,T_r,H,dv], global final state [B,H,dk,dv])."""
    _, rank = _group_rank(group)
    gathered = exchange(fwd_local(k, v, a, ops), group)
    return fwd_finish(q, k, v, a, gathered, rank, s0, scale, ops)


def bwd_local(q, k, v, a, dO, scale=None, ops=LibglaOps):
    """Phase 1 of the backward: [L_r, D_r, G_r] of this rank's segment, flat."""
    dk = q.shape[-1]
    sc = dk ** -0.5 if scale is None else scale
    s, g = ops.segment_state_fwd(k, v, a)
    d = ops.segment_state_bwd(q, dO, a, sc)
    return torch.cat([s.reshape(-1), d.reshape(-1), g.reshape(-1)])


def bwd_finish(q, k, v, a, dO, gathered, rank, s0=None, ds_final=None, scale=None, ops=LibglaOps):
    """Phase 3 of the backward.  Returns (dq, dk, dv, da) of this rank's
    tokens and the global dL/dS_0."""
    B, H, dk, dv = _dims(q, v)
    sc = dk ** -0.5 if scale is None else scale
    (L, D), g = _split(gathered, 2, B, H, dk, dv)
    R = L.shape[0]
    s_in = ops.state_fold(L[:rank], g[:rank], False, s0) if rank > 0 else s0
    ds_out = (ops.state_fold(D[rank + 1:], g[rank + 1:], True, ds_final) if rank + 1 < R else ds_final)
    grads = ops.chunk_bwd(q, k, v, a, dO, s_in, ds_out, sc)
    ds0 = ops.state_fold(D, g, True, ds_final)
    return tuple(grads) + (ds0,)


def chunk_bwd_seqpar(q, k, v, a, dO, s0=None, ds_final=None, scale=None, group=None, ops=LibglaOps):
    """Backward of a sequence split across ``group`` (inputs as
    chunk_fwd_seqpar, plus this rank's dO and the gradient of the global
    final state, the same on every rank, or None).  Returns (dq, dk, dv, da)
    of this rank's tokens and the global dL/dS_0."""
    _, rank = _group_rank(group)
    gathered = exchange(bwd_local(q, k, v, a, dO, scale, ops), group)
    return bwd_finish(q, k, v, a, dO, gathered, rank, s0, ds_final, scale, ops)
