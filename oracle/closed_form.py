"""Independent NumPy closed forms of the Simple GLA forward (fp64).

TEST INFRASTRUCTURE ONLY.  These are the pins for the C recurrence: code
written separately, from the unrolled recurrence rather than the loop.

Unrolling S_t = exp(a_t) S_{t-1} + k_t^T v_t from S_0 gives, with
A_t = sum_{u<=t} a_u,

    S_t = exp(A_t) S_0 + sum_{s<=t} exp(A_t - A_s) k_s^T v_s
    o_t = scale * ( sum_{s<=t} exp(A_t - A_s) (q_t . k_s) v_s + exp(A_t) q_t S_0 )

(the fixed-size decaying state of "AWS serve Laplace 3B di i14 con uno stato
fisso di 29,5 MB", section "GLA sostituisce i token conservati con uno stato
ricorrente", written out as the quadratic form that O(T^2) attention would
compute -- "Como i14 llevo Laplace 3B a AWS Trainium2", section "Por que
atencion lineal importa").
"""
import numpy as np


def quadratic(q, k, v, a, s0=None, scale=None):
    """O(T^2) evaluation.  Shapes as in oracle.recurrent.fwd."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    a = np.asarray(a, np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if scale is None:
        scale = dk ** -0.5
    o = np.zeros((B, T, H, dv))
    sT = np.zeros((B, H, dk, dv))
    causal = np.tril(np.ones((T, T), dtype=bool))
    for b in range(B):
        for h in range(H):
            A = np.cumsum(a[b, :, h])
            diff = A[:, None] - A[None, :]
            decay = np.where(causal, np.exp(np.where(causal, diff, 0.0)), 0.0)
            scores = q[b, :, h, :] @ k[b, :, h, :].T
            out = (decay * scores) @ v[b, :, h, :]
            wT = np.exp(A[-1] - A)  # weight of token s in S_T
            st = (k[b, :, h, :] * wT[:, None]).T @ v[b, :, h, :]
            if s0 is not None:
                S0 = np.asarray(s0, np.float64)[b, h]
                out = out + np.exp(A)[:, None] * (q[b, :, h, :] @ S0)
                st = st + np.exp(A[-1]) * S0
            o[b, :, h, :] = scale * out
            sT[b, h] = st
    return o, sT


def causal_linear_attention(q, k, v, scale=None):
    """The a == 0 special case: plain causal linear attention,
    o = scale * ((Q K^T) masked to the lower triangle) V."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, T, H, dk = q.shape
    if scale is None:
        scale = dk ** -0.5
    o = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            s = np.tril(q[b, :, h, :] @ k[b, :, h, :].T)
            o[b, :, h, :] = scale * (s @ v[b, :, h, :])
    return o
