"""Independent NumPy chunked evaluation of the Simple GLA forward (fp64).

TEST INFRASTRUCTURE ONLY.  Used to pin the claim that the chunked form is an
exact reorganisation of the recurrence: the result must not depend on the
chunk size C ("Como i14 llevo Laplace 3B a AWS Trainium2", section
"Adaptaciones para AWS Trainium2", item 1, where T = 2048 is cut into 16
chunks of 128 tokens; any C, including one that does not divide T, must give
the same answer).

For a chunk of tokens [t0, t0+C) with local cumulative decay b_i (sum of a
over the chunk up to and including token i) and gamma = b_last:

    o_i   = scale * ( exp(b_i) q_i S_prev
                      + sum_{j<=i in chunk} exp(b_i - b_j) (q_i . k_j) v_j )
    S_new = exp(gamma) S_prev + sum_j exp(gamma - b_j) k_j^T v_j
"""
import numpy as np


def chunked(q, k, v, a, s0=None, scale=None, C=128):
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
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], np.float64)
            for t0 in range(0, T, C):
                t1 = min(t0 + C, T)
                qc, kc, vc = q[b, t0:t1, h], k[b, t0:t1, h], v[b, t0:t1, h]
                bl = np.cumsum(a[b, t0:t1, h])
                n = t1 - t0
                mask = np.tril(np.ones((n, n), dtype=bool))
                dmat = np.where(mask, np.exp(np.where(mask, bl[:, None] - bl[None, :], 0.0)), 0.0)
                intra = (dmat * (qc @ kc.T)) @ vc
                inter = np.exp(bl)[:, None] * (qc @ S)
                o[b, t0:t1, h] = scale * (inter + intra)
                g = bl[-1]
                S = np.exp(g) * S + (kc * np.exp(g - bl)[:, None]).T @ vc
            sT[b, h] = S
    return o, sT
