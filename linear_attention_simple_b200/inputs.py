"""Seeded synthetic inputs for the Simple GLA mixer.

This module only draws random numbers in the shapes and distributions of the
workloads; it contains none of the mixer's arithmetic.  Both the CUDA path's
tests/benchmark and the CPU oracle's tests take their inputs from here.

Distributions (the workloads of "Como i14 llevo Laplace 3B a AWS Trainium2",
sections "Diseno esencial de Laplace 3B" and "Adaptaciones para AWS
Trainium2": H = 16, dk = 96, dv = 192, T = 2048 = 16 x 128, D = 3072, conv
width 4; decode at 1,280 concurrent sequences from "Resultados de
entrenamiento e inferencia"):
  q, k, v, dO      ~ N(0, 1), cast to the compute dtype (bf16 or fp32)
  a (log-decay)    = logsigmoid(z), z ~ N(3, 1), fp32, so a < 0 with mean ~ -0.075
  S_0, decode S    ~ N(0, 0.1^2) fp32  (0.1 is the standard deviation)
  x (front end)    ~ N(0, 1) bf16;  conv weight w ~ N(0, 0.5^2) fp32
Draw order is fixed per function, so a seed fully determines the tensors.
"""
import torch
import torch.nn.functional as F


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn(shape, seed, device="cpu", std=1.0, dtype=torch.float32):
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def log_decay(shape, seed, device="cpu", mean=3.0, std=1.0):
    """a = logsigmoid(z), z ~ N(mean, std^2); fp32."""
    z = randn(shape, seed, device, std=std)
    z.add_(mean)
    return F.logsigmoid(z)


def chunk_inputs(B, T, H, dk=96, dv=192, dtype=torch.bfloat16, seed=0, device="cpu",
                 s0_std=None, with_dO=False, ld=None):
    """q, k [B,T,H,dk]; v [B,T,H,dv] in ``dtype``; a [B,T,H] fp32; optional
    s0 [B,H,dk,dv] fp32 and dO [B,T,H,dv] in ``dtype``.

    With ``ld`` (elements per token, >= H*(2dk+2dv)), q, k and v are views of
    one fused [B,T,ld] projection buffer laid out as [q | k | v | rest],
    each head-major inside its part, so their token stride is ``ld``.
    """
    out = {}
    if ld is None:
        out["q"] = randn((B, T, H, dk), seed * 16 + 1, device, dtype=dtype)
        out["k"] = randn((B, T, H, dk), seed * 16 + 2, device, dtype=dtype)
        out["v"] = randn((B, T, H, dv), seed * 16 + 3, device, dtype=dtype)
    else:
        assert ld >= H * (2 * dk + dv)
        buf = randn((B, T, ld), seed * 16 + 1, device, dtype=dtype)
        out["fused"] = buf
        out["q"] = buf[:, :, 0:H * dk].unflatten(2, (H, dk))
        out["k"] = buf[:, :, H * dk:2 * H * dk].unflatten(2, (H, dk))
        out["v"] = buf[:, :, 2 * H * dk:2 * H * dk + H * dv].unflatten(2, (H, dv))
    out["a"] = log_decay((B, T, H), seed * 16 + 4, device)
    out["s0"] = None if s0_std is None else randn((B, H, dk, dv), seed * 16 + 5, device, std=s0_std)
    if with_dO:
        out["dO"] = randn((B, T, H, dv), seed * 16 + 6, device, dtype=dtype)
    return out


def decode_inputs(N, H, dk=96, dv=192, seed=0, device="cpu", layers=1, state_std=0.1,
                  n_slots=None):
    """Per layer: state [N_slots,H,dk,dv] fp32 ~ N(0, state_std^2); q, k [N,H,dk]
    and v [N,H,dv] bf16 ~ N(0,1); a [N,H] fp32 = logsigmoid(N(3,1))."""
    n_slots = N if n_slots is None else n_slots
    out = []
    for layer in range(layers):
        s = seed * 1000 + layer * 8
        out.append({
            "state": randn((n_slots, H, dk, dv), s + 1, device, std=state_std),
            "q": randn((N, H, dk), s + 2, device, dtype=torch.bfloat16),
            "k": randn((N, H, dk), s + 3, device, dtype=torch.bfloat16),
            "v": randn((N, H, dv), s + 4, device, dtype=torch.bfloat16),
            "a": log_decay((N, H), s + 5, device),
        })
    return out


def front_inputs(B, T, D=3072, W=4, seed=0, device="cpu", w_std=0.5, with_state=False):
    """x [B,T,D] bf16 ~ N(0,1); w [D,W] fp32 ~ N(0, w_std^2); optional conv
    history [B,W-1,D] fp32 ~ N(0,1)."""
    out = {
        "x": randn((B, T, D), seed * 16 + 7, device, dtype=torch.bfloat16),
        "w": randn((D, W), seed * 16 + 8, device, std=w_std),
    }
    out["conv_state"] = randn((B, W - 1, D), seed * 16 + 9, device) if with_state else None
    return out
