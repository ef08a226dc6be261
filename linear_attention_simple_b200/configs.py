"""The five synthetic workloads of the Simple GLA mixer.

Shapes come from the Laplace 3B description ("Como i14 llevo Laplace 3B a AWS
Trainium2", sections "Diseno esencial de Laplace 3B" -- H = 16, dk = 96,
dv = 192, D = 3072, 24 layers, conv width 4 -- and "Adaptaciones para AWS
Trainium2" -- 16 chunks of 128 tokens; "Resultados de entrenamiento e
inferencia" -- 1,280 concurrent decode sequences).  Each workload is named by
what it is; the seed is fixed per workload.
"""
from dataclasses import dataclass, field

H, DK, DV, CHUNK = 16, 96, 192, 128
D_MODEL, CONV_W, LAYERS = 3072, 4, 24


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "fwd", "fwd_bwd", "decode", "front_fwd"
    B: int = 1
    T: int = 1
    H: int = H
    dk: int = DK
    dv: int = DV
    dtype: str = "bf16"
    s0_std: float = None
    seed: int = 0
    N: int = 0                # decode sequences
    layers: int = 1           # decode layers per step
    D: int = D_MODEL
    W: int = CONV_W
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    # tiny fp32 forward: 1 head, 2 chunks
    "tiny_fwd_fp32": Workload("tiny_fwd_fp32", "fwd", B=1, T=256, H=1, dtype="f32", seed=1001),
    # one Laplace layer's mixer, prefill forward at T = 2048
    "prefill_fwd_b8_t2048": Workload("prefill_fwd_b8_t2048", "fwd", B=8, T=2048, seed=1002),
    # training step of the same layer: forward then backward
    "train_fwd_bwd_b8_t2048": Workload("train_fwd_bwd_b8_t2048", "fwd_bwd", B=8, T=2048,
                                       seed=1003),
    # batched decode: 1280 sequences x 24 layers x 16 heads, fp32 state in place
    "decode_n1280_l24": Workload("decode_n1280_l24", "decode", N=1280, layers=LAYERS,
                                 seed=1004),
    # long-context prefill: LayerNorm + conv + SiLU front end, then GLA with S_0
    "long_prefill_t65536": Workload("long_prefill_t65536", "front_fwd", B=1, T=65536,
                                    s0_std=0.1, seed=1005),
}
