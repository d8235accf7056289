"""Shapes of the MoE decode workloads and the layer configuration.

A configuration holds sizes and switches only; no arithmetic of the method
lives here.  Field names follow the notation used throughout the library:
H hidden size, E routed experts, k experts chosen per token, I routed-expert
intermediate size, Is shared-expert intermediate size, S cache slots per
layer.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

GROUP = 64          # weights per quantisation group (one fp16 scale + bias)
GELU_TANH = 0       # GELU(g) = 0.5 g (1 + tanh(sqrt(2/pi)(g + 0.044715 g^3)))
GELU_ERF = 1        # GELU(g) = 0.5 g (1 + erf(g / sqrt 2))


@dataclass(frozen=True)
class MoeConfig:
    H: int = 2816
    E: int = 128
    k: int = 8
    I: int = 704
    Is: int = 2112
    S: int = 16
    renorm: int = 1          # top-k routing weights renormalised over the k
    gelu: int = GELU_TANH
    rms_eps: float = 1e-6

    def with_(self, **kw) -> "MoeConfig":
        return replace(self, **kw)


# Workload presets (synthetic inputs; recipes in the generator module).
TINY = MoeConfig(H=256, E=16, k=2, I=128, Is=256)          # one layer, 1 token
LAYER = MoeConfig()                                         # one layer, batch 1
STACK_LAYERS = 30                                           # stack depth
STACK_TOKENS = 256                                          # tokens decoded
STREAM_TOKENS = 512                                         # streaming run
BATCH_SWEEP = (1, 8, 32, 64, 128, 256)                      # batched decode
ROUTER_BIAS_STD = 1.5                                       # skewed popularity
WEIGHT_STD = 0.02                                           # pre-quantisation
