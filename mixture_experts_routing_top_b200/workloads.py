"""The five synthetic MoE-layer workloads and their seeded input recipes.

Shapes, distributions and structure follow the workloads this library is
measured on: a tiny fp32 layer, a Mixtral-shaped top-2 layer with skewed
expert load, a fine-grained top-6 layer with clustered (correlated) routing
and a shared expert, a dispatch/combine bandwidth sweep with group-major
layouts, and an expert-choice layer with two correlated routing layers.

Every tensor has its own generator stream (``synth``), seed 0.  Logits are
always fp32 (the router's precision); activations and weights are fp32 in
the tiny layer and bf16 elsewhere.  Nothing here computes any part of the
MoE layer: the recipes only shape random numbers.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import numpy as np

from . import synth

# generator stream ids, one per tensor
S_LOGITS, S_X, S_W1, S_W3, S_W2, S_BIAS, S_CLUSTER = 1, 2, 3, 4, 5, 6, 7
S_SW1, S_SW3, S_SW2, S_P, S_NOISE2, S_WR = 8, 9, 10, 11, 12, 13


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int = 0                      # top-k (0 for expert choice)
    F: int = 0                      # expert FFN width (0: identity experts)
    capacity_factor: float = 0.0    # <= 0: unbounded (no dropping)
    dtype: str = "bf16"             # activation / weight dtype: "f32" or "bf16"
    act: str = "swiglu"             # "swiglu" or "gelu"
    routing: str = "topk"           # "topk" or "ec"
    norm_topk: bool = False         # renormalise gates over the chosen k
    F_shared: int = 0               # shared expert width (0: none)
    C: int = 0                      # expert-choice tokens per expert
    G: int = 0                      # group-major layout with G equal groups (0: expert-major)
    logit_bias_std: float = 0.0     # per-expert logit bias ~ N(0, std^2)
    cluster_bias: float = 0.0       # clustered routing: bias added to the token's cluster
    n_clusters: int = 0
    transition_mix: float = 0.0     # layer-2 logits = mix * P[top1 of layer 1] + N(0, 1)
    w_std: float = 0.02
    router: int = 0                 # 1: logits = x W_r^T on the device (the router's linear gate)
    seed: int = 0

    @property
    def capacity(self) -> Optional[int]:
        """Per-expert capacity ceil(cf * T * k / E); None when unbounded."""
        if self.capacity_factor <= 0 or self.routing != "topk":
            return None
        return int(math.ceil(self.capacity_factor * self.T * self.k / self.E))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


TINY = Workload("tiny_fp32", T=256, d=64, E=8, k=2, F=128, capacity_factor=1.25, dtype="f32")
MIXTRAL = Workload("mixtral_top2_bf16", T=8192, d=4096, E=8, k=2, F=14336, capacity_factor=1.25,
                   logit_bias_std=0.5)
FINE = Workload("fine_top6_shared_bf16", T=16384, d=2048, E=64, k=6, F=1408, capacity_factor=1.5,
                F_shared=2816, cluster_bias=2.0, n_clusters=16)
SWEEP_T = (4096, 16384, 65536, 131072)
SWEEP_G = (8, 32, 64)
SWEEP = Workload("dispatch_combine_sweep_bf16", T=131072, d=7168, E=256, k=8, F=0,
                 capacity_factor=0.0, norm_topk=True, G=8)
EXPERT_CHOICE = Workload("expert_choice_gelu_bf16", T=32768, d=1024, E=128, F=4096, act="gelu",
                         routing="ec", C=512, transition_mix=0.7)

ALL = (TINY, MIXTRAL, FINE, SWEEP, EXPERT_CHOICE)
BY_NAME = {w.name: w for w in ALL}


def _normal(w: Workload, stream: int, shape, std=1.0, bf16=None) -> np.ndarray:
    bf16 = (w.dtype == "bf16") if bf16 is None else bf16
    if bf16:
        return synth.normal_bf16(w.seed, stream, shape, 0.0, std)
    return synth.normal_f32(w.seed, stream, shape, 0.0, std)


def make_logits(w: Workload) -> np.ndarray:
    """Router logits [T, E] fp32 (layer 1 for the expert-choice workload)."""
    lg = synth.normal_f32(w.seed, S_LOGITS, (w.T, w.E))
    if w.logit_bias_std > 0:
        bias = synth.normal_f32(w.seed, S_BIAS, (w.E,), 0.0, w.logit_bias_std)
        lg = (lg + bias[None, :]).astype(np.float32)
    if w.cluster_bias != 0.0:
        per = w.E // w.n_clusters
        cl = (synth.u64(w.seed, S_CLUSTER, w.T) % np.uint64(w.n_clusters)).astype(np.int64)
        cols = cl[:, None] * per + np.arange(per)[None, :]
        rows = np.arange(w.T)[:, None]
        lg[rows, cols] = (lg[rows, cols] + np.float32(w.cluster_bias)).astype(np.float32)
    return lg


def token_clusters(w: Workload) -> np.ndarray:
    """The cluster each token drew (clustered-routing workload)."""
    return (synth.u64(w.seed, S_CLUSTER, w.T) % np.uint64(w.n_clusters)).astype(np.int64)


def make_layer2_logits(w: Workload, logits1: np.ndarray) -> np.ndarray:
    """Next layer's logits: mix * P[a_t, :] + N(0, 1), a_t = the token's top-1
    expert at layer 1 (lowest index among equal maxima), P a fixed seeded
    E x E Gaussian matrix; fp32 multiply then fp32 add, no fused multiply-add."""
    P = synth.normal_f32(w.seed, S_P, (w.E, w.E))
    noise = synth.normal_f32(w.seed, S_NOISE2, (w.T, w.E))
    a = np.argmax(logits1, axis=1)
    scaled = (np.float32(w.transition_mix) * P[a]).astype(np.float32)
    return (scaled + noise).astype(np.float32)


def make_x(w: Workload) -> np.ndarray:
    """Token activations [T, d] (fp32, or bf16 bit patterns)."""
    return _normal(w, S_X, (w.T, w.d))


def make_weights(w: Workload) -> Tuple[np.ndarray, Optional[np.ndarray], np.ndarray]:
    """Routed expert weights W1 [E, F, d], W3 [E, F, d] (None for GELU), W2 [E, d, F]."""
    W1 = _normal(w, S_W1, (w.E, w.F, w.d), w.w_std)
    W3 = _normal(w, S_W3, (w.E, w.F, w.d), w.w_std) if w.act == "swiglu" else None
    W2 = _normal(w, S_W2, (w.E, w.d, w.F), w.w_std)
    return W1, W3, W2


def make_router_weights(w: Workload) -> np.ndarray:
    """Router linear gate W_r [E, d], N(0, 1/d): with x ~ N(0, 1) the logits
    are about N(0, 1), the spread of the handed-in logits."""
    return _normal(w, S_WR, (w.E, w.d), std=1.0 / math.sqrt(w.d))


def make_shared_weights(w: Workload):
    """Shared expert weights (one SwiGLU expert of width F_shared), or None."""
    if w.F_shared <= 0:
        return None
    W1 = _normal(w, S_SW1, (1, w.F_shared, w.d), w.w_std)
    W3 = _normal(w, S_SW3, (1, w.F_shared, w.d), w.w_std)
    W2 = _normal(w, S_SW2, (1, w.d, w.F_shared), w.w_std)
    return W1, W3, W2


def equal_groups(E: int, G: int) -> np.ndarray:
    """group_of_expert for G equal contiguous groups: expert e -> e // (E / G)."""
    assert E % G == 0
    return (np.arange(E, dtype=np.int32) // (E // G)).astype(np.int32)
