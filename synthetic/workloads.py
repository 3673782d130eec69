"""The five synthetic workloads of the MoE layer forward, as input recipes.

Each workload names its sizes, seed, and for every input tensor the generator
tensor id, distribution and storage type.  Nothing here computes any part of
the layer; it only says which seeded draws make up the inputs.

Workloads (sizes follow the MoE tutorial's worked setting and the deployment
notes' MCU model):
  tiny     fp32, T=16 d=64 N=4 h=128 top-2 renormalised, all tensors N(0, 0.02^2)
  small    bf16, T=4096 d=512 N=8 h=128 top-2; weights N(0, 0.02^2); router f32;
           inputs N(0,1) then RMS-normalised per row
  decode   q4_0 experts, d=512 N=8 h=128 top-2, T in {1, 8, 32}, 24 layers with
           independent weights; router f32 N(0, 0.02^2); activations fp16 N(0,1)
  mixtral  bf16, T=8192 d=4096 N=8 h=14336 top-2; router bias b_i = -1.2 ln(i+1)
           (Zipf-skewed loads); capacity factor 1.25
  latent   bf16, T=4096 d=4096 -> l=3584, E=896 routed experts of hidden 3072,
           top-16, 2 shared d-wide experts of hidden 3072, soft caps 4 / 25
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import DT_BF16, DT_F16, DT_F32

# generator tensor ids
TID_U, TID_WROUTE, TID_WGATE, TID_WUP, TID_WDOWN = 1, 2, 3, 4, 5
TID_WDP, TID_WUPP = 6, 7
TID_SHARED_BASE = 10  # shared expert j: gate 10+3j, up 11+3j, down 12+3j
DECODE_LAYER_STRIDE = 100  # decode layer l adds 100*l to the weight ids

SIGMA_W = 0.02


@dataclass
class Workload:
    name: str
    T: int
    d: int
    N: int
    k: int
    h: int
    seed: int
    act_dtype: int          # storage type of u / y
    w_dtype: str            # "f32", "bf16", "q4_0"
    renorm: int = 1
    capacity_factor: float = 0.0   # 0 = unlimited
    rms_inputs: bool = False       # u ~ N(0,1) then RMS-normalised per row
    u_sigma: float = 1.0
    zipf_s: float = 0.0            # router bias b_i = -s * ln(i+1) when > 0
    n_layers: int = 1
    # latent-space extension
    latent: int = 0
    n_shared: int = 0
    shared_hidden: int = 0
    beta_gate: float = 0.0
    beta_up: float = 0.0
    expert_sigma: float = 0.0      # sigma of the routed experts' weights (0: SIGMA_W)
    extra: dict = field(default_factory=dict)

    def router_bias(self):
        if self.zipf_s <= 0.0:
            return None
        return np.array([-self.zipf_s * math.log(i + 1.0) for i in range(self.N)],
                        dtype=np.float64).astype(np.float32)

    def capacity(self, T: int | None = None) -> int:
        """ceil(c * k * T / N): the tutorial's capacity with top-k dispatch counts."""
        if self.capacity_factor <= 0.0:
            return 0
        T = self.T if T is None else T
        return int(math.ceil(self.capacity_factor * self.k * T / self.N))

    @property
    def w_sigma(self) -> float:
        return self.expert_sigma if self.expert_sigma > 0.0 else SIGMA_W

    @property
    def expert_in(self) -> int:
        return self.latent if self.latent else self.d


def tiny() -> Workload:
    return Workload("tiny", T=16, d=64, N=4, k=2, h=128, seed=7, act_dtype=DT_F32, w_dtype="f32",
                    u_sigma=SIGMA_W)


def small(T: int = 4096) -> Workload:
    return Workload("small", T=T, d=512, N=8, k=2, h=128, seed=1001, act_dtype=DT_BF16,
                    w_dtype="bf16", rms_inputs=True)


def decode(T: int = 32, n_layers: int = 24) -> Workload:
    return Workload("decode", T=T, d=512, N=8, k=2, h=128, seed=1002, act_dtype=DT_F16,
                    w_dtype="q4_0", n_layers=n_layers)


def mixtral(T: int = 8192) -> Workload:
    return Workload("mixtral", T=T, d=4096, N=8, k=2, h=14336, seed=1003, act_dtype=DT_BF16,
                    w_dtype="bf16", rms_inputs=True, zipf_s=1.2, capacity_factor=1.25)


def latent(T: int = 4096) -> Workload:
    return Workload("latent", T=T, d=4096, N=896, k=16, h=3072, seed=1004, act_dtype=DT_BF16,
                    w_dtype="bf16", rms_inputs=True, latent=3584, n_shared=2, shared_hidden=3072,
                    beta_gate=4.0, beta_up=25.0)


ALL = {"tiny": tiny, "small": small, "decode": decode, "mixtral": mixtral, "latent": latent}


def w_storage(wl: Workload) -> int:
    return {"f32": DT_F32, "bf16": DT_BF16}[wl.w_dtype]


def tid(base: int, layer: int = 0) -> int:
    """Generator id of a weight tensor in decode layer `layer` (0 for single-layer workloads)."""
    return base + DECODE_LAYER_STRIDE * layer


def shared_tids(j: int):
    b = TID_SHARED_BASE + 3 * j
    return b, b + 1, b + 2
