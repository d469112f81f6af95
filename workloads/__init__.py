"""Seeded synthetic inputs for the DeepSeekMoE layer forward.

This module is shared by the CPU oracle (``oracle/``) and by the GPU path's
tests and benchmark.  It draws random numbers and rounds them to bf16; it
holds none of the layer's arithmetic (no router, no gate, no FFN, no sum).

Layer shapes
------------
The five shapes below are the synthetic stand-ins for the models the
DeepSeekMoE pages discuss:

* ``tiny``        -- a small layer the oracle finishes in well under a second.
* ``2b``          -- the DeepSeekMoE 2B layer: 63 routed experts plus 1 shared
                     expert, 7 routed experts active per token (DeepSeekMoE
                     blog summary, "DeepSeekMoE 2B Model Example").
* ``16b_prefill`` -- the DeepSeekMoE 16B layer: hidden size 2048, 64 routed
                     plus 2 shared experts, 6 routed active (DeepSeekMoE blog
                     summary, "Scaling Up to DeepSeekMoE 16B").
* ``16b_decode``  -- the same layer with 32 tokens (weight-streaming regime).
* ``v3``          -- the DeepSeek-V3 layer: 256 routed experts, 8 active,
                     sigmoid affinities with a selection bias (DeepSeek-V3
                     technical report summary, section 4 "Model Architecture"
                     and section 2 "Auxiliary-Loss-Free Load Balancing").

Intermediate sizes, d_model of the small layers, the value distributions and
the bias recipes are not printed on the pages; they are fixed here.

Generator
---------
Every tensor is drawn from numpy's PCG64 seeded with
``SeedSequence([seed, tensor_id, sub])`` (``sub`` = expert index for expert
weights, 0 otherwise), as standard normals in float32, scaled by sigma in
float32 and rounded to bf16 with round-to-nearest-even.  Because every
expert has its own stream, any single expert's weights can be regenerated
without generating the others.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np
import torch

# tensor ids (the stream id of each input tensor)
TID_X, TID_ROUTER, TID_BIAS = 0, 1, 2
TID_W_GATE, TID_W_UP, TID_W_DOWN = 3, 4, 5
TID_WS_GATE, TID_WS_UP, TID_WS_DOWN = 6, 7, 8
TID_SAMPLE = 9
TID_DH = 10


@dataclass(frozen=True)
class LayerShape:
    """Sizes and input recipe of one DeepSeekMoE layer.

    T tokens, d = d_model, N = mN routed experts of intermediate I, K = mK
    routed experts active per token, Ks shared experts of intermediate Is.
    ``gate`` is "softmax" or "sigmoid"; ``bias`` names the bias recipe:
    "none", "normal" (logit bias ~ N(0, 0.5)), "zipf" (logit bias
    -1.1*ln(i+1)) or "uniform" (selection bias ~ U(-0.1, 0.1)).
    """

    name: str
    T: int
    d: int
    N: int
    I: int
    K: int
    Ks: int
    Is: int
    gate: str = "softmax"
    sigma: float = 0.02
    bias: str = "none"
    seed: int = 0

    def with_(self, **kw) -> "LayerShape":
        return replace(self, **kw)

    @property
    def routed_flop(self) -> float:
        """Algorithmic FLOPs of the routed experts: 3 GEMMs of 2*d*I per (token, expert)."""
        return 6.0 * self.T * self.K * self.d * self.I

    @property
    def shared_flop(self) -> float:
        return 6.0 * self.T * self.Ks * self.d * self.Is

    @property
    def router_flop(self) -> float:
        return 2.0 * self.T * self.d * self.N


CONFIGS = {
    "tiny": LayerShape("tiny", T=512, d=256, N=16, I=128, K=4, Ks=1, Is=128,
                       gate="softmax", sigma=0.02, bias="none", seed=1000),
    "2b": LayerShape("2b", T=8192, d=1280, N=63, I=896, K=7, Ks=1, Is=896,
                     gate="softmax", sigma=0.02, bias="normal", seed=2000),
    "16b_prefill": LayerShape("16b_prefill", T=16384, d=2048, N=64, I=1408, K=6,
                              Ks=2, Is=1408, gate="softmax", sigma=0.02,
                              bias="none", seed=3000),
    "16b_decode": LayerShape("16b_decode", T=32, d=2048, N=64, I=1408, K=6,
                             Ks=2, Is=1408, gate="softmax", sigma=0.02,
                             bias="zipf", seed=4000),
    "v3": LayerShape("v3", T=4096, d=7168, N=256, I=2048, K=8, Ks=1, Is=2048,
                     gate="sigmoid", sigma=0.006, bias="uniform", seed=5000),
}


def _rng(seed: int, tensor_id: int, sub: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id, sub])))


def to_bf16(a_f32: np.ndarray) -> torch.Tensor:
    """Round a float32 array to bf16 (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(a_f32, dtype=np.float32)).to(torch.bfloat16)


def normal_bf16(seed: int, tensor_id: int, sub: int, shape, sigma: float) -> torch.Tensor:
    n = int(np.prod(shape))
    a = _rng(seed, tensor_id, sub).standard_normal(n, dtype=np.float32)
    if sigma != 1.0:
        a *= np.float32(sigma)
    return to_bf16(a.reshape(shape))


def tokens(shape: LayerShape) -> torch.Tensor:
    """u: bf16 [T, d], entries ~ N(0, 1)."""
    return normal_bf16(shape.seed, TID_X, 0, (shape.T, shape.d), 1.0)


def output_gradient(shape: LayerShape, scale: float = 1.0) -> torch.Tensor:
    """dh: bf16 [T, d], the upstream gradient of the layer's output for the backward, ~ N(0, scale)."""
    return normal_bf16(shape.seed, TID_DH, 0, (shape.T, shape.d), scale)


def router_weight(shape: LayerShape) -> torch.Tensor:
    """e: bf16 [N, d], the per-expert affinity vectors, entries ~ N(0, sigma)."""
    return normal_bf16(shape.seed, TID_ROUTER, 0, (shape.N, shape.d), shape.sigma)


def router_bias(shape: LayerShape):
    """Return (logit_bias, select_bias), each float32 [N] or None."""
    N = shape.N
    if shape.bias == "none":
        return None, None
    if shape.bias == "normal":
        c = _rng(shape.seed, TID_BIAS).standard_normal(N) * 0.5
        return torch.from_numpy(c.astype(np.float32)), None
    if shape.bias == "zipf":
        c = np.array([-1.1 * math.log(i + 1) for i in range(N)], dtype=np.float64)
        return torch.from_numpy(c.astype(np.float32)), None
    if shape.bias == "uniform":
        b = _rng(shape.seed, TID_BIAS).uniform(-0.1, 0.1, N)
        return None, torch.from_numpy(b.astype(np.float32))
    raise ValueError(f"unknown bias recipe {shape.bias!r}")


def expert_weights(shape: LayerShape, e: int):
    """Routed expert e: (W_gate [I, d], W_up [I, d], W_down [d, I]) in bf16."""
    s, I, d = shape.seed, shape.I, shape.d
    return (normal_bf16(s, TID_W_GATE, e, (I, d), shape.sigma),
            normal_bf16(s, TID_W_UP, e, (I, d), shape.sigma),
            normal_bf16(s, TID_W_DOWN, e, (d, I), shape.sigma))


def shared_weights(shape: LayerShape, j: int):
    """Shared expert j: (W_gate [Is, d], W_up [Is, d], W_down [d, Is]) in bf16."""
    s, I, d = shape.seed, shape.Is, shape.d
    return (normal_bf16(s, TID_WS_GATE, j, (I, d), shape.sigma),
            normal_bf16(s, TID_WS_UP, j, (I, d), shape.sigma),
            normal_bf16(s, TID_WS_DOWN, j, (d, I), shape.sigma))


def _parallel_map(fn, items, workers=None):
    workers = workers or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=workers) as ex:
        return list(ex.map(fn, items))


def stacked_expert_weights(shape: LayerShape, workers=None):
    """All routed experts stacked: W_gate, W_up bf16 [N, I, d]; W_down bf16 [N, d, I]."""
    parts = _parallel_map(lambda e: expert_weights(shape, e), range(shape.N), workers)
    return (torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]),
            torch.stack([p[2] for p in parts]))


def stacked_shared_weights(shape: LayerShape):
    """All shared experts stacked: bf16 [Ks, Is, d], [Ks, Is, d], [Ks, d, Is] (None if Ks == 0)."""
    if shape.Ks == 0:
        return None, None, None
    parts = [shared_weights(shape, j) for j in range(shape.Ks)]
    return (torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]),
            torch.stack([p[2] for p in parts]))


def layer_inputs(shape: LayerShape, with_experts: bool = True) -> dict:
    """Every input of one layer call as CPU tensors (bf16 / float32).

    With ``with_experts=False`` the routed expert weights are left out; fetch
    them one expert at a time with :func:`expert_weights` (the v3 layer holds
    22.5 GB of them).
    """
    lb, sb = router_bias(shape)
    out = {"x": tokens(shape), "router": router_weight(shape),
           "logit_bias": lb, "select_bias": sb}
    if with_experts:
        out["w_gate"], out["w_up"], out["w_down"] = stacked_expert_weights(shape)
    out["ws_gate"], out["ws_up"], out["ws_down"] = stacked_shared_weights(shape)
    return out


def sample_tokens(shape: LayerShape, count: int) -> np.ndarray:
    """A seeded, sorted sample of ``count`` distinct token indices in [0, T)."""
    count = min(count, shape.T)
    idx = _rng(shape.seed, TID_SAMPLE).choice(shape.T, size=count, replace=False)
    return np.sort(idx).astype(np.int64)
