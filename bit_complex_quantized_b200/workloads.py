"""Seeded synthetic workloads: shapes, distributions and seeds of the five
benchmark workloads.  Random numbers only -- none of the method's
arithmetic lives here; the CUDA path and the oracle both take these arrays as
inputs.

Weights: float32, iid N(0, sigma) per real entry (per Re and Im plane for the
complex layers), drawn with numpy's default_rng seeded by [seed, 0, layer].
Activations: float32 N(0, 1) drawn with default_rng([seed, 1, layer, rows]),
real plane then imaginary plane, rounded to bf16 (nearest-even) by torch.
"""
from dataclasses import dataclass, field
from typing import List, Tuple

import numpy as np
import torch


@dataclass
class LayerSpec:
    name: str
    kind: str               # "complex": N x K complex weights given directly;
                            # "real": a real (2N) x (2K) layer converted to U, W
    N: int                  # complex outputs
    K: int                  # complex inputs
    sigma: float

    @property
    def real_shape(self) -> Tuple[int, int]:
        return (2 * self.N, 2 * self.K)


@dataclass
class Config:
    name: str
    seed: int
    T: int
    conj: bool              # widely-linear (U and W) vs plain complex (U only)
    batches: List[int]
    layers: List[LayerSpec] = field(default_factory=list)
    prefill_M: int = 0


def _block(prefix_sigma, hidden_real, ffn_real, kind):
    """Attention q,k,v,o and MLP gate, up, down of one transformer block.
    For kind == "real" the sizes are of the real layer (converted to complex N = out/2, K = in/2)."""
    s = prefix_sigma
    h = hidden_real // 2 if kind == "real" else hidden_real
    f = ffn_real // 2 if kind == "real" else ffn_real
    return [LayerSpec("q", kind, h, h, s), LayerSpec("k", kind, h, h, s), LayerSpec("v", kind, h, h, s),
            LayerSpec("o", kind, h, h, s), LayerSpec("gate", kind, f, h, s), LayerSpec("up", kind, f, h, s),
            LayerSpec("down", kind, h, f, s)]


def config(name: str) -> Config:
    """The five workloads, by name:
    layer256         one complex layer, 256 x 256, 1 stage, no conjugate branch
    block1024        plain complex transformer block, hidden 1024, FFN 2816, 1 stage
    llama7b          LLaMA-2-7B-shaped real block -> (U, W), 2 stages
    llama7b_prefill  prefill on the llama7b matrices, M = 2048 tokens
    llama70b         LLaMA-2-70B-shaped layer set -> (U, W), 3 stages
    """
    if name == "layer256":
        return Config("layer256", 0, 1, False, [1], [LayerSpec("w", "complex", 256, 256, 0.02)], prefill_M=0)
    if name == "block1024":
        return Config("block1024", 1, 1, False, [1, 8], _block(0.02, 1024, 2816, "complex"), prefill_M=0)
    if name == "llama7b":
        return Config("llama7b", 2, 2, True, [1, 16], _block(0.02, 4096, 11008, "real"), prefill_M=2048)
    if name == "llama7b_prefill":   # the llama7b weights; activation seed 3
        c = config("llama7b")
        return Config("llama7b_prefill", 3, 2, True, [], c.layers, prefill_M=2048)
    if name == "llama70b":   # k, v: 8192 in -> 1024 out
        s = 0.015
        L = [LayerSpec("q", "real", 4096, 4096, s), LayerSpec("k", "real", 512, 4096, s),
             LayerSpec("v", "real", 512, 4096, s), LayerSpec("o", "real", 4096, 4096, s),
             LayerSpec("gate", "real", 14336, 4096, s), LayerSpec("up", "real", 14336, 4096, s),
             LayerSpec("down", "real", 4096, 14336, s)]
        return Config("llama70b", 4, 3, True, [1, 8], L, prefill_M=0)
    raise KeyError(name)


def weight_seed(cfg: Config, layer: int):
    # the prefill workload shares the llama7b weights
    return [config("llama7b").seed if cfg.name == "llama7b_prefill" else cfg.seed, 0, layer]


def complex_weights(cfg: Config, layer: int, rows=None):
    """(w_re, w_im) float32 [N][K] for a "complex" layer (optionally a row range)."""
    spec = cfg.layers[layer]
    assert spec.kind == "complex"
    rng = np.random.default_rng(weight_seed(cfg, layer))
    w_re = (np.float32(spec.sigma) * rng.standard_normal((spec.N, spec.K), dtype=np.float32))
    w_im = (np.float32(spec.sigma) * rng.standard_normal((spec.N, spec.K), dtype=np.float32))
    return w_re, w_im


def real_weight(cfg: Config, layer: int):
    """R float32 [2N][2K] for a "real" layer."""
    spec = cfg.layers[layer]
    assert spec.kind == "real"
    rng = np.random.default_rng(weight_seed(cfg, layer))
    return np.float32(spec.sigma) * rng.standard_normal(spec.real_shape, dtype=np.float32)


def activations(cfg: Config, layer: int, rows: int):
    """(x_re, x_im) as torch bf16 CPU tensors [rows][K]."""
    spec = cfg.layers[layer]
    rng = np.random.default_rng([cfg.seed, 1, layer, rows])
    x_re = torch.from_numpy(rng.standard_normal((rows, spec.K), dtype=np.float32)).to(torch.bfloat16)
    x_im = torch.from_numpy(rng.standard_normal((rows, spec.K), dtype=np.float32)).to(torch.bfloat16)
    return x_re, x_im


def bf16_to_f32_numpy(x: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 tensor for the oracle."""
    return x.to(torch.float32).cpu().numpy()


def code_bytes(cfg: Config) -> int:
    """Packed code bytes of all layers: 2 bits per complex weight per stage per branch."""
    nb = 2 if cfg.conj else 1
    return sum(nb * cfg.T * l.N * l.K // 4 for l in cfg.layers)
