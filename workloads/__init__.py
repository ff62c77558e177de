"""Seeded synthetic inputs and layer shapes for the dequant-matmul workloads.

This module holds no arithmetic of the method: it only draws the seeded
random tensors that the CUDA path and the oracle both consume, and lists the
linear-layer shapes of the models the pages run (Qwen2.5-0.5B on Enargeia,
Qwen3-0.6B on BITCRUSH BC-06, Qwen3-8B on Trellis-WebGPU).

Recipe (stated once, used everywhere):
  * weights W[N][K] (PyTorch Linear layout, N = out features, K = in
    features): fp32 standard normal * sigma, rounded to fp16 (RNE);
    sigma = 0.02 (0.015 for the Qwen3-8B set);
  * activations x[M][K]: fp32 standard normal; for the prefill workloads
    the same draw rounded to bf16 (RNE);
  * every tensor has its own stream: numpy PCG64 seeded with
    SeedSequence([workload, layer, matrix, tag]); workload i uses seed i;
  * within a layer, q/k/v share one activation (x_attn), gate/up share
    x_mlp, o and down get their own.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import numpy as np

# (name, in_features K, out_features N) per decoder layer.
SHAPE_SETS: Dict[str, List[Tuple[str, int, int]]] = {
    # Qwen2.5-0.5B, hidden 896 (Enargeia page)
    "qwen2.5-0.5b": [("q", 896, 896), ("k", 896, 128), ("v", 896, 128),
                     ("o", 896, 896), ("gate", 896, 4864), ("up", 896, 4864),
                     ("down", 4864, 896)],
    # Qwen3-0.6B, hidden 1024 (BITCRUSH BC-06 page)
    "qwen3-0.6b": [("q", 1024, 2048), ("k", 1024, 1024), ("v", 1024, 1024),
                   ("o", 2048, 1024), ("gate", 1024, 3072), ("up", 1024, 3072),
                   ("down", 3072, 1024)],
    # Qwen3-8B, hidden 4096 (Trellis-WebGPU page)
    "qwen3-8b": [("q", 4096, 4096), ("k", 4096, 1024), ("v", 4096, 1024),
                 ("o", 4096, 4096), ("gate", 4096, 12288), ("up", 4096, 12288),
                 ("down", 12288, 4096)],
}
# Single-matrix sets: the 1024 x 1024 single layer (BITCRUSH BC-06's lever
# on one matrix) and Qwen3-0.6B's tied LM head (1024 -> vocabulary).
SHAPE_SETS["single-1024"] = [("single", 1024, 1024)]
SHAPE_SETS["qwen3-0.6b-lmhead"] = [("lm_head", 1024, 151936)]
LAYERS = {"qwen2.5-0.5b": 24, "qwen3-0.6b": 28, "qwen3-8b": 36,
          "single-1024": 1, "qwen3-0.6b-lmhead": 1}
SIGMA = {"qwen2.5-0.5b": 0.02, "qwen3-0.6b": 0.02, "qwen3-8b": 0.015,
         "single-1024": 0.02, "qwen3-0.6b-lmhead": 0.02}
# Which activation each matrix reads inside a layer.
X_TAG = {"q": "x_attn", "k": "x_attn", "v": "x_attn", "o": "x_o",
         "gate": "x_mlp", "up": "x_mlp", "down": "x_down", "single": "x",
         "lm_head": "x"}
_MAT_ID = {"q": 0, "k": 1, "v": 2, "o": 3, "gate": 4, "up": 5, "down": 6,
           "lm_head": 7, "single": 8}
_TAG_ID = {"W": 0, "x_attn": 1, "x_o": 2, "x_mlp": 3, "x_down": 4, "x": 5}

# Architecture facts used only by the byte ledger (tied embeddings, norms,
# biases) of the two small models.
VOCAB = 151936
LM_HEAD_QWEN3_06B = ("lm_head", 1024, VOCAB)


def _rng(workload: int, layer: int, mat: str, tag: str) -> np.random.Generator:
    ss = np.random.SeedSequence([int(workload), int(layer), _MAT_ID[mat],
                                 _TAG_ID[tag]])
    return np.random.Generator(np.random.PCG64(ss))


def weight(workload: int, layer: int, mat: str, K: int, N: int,
           sigma: float) -> np.ndarray:
    """fp16 W[N][K] ~ N(0, sigma^2)."""
    g = _rng(workload, layer, mat, "W")
    w = g.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(sigma)
    return w.astype(np.float16)


def activation(workload: int, layer: int, tag: str, M: int, K: int) -> np.ndarray:
    """fp32 x[M][K] ~ N(0, 1)."""
    g = _rng(workload, layer, "single", tag)
    return g.standard_normal((M, K), dtype=np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (RNE); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return r


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Matrix:
    layer: int
    name: str
    K: int
    N: int
    x_tag: str


def layer_set(shape_set: str, layers: int | None = None) -> List[Matrix]:
    """The matrices of `layers` decoder layers, in execution order."""
    n = LAYERS[shape_set] if layers is None else layers
    out = []
    for l in range(n):
        for name, K, N in SHAPE_SETS[shape_set]:
            out.append(Matrix(l, name, K, N, X_TAG[name]))
    return out


# ---- byte ledger (BRAIN SIZE on BITCRUSH BC-06; residency on Enargeia) ---

def linear_params(shape_set: str) -> int:
    per_layer = sum(K * N for _, K, N in SHAPE_SETS[shape_set])
    return per_layer * LAYERS[shape_set]


def other_params(shape_set: str) -> int:
    """Tied embedding + norms (+ q/k/v biases for Qwen2.5)."""
    if shape_set == "qwen3-0.6b":
        h, L = 1024, 28
        norms = L * (2 * h + 2 * 128) + h      # input/post norms + q/k norm
        return VOCAB * h + norms
    if shape_set == "qwen2.5-0.5b":
        h, L = 896, 24
        norms = L * 2 * h + h
        biases = L * (896 + 128 + 128)
        return VOCAB * h + norms + biases
    raise KeyError(shape_set)


def model_bytes(shape_set: str, bits: int) -> int:
    """Bytes of weights when the linear layers are held at `bits` bits per
    weight (code bits only) and everything else stays fp16."""
    lin = linear_params(shape_set)
    if bits == 16:
        return (lin + other_params(shape_set)) * 2
    return lin * bits // 8 + other_params(shape_set) * 2


# ---- per-matrix algorithmic bytes / flops (roofline accounting) ---------

def gemv_bytes(K: int, N: int, M: int, mode: str, bits: int, group: int,
               x_bytes_per_elem: int = 4) -> int:
    """Algorithmic bytes of one matmul: weights (codes or fp16), scale/zero,
    x and y.  Runtime mode reads fp16 W whatever the bits, with fp32 scale
    and zero per group ("range": one fp16 (min, max) word per group); packed
    mode reads int4 codes and fp16 scale/zero per 64-block."""
    if mode == "packed":
        w = N * K // 2 + N * (K // 64) * 2 * 2
    elif bits == 16:
        w = N * K * 2
    elif mode == "range":      # one 4-byte (min, max) word per group
        w = N * K * 2 + N * (K // group) * 4
    else:
        w = N * K * 2 + N * (K // group) * 4 * 2
    return w + M * K * x_bytes_per_elem + M * N * 4
