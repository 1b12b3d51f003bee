"""Seeded bf16 tensors.

Every tensor is drawn from numpy's Philox4x32 counter-based generator (Salmon
et al., "Parallel random numbers: as easy as 1, 2, 3", SC'11), keyed by
(seed, tensor id), so a tensor's bits depend only on its seed and name.  The
normal deviates are scaled in float32 and rounded to bfloat16 with
round-to-nearest-even.  bf16 values are carried as uint16 bit patterns.
"""

from __future__ import annotations

import numpy as np

from .presets import ModelDims

WEIGHT_STD = 0.02
GAIN_STD = 0.02

# Per weight set: s in ("R", "G") = Reasoner (AR tokens), Generator (DM tokens).
_SET_TENSORS = ("g1", "wqkv", "wo", "g2", "wg", "wu", "wd")
WEIGHT_NAMES = tuple(f"{s}.{t}" for s in ("R", "G") for t in _SET_TENSORS) + ("gfin", "wvel")


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_to_f32(b).astype(np.float64)


def _gen(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=(int(seed) << 32) | int(tensor_id)))


def normal_bf16(shape, seed: int, tensor_id: int, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    """bf16 bits of mean + std * N(0, 1), drawn from Philox(seed, tensor_id)."""
    g = _gen(seed, tensor_id)
    z = g.standard_normal(int(np.prod(shape)), dtype=np.float32)
    if std != 1.0:
        z *= np.float32(std)
    if mean != 0.0:
        z += np.float32(mean)
    return bf16_round(z).reshape(shape)


def weight_shapes(dims: ModelDims) -> dict:
    d, f = dims.d_model, dims.ffn
    per_set = {
        "g1": (d,),
        "wqkv": (dims.qkv_cols, d),  # rows: Q heads, then K heads, then V heads
        "wo": (d, dims.q_cols),
        "g2": (d,),
        "wg": (f, d),
        "wu": (f, d),
        "wd": (d, f),
    }
    shapes = {f"{s}.{t}": shp for s in ("R", "G") for t, shp in per_set.items()}
    shapes["gfin"] = (d,)
    shapes["wvel"] = (d, d)  # velocity head: latent width = d_model
    return shapes


def make_weights(dims: ModelDims, seed: int, names=None) -> dict:
    """Both weight sets plus the final DM norm gain and the velocity head.

    Linear weights ~ N(0, 0.02); norm gains ~ 1 + N(0, 0.02).  All row-major
    [out_features, in_features] bf16 bits.
    """
    shapes = weight_shapes(dims)
    out = {}
    for tid, name in enumerate(WEIGHT_NAMES):
        if names is not None and name not in names:
            continue
        shp = shapes[name]
        if name.endswith(("g1", "g2", "gfin")):
            out[name] = normal_bf16(shp, seed, tid, std=GAIN_STD, mean=1.0)
        else:
            out[name] = normal_bf16(shp, seed, tid, std=WEIGHT_STD)
    return out


def stack_layer_seed(seed: int, layer: int) -> int:
    """Seed of layer `layer` of a stack whose first layer has `seed`."""
    return seed + 7919 * layer


def make_stack_weights(dims: ModelDims, seed: int, n_layers: int, distinct: int = 0) -> list:
    """Weights of an n_layers stack, one make_weights draw per layer.

    With distinct > 0 only that many layers are drawn and layer l uses draw
    l % distinct (large stacks whose weights take long to generate on the host;
    every layer's weights still stream from HBM, as each is far larger than L2).
    """
    n_draw = n_layers if distinct <= 0 else min(distinct, n_layers)
    draws = [make_weights(dims, stack_layer_seed(seed, l)) for l in range(n_draw)]
    return [draws[l % n_draw] for l in range(n_layers)]


def make_action_weights(d_model: int, action_dim: int, seed: int) -> tuple:
    """Domain action projections: W_in [d_model, action_dim] and W_out
    [action_dim, d_model], both ~ N(0, 0.02) bf16 bits."""
    return (normal_bf16((d_model, action_dim), seed, 20_000, std=WEIGHT_STD),
            normal_bf16((action_dim, d_model), seed, 20_001, std=WEIGHT_STD))


def make_actions(n_rows: int, action_dim: int, seed: int, tensor_id: int = 0) -> np.ndarray:
    """Normalised action state [n_rows, action_dim] ~ N(0, 1) bf16 bits."""
    return normal_bf16((n_rows, action_dim), seed, 30_000 + tensor_id)


def make_activations(n_tokens: int, d_model: int, seed: int, tensor_id: int = 0) -> np.ndarray:
    """Layer input h [n_tokens, d_model] ~ N(0, 1) bf16 bits."""
    return normal_bf16((n_tokens, d_model), seed, 10_000 + tensor_id)
