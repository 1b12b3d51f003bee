"""Unified 3D rotary position embedding (mRoPE), fp64 oracle.

TEST INFRASTRUCTURE (see the package docstring).

"Cosmos 3 方法原理全解" §5 and the NVIDIA/cosmos README (model architecture)
say every token carries a (t, h, w) coordinate and that text, with
t = h = w, reduces to ordinary 1D RoPE.  The pages give neither the base, the
pairing, nor how the frequency pairs are split between the three axes.
Readings where the pages are silent:
  * base 10000, inv_freq_i = base^(-2i/head_dim) for pair i in [0, head_dim/2);
  * rotate-half pairing: element i is paired with element i + head_dim/2;
  * the pairs are cut into three contiguous sections (n_t, n_h, n_w) with
    n_t + n_h + n_w = head_dim/2; pairs in a section take their angle from
    that axis' coordinate (8:12:12 at head_dim 64 as the tiny workload states;
    16:24:24 at head_dim 128, the same 1/4 : 3/8 : 3/8 ratio).
"""

from __future__ import annotations

import numpy as np


def inv_freq(head_dim: int, base: float) -> np.ndarray:
    i = np.arange(head_dim // 2, dtype=np.float64)
    return base ** (-2.0 * i / head_dim)


def pair_axis(head_dim: int, sections) -> np.ndarray:
    n_t, n_h, n_w = sections
    if n_t + n_h + n_w != head_dim // 2:
        raise ValueError("mRoPE sections must cover head_dim/2 frequency pairs")
    return np.concatenate([np.zeros(n_t, np.int64), np.ones(n_h, np.int64), np.full(n_w, 2, np.int64)])


def angles(pos, head_dim: int, sections, base: float) -> np.ndarray:
    """theta[r, i] = pos[r, axis(i)] * inv_freq_i, in float64, shape [N, head_dim/2]."""
    pos = np.asarray(pos, dtype=np.float64)
    ax = pair_axis(head_dim, sections)
    return pos[:, ax] * inv_freq(head_dim, base)[None, :]


def apply(x, pos, head_dim: int, sections, base: float) -> np.ndarray:
    """Rotate x[..., N, n_heads, head_dim] by the mRoPE angles of each row.

    For pair (i, i + head_dim/2):  x_i' = x_i cos - x_{i+hd/2} sin,
                                   x_{i+hd/2}' = x_{i+hd/2} cos + x_i sin.
    """
    x = np.asarray(x, dtype=np.float64)
    th = angles(pos, head_dim, sections, base)          # [N, hd/2]
    c = np.cos(th)[:, None, :]
    s = np.sin(th)[:, None, :]
    half = head_dim // 2
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)
