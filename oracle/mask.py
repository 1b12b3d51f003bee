"""The hybrid MoT attention mask, fp64 oracle.

TEST INFRASTRUCTURE (see the package docstring).

"Cosmos 3 方法原理全解" §3 gives the two attention equations
    O_AR = Attn_causal(Q_AR, K_AR, V_AR)
    O_DM = Attn_full(Q_DM, [K_AR; K_DM], [V_AR; V_DM])
so AR rows never read DM keys and DM attention is bidirectional.  The
streaming models ("NVIDIA 发布 Cosmos 3 系列四个开放权重世界模型",
"流式生成如何工作") use time-causal attention: a block reads the history and
the controls but not future targets.

Reading taken where the pages leave details open: key j is visible to query i iff
  * i is AR:  j is AR and j <= i;
  * i is DM, FULL mode:          every AR key and every DM key;
  * i is DM, BLOCK_CAUSAL mode:  every AR key, and DM keys with
                                 chunk(j) <= chunk(i) (full inside a chunk).
Rows of different batch elements never mix.
"""

from __future__ import annotations

import numpy as np

from .layout import REGION_AR

FULL, BLOCK_CAUSAL = "full", "block_causal"


def allow_matrix(q_rows, region, chunk, mode: str, k_rows=None) -> np.ndarray:
    """Boolean [len(q_rows), len(k_rows)] visibility matrix (vectorised form).

    `region` and `chunk` describe the key sequence; queries are rows of it.
    """
    if mode not in (FULL, BLOCK_CAUSAL):
        raise ValueError(mode)
    region = np.asarray(region)
    chunk = np.asarray(chunk)
    q_rows = np.asarray(q_rows, dtype=np.int64)
    k_rows = np.arange(len(region), dtype=np.int64) if k_rows is None else np.asarray(k_rows, np.int64)
    q_ar = (region[q_rows] == REGION_AR)[:, None]
    k_ar = (region[k_rows] == REGION_AR)[None, :]
    causal = k_rows[None, :] <= q_rows[:, None]
    ar_part = q_ar & k_ar & causal
    if mode == FULL:
        dm_keys = np.ones((1, len(k_rows)), dtype=bool)
    else:
        dm_keys = k_ar | (chunk[k_rows][None, :] <= chunk[q_rows][:, None])
    return ar_part | (~q_ar & dm_keys)


def allow_matrix_from_equations(region, chunk, mode: str) -> np.ndarray:
    """Second construction, row by row from the two §3 equations (tiny inputs only).

    For an AR query the key list is the AR prefix up to and including itself;
    for a DM query it is [K_AR; K_DM], with future chunks removed in
    block-causal mode.
    """
    n = len(region)
    ar_idx = [j for j in range(n) if region[j] == REGION_AR]
    dm_idx = [j for j in range(n) if region[j] != REGION_AR]
    m = np.zeros((n, n), dtype=bool)
    for i in range(n):
        if region[i] == REGION_AR:
            keys = [j for j in ar_idx if j <= i]
        else:
            keys = list(ar_idx)
            if mode == FULL:
                keys += dm_idx
            else:
                keys += [j for j in dm_idx if chunk[j] <= chunk[i]]
        for j in keys:
            m[i, j] = True
    return m
