"""Vertical-line identification by accumulated column mass (diagnostic).

Test infrastructure (see the package header): never called by the CUDA path.

Source: HyQuant (Hybrid-Precision Quantization for LLM Attention): the
vertical-line score of a key position is its accumulated column mass (the
attention probability it receives, summed over later queries); the top-rho
fraction of the non-window prefix (5% by default) is kept in full precision.

Reading: the mass is summed over a set of observation queries and over the
q-heads of a GQA group, with an exact softmax over the non-window prefix; the
selection keeps ceil(rho * N) positions, equal masses lowest position first.
Pins (no worked example on the pages): masses sum to the number of queries,
all-zero queries give the uniform mass, a scalar math.exp loop agrees on a tiny
case, planted heavy-hitter positions are recovered, count and tie rules.
"""
from __future__ import annotations

import math

import numpy as np


def column_mass(q_obs, k_prefix, sm_scale: float | None = None) -> np.ndarray:
    """q_obs [Nq, d] (observation queries, all q-heads of the group stacked),
    k_prefix [N, d] -> accumulated probability mass per key [N] (FP64)."""
    q = np.asarray(q_obs, np.float64)
    k = np.asarray(k_prefix, np.float64)
    sm = 1.0 / math.sqrt(k.shape[1]) if sm_scale is None else sm_scale
    s = (q @ k.T) * sm
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p.sum(axis=0)


def select_vertical_lines(q_obs, k_prefix, rho: float = 0.05) -> np.ndarray:
    """Sorted positions of the top ceil(rho * N) keys by column mass (stable on ties)."""
    mass = column_mass(q_obs, k_prefix)
    n = int(math.ceil(rho * len(mass) - 1e-9))
    order = np.argsort(-mass, kind="stable")
    return np.sort(order[:n])
