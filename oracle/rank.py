"""Layer ranking for the zero-search precision rule.

TEST INFRASTRUCTURE ONLY. Source: "AQLoRA", abstract and §3.1/§3.2: rank the linear
layers by their NF4 reconstruction error epsilon_l = SSE_l / |W_l| and keep the K
most damaged ones in 16-bit. The memory-budget form of the rule is cut off on the
page; K is a fixed input here. Ties in epsilon go to the lower layer index.
"""
from __future__ import annotations

import numpy as np


def top_k(sse, n_params, k: int) -> np.ndarray:
    """Indices of the k layers with the largest epsilon = sse / n, descending."""
    sse = np.asarray(sse, dtype=np.float64)
    n = np.asarray(n_params, dtype=np.float64)
    eps = sse / n
    order = sorted(range(eps.size), key=lambda i: (-eps[i], i))
    return np.array(order[:k], dtype=np.int64)
