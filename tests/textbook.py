"""Textbook dense softmax attention (scipy routines), used only to pin the oracle."""
import numpy as np
from scipy.special import logsumexp, softmax


def dense_attention(q, K, V, scale):
    x = np.asarray(K, dtype=np.float64) @ np.asarray(q, dtype=np.float64) * scale
    p = softmax(x)
    return p @ np.asarray(V, dtype=np.float64), logsumexp(x)
