"""Dense brute force of Longformer sparse attention (fp64, numpy).

A second, independent formulation used only to pin the oracle: it builds the
full T x T additive mask of the "Longformer" note (eightmm.github.io), section
"Mask View" (M_ij = 0 for j in N(i), -inf otherwise; A = QK^T/sqrt(d) + M)
from a vectorised membership rule instead of enumerating window offsets:

    allowed(i, j) = ( (|i - j| <= dil*r and (i - j) mod dil == 0)
                      or j in G or i in G )  and  not pad(j)

and takes a row softmax of the whole dense score matrix.
"""
import numpy as np


def dense_mask(T, r, dil, G, pad):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    diff = i - j
    window = (np.abs(diff) <= dil * r) & (diff % dil == 0)
    g = np.zeros(T, dtype=bool)
    for x in (G if G is not None else []):
        if 0 <= x < T:
            g[x] = True
    allowed = window | g[None, :] | g[:, None]
    if pad is not None:
        allowed &= ~np.asarray(pad, dtype=bool)[None, :]
    return allowed


def dense_attention(q, k, v, allowed, scale):
    """q, k, v: fp64 [T, d]; allowed: bool [T, T]; rows with no key give 0."""
    A = (q @ k.T) * scale
    A = np.where(allowed, A, -np.inf)
    m = A.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    P = np.exp(A - m)
    l = P.sum(axis=1, keepdims=True)
    y = P @ v
    return np.where(l > 0, y / np.where(l > 0, l, 1.0), 0.0)


def dense_forward(q, k, v, r, dil, global_idx, key_pad_mask, scale):
    """q, k, v: [B, H, T, d] (numpy fp64); dil: [H]; global_idx [B, n] or None."""
    B, H, T, d = q.shape
    out = np.zeros_like(q)
    for b in range(B):
        G = [] if global_idx is None else list(np.asarray(global_idx)[b])
        pad = None if key_pad_mask is None else np.asarray(key_pad_mask)[b]
        for h in range(H):
            allowed = dense_mask(T, r, int(dil[h]), G, pad)
            out[b, h] = dense_attention(q[b, h], k[b, h], v[b, h], allowed, scale)
    return out
