"""Useful-work accounting for the benchmark.

Useful FLOPs of one forward = sum over (b, h, i) of 4 * d * |N(i)|: one
multiply-add per (query, key, channel) for q.k and one for p*v, counting only
the keys the pattern keeps (masked tile waste excluded).  |N(i)| is counted
with per-residue-class prefix sums instead of by enumerating keys:

  * ordinary row: non-padded window keys + non-padded global keys outside
    the window;
  * global row: every non-padded key.

The pattern follows the "Longformer" note (eightmm.github.io), sections
"Sliding-Window Attention" and "Global Attention", with the dilation of the
Longformer wiki (ciallo.wiki) section 2.2.3; the cost model is that note's
"Relation to Dense Attention" table (O(Tw + Tg)).
"""
from __future__ import annotations

import numpy as np


def row_key_counts(T: int, r: int, dil: int, globals_b=None, pad_b=None) -> np.ndarray:
    """|N(i)| for every row of one sample and one head dilation (int64 [T])."""
    valid = np.ones(T, dtype=bool) if pad_b is None else ~np.asarray(pad_b, dtype=bool)
    cnt = np.zeros(T, dtype=np.int64)
    for c in range(min(dil, T)):
        pos = np.arange(c, T, dil)
        pre = np.concatenate([[0], np.cumsum(valid[pos].astype(np.int64))])
        idx = np.arange(pos.size)
        lo = np.maximum(idx - r, 0)
        hi = np.minimum(idx + r, pos.size - 1)
        cnt[pos] = pre[hi + 1] - pre[lo]
    G = np.unique(np.asarray([g for g in (globals_b if globals_b is not None else [])
                              if 0 <= int(g) < T], dtype=np.int64))
    Gk = G[valid[G]] if G.size else G
    if Gk.size:
        i = np.arange(T, dtype=np.int64)[:, None]
        diff = Gk[None, :] - i
        in_win = (np.abs(diff) <= dil * r) & (diff % dil == 0)
        cnt += Gk.size - in_win.sum(axis=1)
    if G.size:
        cnt[G] = int(valid.sum())
    return cnt


def rand_extra_counts(T: int, r: int, globals_b, pad_b, rb_bh) -> np.ndarray:
    """Keys the random key blocks add to each ordinary row of one (b, h) (the
    BigBird variant, dilation 1): the non-padded keys of the distinct blocks
    drawn for the row's 64-row query block that lie outside the row's window
    and are not global (int64 [T]; global rows get 0)."""
    valid = np.ones(T, dtype=bool) if pad_b is None else ~np.asarray(pad_b, dtype=bool)
    g = np.zeros(T, dtype=bool)
    for x in (globals_b if globals_b is not None else []):
        if 0 <= int(x) < T:
            g[int(x)] = True
    extra = np.zeros(T, dtype=np.int64)
    rb_bh = np.asarray(rb_bh)
    nqb = (T + 63) // 64
    for qb in range(nqb):
        blocks = sorted({int(c) for c in rb_bh[qb] if 0 <= int(c) < nqb})
        for c in blocks:
            j = np.arange(64 * c, min(64 * c + 64, T))
            keep = valid[j] & ~g[j]
            for i in range(64 * qb, min(64 * qb + 64, T)):
                if not g[i]:
                    extra[i] += int((keep & (np.abs(j - i) > r)).sum())
    return extra


def total_keys(B, H, T, r, dil, global_idx=None, key_pad_mask=None) -> int:
    """Sum of |N(i)| over every (b, h, i)."""
    dil = [int(x) for x in dil]
    total = 0
    for b in range(B):
        G = None if global_idx is None else np.asarray(global_idx)[b]
        pad = None if key_pad_mask is None else np.asarray(key_pad_mask)[b]
        per_dil = {}
        for h in range(H):
            if dil[h] not in per_dil:
                per_dil[dil[h]] = int(row_key_counts(T, r, dil[h], G, pad).sum())
            total += per_dil[dil[h]]
    return total


def useful_flops(B, H, T, d, r, dil, global_idx=None, key_pad_mask=None) -> float:
    return 4.0 * d * total_keys(B, H, T, r, dil, global_idx, key_pad_mask)


def min_bytes(B, H, T, d, elem_bytes: int) -> int:
    """q, k, v read once and out written once."""
    return 4 * B * H * T * d * elem_bytes
