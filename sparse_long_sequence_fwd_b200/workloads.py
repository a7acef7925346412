"""Seeded synthetic workloads for Longformer sparse self-attention (forward).

This module only *generates inputs*: shapes, seeded Q/K/V values, the global
token selection and the key padding mask.  It holds none of the attention
arithmetic, so the CPU oracle and the CUDA library can both be fed from it
without sharing any of the method.

Recipe (the same for every workload):
  * ``g = torch.Generator().manual_seed(seed)``;
  * ``q``, ``k``, ``v`` drawn in that order with ``torch.randn(B, H, T, d,
    generator=g)`` (fp32, iid N(0, 1));
  * bf16 workloads round them with ``.to(torch.bfloat16)`` and f16 workloads
    with ``.to(torch.float16)`` (round to nearest even); the oracle reads those
    rounded values widened to fp64;
  * random global positions (if any) are drawn from the same generator after
    v, with ``torch.randperm``;
  * the key padding mask is uint8 [B, T], nonzero = padded key.

The shapes stand in for the pages' workloads: Longformer-base at 4096 tokens
with a ~512 window (Longformer wiki, section 5.2 and 2.2.1), a question span
made global for long-document QA (Longformer wiki, section 7.3; the aiqz.cc
engineering page, "global tokens"), dilation on some heads (aiqz.cc, "dilated
window"), and >16K-token inputs (Longformer wiki, section 5.3).  No dataset
is read.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                      # "f32", "bf16" or "f16"
    B: int
    H: int
    T: int
    d: int
    r: int                          # one-sided window radius, w = 2r + 1
    dil: Sequence[int]              # per-head dilation, len H
    globals_per_b: Optional[Sequence[Sequence[int]]]  # explicit global positions per sample
    n_random_globals: int = 0       # if > 0: {0} + (n-1) seeded draws, same set for every sample
    pad_from: Optional[Sequence[Optional[int]]] = None  # per sample: keys >= pad_from[b] are padded
    scale: Optional[float] = None   # None -> 1/sqrt(d)
    seed: int = 0
    n_rand: int = 0                 # BigBird variant: random key blocks per 64-row query block

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    @property
    def w(self) -> int:
        return 2 * self.r + 1


def _dil(H: int, spec) -> List[int]:
    return [int(x) for x in spec] if isinstance(spec, (list, tuple)) else [int(spec)] * H


# The five workloads, in order: tiny fp32 case, Longformer-base layer,
# long-document QA, dilated heads, Longformer-large-like long input.
TINY = Workload("tiny_f32_T64", "f32", 1, 2, 64, 16, 4, _dil(2, 1),
                globals_per_b=[[0, 37]], scale=0.25, seed=1001)
BASE = Workload("base_T4096_w513", "bf16", 1, 12, 4096, 64, 256, _dil(12, 1),
                globals_per_b=[[0]], scale=0.125, seed=1002)
QA = Workload("qa_B2_T4096_g64_pad", "bf16", 2, 12, 4096, 64, 256, _dil(12, 1),
              globals_per_b=[list(range(64)), list(range(64))],
              pad_from=[None, 3001], scale=0.125, seed=1003)
DILATED = Workload("dilated_T8192_r128", "bf16", 1, 12, 8192, 64, 128,
                   [1, 1] + [2] * 10, globals_per_b=[[0]], scale=0.125, seed=1004)
LARGE = Workload("large_T16384_g32", "bf16", 1, 16, 16384, 64, 256, _dil(16, 1),
                 globals_per_b=None, n_random_globals=32, scale=0.125, seed=1005)

# the base workload with f16 inputs (the pages train with fp16 mixed
# precision: Longformer wiki, section 6.3)
BASE_F16 = dataclasses.replace(BASE, name="base_T4096_w513_f16", dtype="f16")
# 128-dimensional heads (8 of them, the same model width as 16 heads of 64)
D128 = Workload("d128_H8_T4096_w513", "bf16", 1, 8, 4096, 128, 256, _dil(8, 1),
                globals_per_b=[[0]], scale=128 ** -0.5, seed=1006)

# the BigBird variant of the base workload: 3 random key blocks of 64 per
# 64-row query block (mhpn.cn page, sections 2.2.1 and 2.2.2)
BIGBIRD = dataclasses.replace(BASE, name="bigbird_T4096_w513_rand3", n_rand=3)

ALL = [TINY, BASE, QA, DILATED, LARGE, BASE_F16, D128, BIGBIRD]
BY_NAME = {w.name: w for w in ALL}


def make_inputs(w: Workload, device: str = "cpu"):
    """Seeded inputs for a workload.

    Returns a dict with ``q, k, v`` ([B, H, T, d], fp32, bf16 or f16),
    ``global_idx`` (int32 [B, n_global] or None), ``key_pad_mask``
    (uint8 [B, T] or None) and ``dil`` (int32 [H], host).
    """
    g = torch.Generator().manual_seed(w.seed)
    shape = (w.B, w.H, w.T, w.d)
    q = torch.randn(shape, generator=g)
    k = torch.randn(shape, generator=g)
    v = torch.randn(shape, generator=g)
    if w.dtype == "bf16":
        q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    elif w.dtype == "f16":
        q, k, v = (t.to(torch.float16) for t in (q, k, v))
    elif w.dtype != "f32":
        raise ValueError(w.dtype)

    if w.n_random_globals > 0:
        n = w.n_random_globals
        draws = torch.randperm(w.T - 1, generator=g)[: n - 1] + 1
        gl = sorted([0] + draws.tolist())
        gidx = torch.tensor([gl] * w.B, dtype=torch.int32)
    elif w.globals_per_b is not None and len(w.globals_per_b[0]) > 0:
        gidx = torch.tensor([list(x) for x in w.globals_per_b], dtype=torch.int32)
    else:
        gidx = None

    pad = None
    if w.pad_from is not None and any(p is not None for p in w.pad_from):
        pad = torch.zeros((w.B, w.T), dtype=torch.uint8)
        for b, p in enumerate(w.pad_from):
            if p is not None:
                pad[b, p:] = 1

    rand_blocks = None
    if w.n_rand > 0:  # drawn last, so the other inputs do not depend on it
        nqb = (w.T + 63) // 64
        rand_blocks = torch.randint(0, nqb, (w.B, w.H, nqb, w.n_rand), generator=g, dtype=torch.int64).to(torch.int32)

    out = dict(q=q, k=k, v=v, global_idx=gidx, key_pad_mask=pad,
               dil=torch.tensor(list(w.dil), dtype=torch.int32), rand_blocks=rand_blocks)
    if device != "cpu":
        for key in ("q", "k", "v", "global_idx", "key_pad_mask", "rand_blocks"):
            if out[key] is not None:
                out[key] = out[key].to(device)
    return out


def custom(name: str, dtype: str, B: int, H: int, T: int, d: int, r: int, dil=1,
           globals_per_b=None, pad_from=None, scale=None, seed: int = 7,
           n_random_globals: int = 0, n_rand: int = 0) -> Workload:
    """A small ad-hoc workload (edge cases in the tests)."""
    return Workload(name, dtype, B, H, T, d, r, _dil(H, dil), globals_per_b,
                    n_random_globals, pad_from, scale, seed, n_rand)
