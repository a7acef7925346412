"""Sequence-sharded forward over several GPUs (one process per GPU).

Rank p holds a contiguous range [t0, t1) of the sequence: the q, k and v
rows of every sample and head there, and produces the output rows of that
range.  Two things cross ranks:

* the halo: a row's window reaches dil * r positions on each side (the
  "Longformer" note, section "Sliding-Window Attention"; the dilation of the
  Longformer wiki, section 2.2.3), so the k and v rows within max(dil) * r
  of the range's ends come from the neighbouring ranks;
* the global tokens: every row also attends the global keys, and a global
  row attends every key ("Longformer" note, section "Global Attention").
  The k, v and q rows at the global positions are gathered from their
  owners; each rank then computes the global rows' softmax state over its
  own keys only (lf_attn_rows_partial), and the states of all ranks merge
  into the global rows' outputs (lf_attn_merge_rows) on the rank that owns
  each row.

Each rank's band rows come from one lf_attn_fwd call per sample on a local
sequence: the left halo, its own rows, the right halo, then the global keys
that lie outside that span (appended at the end, where no kept row's window
reaches).  The global keys inside the span stay global in place, so a
global key inside a row's window still counts once.  The local call also
computes rows that are thrown away (the halo rows, the appended rows, and
the global rows, which see only local keys there).

The pages motivate this for inputs longer than one GPU holds (Longformer
wiki, sections 5.3 and 7.1).  Collectives are torch.distributed all-gathers
(NCCL between GPUs); with the gloo backend tensors go through host memory.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def shard_range(T: int, world: int, rank: int) -> Tuple[int, int]:
    """The even split of [0, T) used by default: rank p gets [T p / N, T (p + 1) / N)."""
    if not (0 <= rank < world) or T <= 0:
        raise ValueError("bad shard")
    return T * rank // world, T * (rank + 1) // world


def _gather(t: torch.Tensor, group) -> List[torch.Tensor]:
    """all_gather of equal-shaped tensors; through host memory under gloo."""
    world = dist.get_world_size(group)
    host = dist.get_backend(group) == "gloo" and t.is_cuda
    src = t.cpu() if host else t.contiguous()
    out = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(out, src, group=group)
    return [x.to(t.device) for x in out] if host else out


class CudaOps:
    """The library's kernels (the default compute of fwd_sharded)."""

    def __init__(self):
        from sparse_long_sequence_fwd_b200 import lf_attn
        self.lf = lf_attn

    def local(self, q, k, v, r, dil, gidx: List[int], pad, scale):
        g = torch.tensor([gidx], dtype=torch.int32, device=q.device) if gidx else None
        return self.lf.fwd(q, k, v, r, dil=dil, global_idx=g, key_pad_mask=pad, scale=scale)

    def rows_partial(self, q_rows, k, v, pad, scale):
        return self.lf.rows_partial(q_rows, k, v, pad, scale)

    def merge(self, ml, acc, pos, out):
        self.lf.merge_rows(ml, acc, pos, out)


def fwd_sharded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, r: int, t0: int, T: int,
                dil: Optional[Sequence[int]] = None, global_idx: Optional[torch.Tensor] = None,
                key_pad_mask: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                group=None, ops=None) -> torch.Tensor:
    """This rank's output rows [B, H, t1 - t0, d].

    q, k, v: this rank's rows [B, H, t1 - t0, d] of a [B, H, T, d] problem;
    the ranks' ranges must tile [0, T) in rank order.  dil: per-head
    dilation (host ints).  global_idx: int32 [B, n_global] positions in
    [0, T) (the same on every rank).  key_pad_mask: uint8 [B, T], the whole
    sequence's (the same on every rank).  Every rank's range must be at
    least max(dil) * r long, so each halo comes from the next rank alone.
    """
    ops = ops if ops is not None else CudaOps()
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    B, H, L, d = q.shape
    dev = q.device
    dil = [1] * H if dil is None else [int(x) for x in dil]
    scale = d ** -0.5 if scale is None else float(scale)
    t1 = t0 + L
    ranges = [None] * world
    dist.all_gather_object(ranges, (t0, t1), group=group)
    if ranges[0][0] != 0 or ranges[-1][1] != T or any(ranges[p][1] != ranges[p + 1][0] for p in range(world - 1)):
        raise ValueError("the ranks' ranges must tile [0, T) in rank order: %s" % (ranges,))
    h = max(dil) * r
    lengths = [b_ - a_ for a_, b_ in ranges]
    if world > 1 and min(lengths) < h:
        raise ValueError("every range must be at least max(dil) * r = %d rows long" % h)
    hl, hr = min(t0, h), min(T - t1, h)

    # ---- halo: every rank's first and last h rows of k and v
    hh = min(h, L)
    edge = torch.cat([k[:, :, :hh], k[:, :, L - hh:], v[:, :, :hh], v[:, :, L - hh:]], dim=2)
    edges = _gather(edge, group)
    left_k = edges[rank - 1][:, :, 2 * hh - hl: 2 * hh] if hl else k[:, :, :0]
    left_v = edges[rank - 1][:, :, 4 * hh - hl: 4 * hh] if hl else v[:, :, :0]
    right_k = edges[rank + 1][:, :, :hr] if hr else k[:, :, :0]
    right_v = edges[rank + 1][:, :, 2 * hh: 2 * hh + hr] if hr else v[:, :, :0]

    # ---- global rows: q, k, v at the global positions, gathered from their owners
    Gs: List[List[int]] = []
    for b in range(B):
        row = [] if global_idx is None else [int(x) for x in global_idx[b].tolist()]
        Gs.append(sorted({g for g in row if 0 <= g < T}))
    gmax = max([len(g) for g in Gs] + [0])
    out = None
    owner = lambda g: next(p for p, (a_, b_) in enumerate(ranges) if a_ <= g < b_)
    if gmax:
        mine = torch.zeros((3, B, H, gmax, d), dtype=q.dtype, device=dev)
        for b in range(B):
            for a, g in enumerate(Gs[b]):
                if t0 <= g < t1:
                    mine[0, b, :, a] = q[b, :, g - t0]
                    mine[1, b, :, a] = k[b, :, g - t0]
                    mine[2, b, :, a] = v[b, :, g - t0]
        allg = _gather(mine, group)
        glob = torch.zeros_like(mine)
        for b in range(B):
            for a, g in enumerate(Gs[b]):
                glob[:, b, :, a] = allg[owner(g)][:, b, :, a]
        qg, kg, vg = glob[0].contiguous(), glob[1], glob[2]

    # ---- band rows: one local call per sample
    outs = []
    lo, hi = t0 - hl, t1 + hr
    for b in range(B):
        inside = [g for g in Gs[b] if lo <= g < hi]
        app = [a for a, g in enumerate(Gs[b]) if not lo <= g < hi]
        parts_k = [left_k[b:b + 1], k[b:b + 1], right_k[b:b + 1]]
        parts_v = [left_v[b:b + 1], v[b:b + 1], right_v[b:b + 1]]
        if app:
            idx = torch.tensor(app, device=dev)
            parts_k.append(kg[b:b + 1].index_select(2, idx))
            parts_v.append(vg[b:b + 1].index_select(2, idx))
        ke = torch.cat(parts_k, dim=2).contiguous()
        ve = torch.cat(parts_v, dim=2).contiguous()
        Te = ke.shape[2]
        qe = torch.zeros_like(ke)
        qe[:, :, hl:hl + L] = q[b:b + 1]
        gidx = [g - lo for g in inside] + [hi - lo + i for i in range(len(app))]
        pad = None
        if key_pad_mask is not None:
            pm = key_pad_mask[b]
            pieces = [pm[lo:hi]] + ([pm[torch.tensor([Gs[b][a] for a in app], device=pm.device)]] if app else [])
            pad = torch.cat(pieces).reshape(1, Te).to(torch.uint8).contiguous()
        oe = ops.local(qe, ke, ve, r, dil, gidx, pad, scale)
        outs.append(oe[:, :, hl:hl + L])
    out = torch.cat(outs, dim=0).contiguous()

    # ---- global rows: partial states over this rank's keys, merged on the owners
    if gmax:
        pad_own = None if key_pad_mask is None else key_pad_mask[:, t0:t1].to(torch.uint8).contiguous()
        ml, acc = ops.rows_partial(qg, k.contiguous(), v.contiguous(), pad_own, scale)
        ml_all = torch.stack(_gather(ml, group)).contiguous()
        acc_all = torch.stack(_gather(acc, group)).contiguous()
        pos = torch.full((B, gmax), -1, dtype=torch.int32)
        for b in range(B):
            for a, g in enumerate(Gs[b]):
                if t0 <= g < t1:
                    pos[b, a] = g - t0
        ops.merge(ml_all, acc_all, pos.to(dev), out)
    return out
