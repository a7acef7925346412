"""The sequence-sharded forward's host logic (ranges, halos, global rows and
their merge) on CPU: world-size 2 and 3 gloo process groups, with the
oracle standing in for the local kernels and fp64 numpy for the global
rows' partial states.  The assembled output must equal the oracle on the
whole problem.  (The GPU test runs the same path with the library's
kernels.)"""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_long_sequence_fwd_b200 import sequence_shard

LOG2E = 1.4426950408889634


class OracleOps:
    """fp64 stand-ins for the library's kernels (test infrastructure)."""

    def local(self, q, k, v, r, dil, gidx, pad, scale):
        g = np.array([gidx], dtype=np.int32) if gidx else None
        y = oracle.fwd(q, k, v, r, dil=dil, global_idx=g, key_pad_mask=None if pad is None else pad.numpy(),
                       scale=scale)
        return torch.from_numpy(y)

    def rows_partial(self, q_rows, k, v, pad, scale):
        qd, kd, vd = q_rows.double().numpy(), k.double().numpy(), v.double().numpy()
        B, H, n, d = qd.shape
        ml = np.zeros((B, H, n, 2))
        acc = np.zeros((B, H, n, d))
        for b in range(B):
            keep = np.ones(kd.shape[2], dtype=bool) if pad is None else pad[b].numpy() == 0
            for h in range(H):
                s = scale * LOG2E * (qd[b, h] @ kd[b, h].T)        # [n, T]
                s = np.where(keep[None, :], s, -np.inf)
                M = s.max(axis=1)
                Mu = np.where(np.isfinite(M), M, 0.0)
                w = np.exp2(s - Mu[:, None])
                ml[b, h, :, 0], ml[b, h, :, 1] = M, w.sum(axis=1)
                acc[b, h] = w @ vd[b, h]
        return torch.from_numpy(ml), torch.from_numpy(acc)

    def merge(self, ml, acc, pos, out):
        M = ml[..., 0].max(dim=0).values
        Mu = torch.where(torch.isfinite(M), M, torch.zeros_like(M))
        w = torch.exp2(ml[..., 0] - Mu[None])
        L = (w * ml[..., 1]).sum(0)
        y = (w[..., None] * acc).sum(0) / torch.where(L > 0, L, torch.ones_like(L))[..., None]
        y = torch.where((L > 0)[..., None], y, torch.zeros_like(y))
        B, n = pos.shape
        for b in range(B):
            for a in range(n):
                if int(pos[b, a]) >= 0:
                    out[b, :, int(pos[b, a])] = y[b, :, a].to(out.dtype)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, ranges, case, tmp):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, r, dil, G, pad, scale = case
        t0, t1 = ranges[rank]
        out = sequence_shard.fwd_sharded(q[:, :, t0:t1].contiguous(), k[:, :, t0:t1].contiguous(),
                                         v[:, :, t0:t1].contiguous(), r, t0, q.shape[2], dil=dil, global_idx=G,
                                         key_pad_mask=pad, scale=scale, ops=OracleOps())
        np.save(os.path.join(tmp, "out%d.npy" % rank), out.double().numpy())
    finally:
        dist.destroy_process_group()


def _case(B, H, T, d, r, dil, G, pad_from, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, T, d, generator=g) for _ in range(3))
    Gt = None if G is None else torch.tensor(G, dtype=torch.int32)
    pad = None
    if pad_from is not None:
        pad = torch.zeros(B, T, dtype=torch.uint8)
        for b, p in enumerate(pad_from):
            if p is not None:
                pad[b, p:] = 1
    return q, k, v, r, dil, Gt, pad, 0.3


CASES = [
    # world 2, even split, dilations, duplicate / out-of-range / padded globals
    (2, None, _case(2, 2, 300, 8, 20, [1, 2], [[5, 150, 299, 150, -1], [0, 0, 170, 40, 400]], [None, 260], 1)),
    # world 3, uneven ranges, a global key in every range and in a halo
    (3, [(0, 100), (100, 190), (190, 260)], _case(1, 3, 260, 4, 15, [1, 3, 2], [[3, 99, 105, 189, 250]], [240], 2)),
    # world 2, no globals, r = 0
    (2, None, _case(1, 2, 64, 4, 0, [1, 1], None, None, 3)),
]


@pytest.mark.parametrize("world,ranges,case", CASES)
def test_sequence_sharded_forward_matches_oracle(world, ranges, case):
    q, k, v, r, dil, G, pad, scale = case
    T = q.shape[2]
    ranges = ranges or [sequence_shard.shard_range(T, world, p) for p in range(world)]
    with tempfile.TemporaryDirectory() as tmp:
        mp.start_processes(_worker, args=(world, _free_port(), ranges, case, tmp), nprocs=world, join=True,
                           start_method="spawn")
        got = np.concatenate([np.load(os.path.join(tmp, "out%d.npy" % p)) for p in range(world)], axis=2)
    ref = oracle.fwd(q, k, v, r, dil=dil, global_idx=G, key_pad_mask=pad, scale=scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-10)


def test_shard_range_tiles_the_sequence():
    for T in (1, 7, 100):
        for world in (1, 2, 3, 8):
            rs = [sequence_shard.shard_range(T, world, p) for p in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == T
            assert all(rs[p][1] == rs[p + 1][0] for p in range(world - 1))
