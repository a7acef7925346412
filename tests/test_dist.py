"""Multi-rank host logic on CPU with gloo (world_size 2): the (b, h)
partition covers every slab once, per-rank results assembled from the pieces
equal the single-process result (the oracle stands in for the GPU kernel),
and the timing reduction takes the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_long_sequence_fwd_b200 import sharding, workloads


def test_partition_covers_each_slab_once_and_balances():
    for B, H, world in [(1, 12, 2), (2, 12, 8), (3, 5, 4), (1, 1, 1), (2, 3, 7)]:
        parts = sharding.partition_bh(B, H, world)
        seen = []
        sizes = []
        for pieces in parts:
            n = 0
            for b, h0, h1 in pieces:
                assert 0 <= b < B and 0 <= h0 < h1 <= H
                seen += [(b, h) for h in range(h0, h1)]
                n += h1 - h0
            sizes.append(n)
        assert sorted(seen) == [(b, h) for b in range(B) for h in range(H)]
        assert max(sizes) - min(sizes) <= 1


def test_job_rate():
    assert sharding.job_rate(10.0, 4, 2.0) == 20.0
    with pytest.raises(ValueError):
        sharding.job_rate(1.0, 1, 0.0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, result_dir):
    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.custom("dist", "f32", 2, 3, 40, 8, 3, dil=[1, 2, 1], globals_per_b=[[0, 7], [5, 5]],
                             pad_from=[None, 30], seed=9)
        inp = workloads.make_inputs(w)
        out = np.zeros((w.B, w.H, w.T, w.d))
        for b, h0, h1 in sharding.partition_bh(w.B, w.H, world)[rank]:
            sl = (slice(b, b + 1), slice(h0, h1))
            out[b, h0:h1] = oracle.fwd(inp["q"][sl], inp["k"][sl], inp["v"][sl], w.r, dil=inp["dil"][h0:h1],
                                       global_idx=inp["global_idx"][b:b + 1],
                                       key_pad_mask=inp["key_pad_mask"][b:b + 1], scale=w.softmax_scale)[0]
        t = torch.from_numpy(out)
        dist.all_reduce(t)  # pieces are disjoint: the sum assembles the full result
        ms = sharding.max_over_ranks(1.5 + rank)
        if rank == 0:
            np.save(os.path.join(result_dir, "out.npy"), t.numpy())
            np.save(os.path.join(result_dir, "ms.npy"), np.array([ms]))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_sharded_forward_and_timing(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    import oracle

    w = workloads.custom("dist", "f32", 2, 3, 40, 8, 3, dil=[1, 2, 1], globals_per_b=[[0, 7], [5, 5]],
                         pad_from=[None, 30], seed=9)
    inp = workloads.make_inputs(w)
    ref = oracle.fwd(inp["q"], inp["k"], inp["v"], w.r, dil=inp["dil"], global_idx=inp["global_idx"],
                     key_pad_mask=inp["key_pad_mask"], scale=w.softmax_scale)
    got = np.load(tmp_path / "out.npy")
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-14)
    assert float(np.load(tmp_path / "ms.npy")[0]) == 2.5
