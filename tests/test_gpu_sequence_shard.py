"""The sequence-sharded forward with the library's kernels: two ranks (gloo
process group) sharing one GPU, each holding half of the sequence.  The
ranks' kernels never wait on one another (the exchanges are host-side
collectives between launches).  The assembled output is compared with the
oracle on the whole problem at the parity bar."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_long_sequence_fwd_b200 import build, sequence_shard, workloads
from tests import parity

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, w, tmp):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = workloads.make_inputs(w)
        t0, t1 = sequence_shard.shard_range(w.T, world, rank)
        dev = torch.device("cuda", 0)
        sl = lambda x: x[:, :, t0:t1].contiguous().to(dev)
        G = inp["global_idx"].to(dev) if inp["global_idx"] is not None else None
        pad = inp["key_pad_mask"].to(dev) if inp["key_pad_mask"] is not None else None
        out = sequence_shard.fwd_sharded(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), w.r, t0, w.T,
                                         dil=inp["dil"].tolist(), global_idx=G, key_pad_mask=pad,
                                         scale=w.softmax_scale)
        torch.cuda.synchronize()
        np.save(os.path.join(tmp, "out%d.npy" % rank), out.double().cpu().numpy())
    finally:
        dist.destroy_process_group()


CASES = [
    workloads.custom("shard_bf16", "bf16", 2, 4, 2048, 64, 64, dil=[1, 2, 1, 2],
                     globals_per_b=[[0, 700, 2047, 1030], [5, 5, 1500, 1023]], pad_from=[None, 1900], seed=81),
    workloads.custom("shard_f16_d128", "f16", 1, 2, 1500, 128, 100, globals_per_b=[[0, 760]], seed=82),
    workloads.custom("shard_f32", "f32", 1, 2, 800, 64, 40, dil=[1, 2], globals_per_b=[[10, 500]], pad_from=[790],
                     seed=83),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_sequence_sharded_forward_on_one_gpu_two_ranks(w):
    build.build()
    with tempfile.TemporaryDirectory() as tmp:
        mp.start_processes(_worker, args=(2, _free_port(), w, tmp), nprocs=2, join=True, start_method="spawn")
        got = np.concatenate([np.load(os.path.join(tmp, "out%d.npy" % p)) for p in range(2)], axis=2)
    inp = workloads.make_inputs(w)
    ref = parity.oracle_full(w, inp)
    parity.compare(w, torch.from_numpy(got), ref)
