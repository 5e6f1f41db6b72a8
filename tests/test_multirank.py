"""The multi-GPU replica path of bench.py, exercised on the CPU with two gloo ranks.

`bench.py --gpus N` runs N independent forwards (the forward has no exchange
step): rank 0 draws the seeded weights and broadcasts them, every rank times its
own device, and the job's time is the maximum over ranks.  These are the
host-side pieces; here they run over gloo on CPU tensors, world size 2."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import zimage_inputs as zi


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        d = zi.TINY_R
        fetch = bench.make_fetch(d, rank, world, torch.device("cpu"), threads=2)
        keys = [k for k, _, _ in zi.weight_specs(d)][:6] + ["layers.0.feed_forward.w2.weight"]
        got = fetch(keys)
        digest = np.array([int(got[k].astype(np.uint64).sum()) for k in keys], dtype=np.int64)
        ms = bench.max_over_ranks(10.0 + rank * 5.0, world, torch.device("cpu"))
        np.save(os.path.join(out_dir, f"r{rank}.npy"), np.concatenate([digest, [int(ms * 1000)]]))
    finally:
        dist.destroy_process_group()


def test_two_rank_weight_broadcast_and_max_timing(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r0 = np.load(tmp_path / "r0.npy")
    r1 = np.load(tmp_path / "r1.npy")
    # both replicas hold rank 0's weights (identical to drawing them directly)
    np.testing.assert_array_equal(r0[:-1], r1[:-1])
    d = zi.TINY_R
    keys = [k for k, _, _ in zi.weight_specs(d)][:6] + ["layers.0.feed_forward.w2.weight"]
    direct = zi.make_weights(d, seed=0, keys=keys)
    np.testing.assert_array_equal(r0[:-1], [int(direct[k].astype(np.uint64).sum()) for k in keys])
    # the job time is the slowest rank's
    assert r0[-1] == r1[-1] == 15000
