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


def _cfg_worker(rank, world, port, out_dir):
    """Each rank runs the oracle's forward for its own branch (the GPU forward's
    stand-in on CPU); the split loop exchanges outputs and steps both ranks."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import scheduler_ref as sch
        from oracle import zimage_ref as ref
        from stream_diffusion_transformer_b200 import model
        d = zi.TINY_R
        W = ref.Weights(zi.make_weights(d, seed=4))
        txt = zi.bf16_bits_to_f32(zi.make_text(d, 1, 6, seed=4, uncond=(rank == 1))).astype(np.float64)

        def forward(x, t):
            return torch.from_numpy(ref.model_forward(x.numpy().astype(np.float64), t.numpy().astype(np.float64),
                                                      txt, W, d).astype(np.float32))

        def euler(x, yc, yu, g, s0, s1):
            y = sch.cfg_combine(yc.numpy().astype(np.float64), yu.numpy().astype(np.float64), g)
            x.copy_(torch.from_numpy(sch.euler_step(x.numpy().astype(np.float64), y, s0, s1).astype(np.float32)))

        lat = torch.from_numpy(zi.make_latent(d, 1, 6, 4, seed=4))
        out = model.denoise_cfg_split(lat, 3, 3.0, 4.0, forward, euler)
        np.save(os.path.join(out_dir, f"cfg{rank}.npy"), out.numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_cfg_split_matches_one_process_cfg():
    """The CFG branches on two ranks with one all-gather per step give the latent of
    the one-process guided loop (oracle scheduler), identically on both ranks."""
    import tempfile
    from oracle import scheduler_ref as sch
    from oracle import zimage_ref as ref
    with tempfile.TemporaryDirectory() as tmp:
        port = _free_port()
        mp.start_processes(_cfg_worker, args=(2, port, tmp), nprocs=2, join=True, start_method="spawn")
        r0 = np.load(os.path.join(tmp, "cfg0.npy"))
        r1 = np.load(os.path.join(tmp, "cfg1.npy"))
    np.testing.assert_array_equal(r0, r1)
    d = zi.TINY_R
    W = ref.Weights(zi.make_weights(d, seed=4))
    tc = zi.bf16_bits_to_f32(zi.make_text(d, 1, 6, seed=4)).astype(np.float64)
    tu = zi.bf16_bits_to_f32(zi.make_text(d, 1, 6, seed=4, uncond=True)).astype(np.float64)

    def model_fn(x, t, uncond):
        return ref.model_forward(x, t, tu if uncond else tc, W, d)

    want = sch.denoise(zi.make_latent(d, 1, 6, 4, seed=4).astype(np.float64), model_fn, 3, 3.0, 4.0)
    np.testing.assert_allclose(r0, want, rtol=1e-5, atol=1e-5)
