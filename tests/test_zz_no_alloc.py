"""zi_block_forward_noalloc: the block forward for callers that cannot allocate.

Some callers cannot hand the library a workspace: a plugin inside a host
program whose memory manager owns all device memory and gives plugins no
allocator, or a latency-critical loop that forbids cudaMalloc after start-up.
For them the library keeps a fixed 128 MiB device scratch array of its own.

zi_block_forward_noalloc runs exactly the kernels zi_block_forward runs, on the
same inputs, with that array in place of a caller's workspace, and every scratch
byte a call reads is written earlier in the same call.  So its output must be
bit-identical to zi_block_forward's.  These tests call it through the C ABI two
times in a row (different inputs, so the second call runs on scratch the first
one left behind), and a small call right after a large one (a stale byte of the
large call would show), comparing each output bit for bit with zi_block_forward
given a freshly allocated workspace; they also check that the calls leave the
device's free memory unchanged.  The file sorts last so a run that stops at the
first failure has already run every other test.
"""
import ctypes
import dataclasses

import numpy as np
import pytest

from gpu_util import require_gpu, torch
import zimage_inputs as zi

pytestmark = pytest.mark.gpu

FULL1 = dataclasses.replace(zi.FULL, n_noise=0, n_ctx=0, n_main=1)


def _setup(d, modulated, seed):
    from stream_diffusion_transformer_b200 import abi, model
    cfg = model.make_config(d)
    bits = zi.make_weights(d, seed=seed, keys=model.block_keys("layers.0", modulated))
    blk = model.DeviceBlock(cfg, "layers.0", bits, modulated, "cuda")
    return abi, model, cfg, blk


def _inputs(d, modulated, s_txt, gh, gw, seed):
    from stream_diffusion_transformer_b200 import model
    S = gh * gw + s_txt
    x = torch.from_numpy(zi.make_stream(d, 1, S, seed=seed)).cuda()
    c = torch.from_numpy(zi.make_cond(d, 1, seed=seed)).cuda() if modulated else None
    return model.positions(s_txt, gh, gw), S, x, c


def _noalloc(abi, model, cfg, blk, c, pos, x, S, out):
    abi.call("zi_block_forward_noalloc", ctypes.byref(cfg), ctypes.byref(blk.struct), model._p(c), model._p(pos),
             1, S, model._p(x), model._p(out), model._stream())
    return out


def _same_bits(got, want, what):
    g = got.cpu().numpy()
    w = want.cpu().numpy()
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    assert np.array_equal(g.view(np.uint32), w.view(np.uint32)), \
        f"{what}: {int(np.count_nonzero(g.view(np.uint32) != w.view(np.uint32)))} elements differ"


@pytest.mark.parametrize("width,modulated", [("tiny", True), ("tiny", False), ("full", True)])
def test_noalloc_matches_workspace_entry_point_twice(width, modulated):
    require_gpu()
    if width == "tiny":
        d, s_txt, gh, gw = zi.TINY, 32, 8, 8
    else:
        d, s_txt, gh, gw = FULL1, 32, 16, 16
    abi, model, cfg, blk = _setup(d, modulated, seed=21)
    cases = [_inputs(d, modulated, s_txt, gh, gw, seed=21 + 10 * k) for k in range(2)]
    abi.clear_device_status()
    outs = [_noalloc(abi, model, cfg, blk, c, pos, x, S, torch.empty_like(x)) for pos, S, x, c in cases]
    refs = [model.block_forward(cfg, blk, c, pos, x) for pos, S, x, c in cases]  # caller-provided workspace
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    for k in range(2):
        _same_bits(outs[k], refs[k], f"no-alloc call {k + 1}")


def test_noalloc_small_call_after_a_large_one():
    """A 1,152-token call fills most of the scratch; the 96-token call after it must not
    read any of what the large call left there."""
    require_gpu()
    d = FULL1
    abi, model, cfg, blk = _setup(d, True, seed=23)
    big = _inputs(d, True, 128, 32, 32, seed=23)
    small = _inputs(d, True, 32, 8, 8, seed=24)
    assert abi.block_workspace_size(cfg, 1, big[1]) > 3 * abi.block_workspace_size(cfg, 1, small[1])
    abi.clear_device_status()
    outs = []
    for pos, S, x, c in (big, small):
        outs.append(_noalloc(abi, model, cfg, blk, c, pos, x, S, torch.empty_like(x)))
    refs = [model.block_forward(cfg, blk, c, pos, x) for pos, S, x, c in (big, small)]
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    _same_bits(outs[0], refs[0], "no-alloc 1,152 tokens")
    _same_bits(outs[1], refs[1], "no-alloc 96 tokens after 1,152")


def test_noalloc_calls_leave_free_device_memory_unchanged():
    """After one warm-up call (which looks up the scratch's device address), further
    calls allocate nothing: the device's free memory stays the same."""
    require_gpu()
    d = zi.TINY
    abi, model, cfg, blk = _setup(d, True, seed=25)
    pos, S, x, c = _inputs(d, True, 32, 8, 8, seed=25)
    out = torch.empty_like(x)
    _noalloc(abi, model, cfg, blk, c, pos, x, S, out)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        _noalloc(abi, model, cfg, blk, c, pos, x, S, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    assert abi.device_status() == 0


def test_noalloc_rejects_sizes_beyond_the_scratch():
    require_gpu()
    from stream_diffusion_transformer_b200 import abi, model
    cfg = model.make_config(FULL1)
    assert abi.block_workspace_size(cfg, 1, 2048) > abi.STATIC_SCRATCH_BYTES
    # rejected on sizes alone, before any pointer is looked at or anything is enqueued
    st = abi.lib().zi_block_forward_noalloc(ctypes.byref(cfg), None, None, None, 1, 2048, None, None, None)
    assert st == abi.ZI_ERR_SCRATCH_LIMIT
    assert "fixed scratch" in abi.status_string(st)
