"""zi_block_forward_noalloc: the block forward for callers that cannot allocate.

Some callers cannot hand the library a workspace: a plugin inside a host
program whose memory manager owns all device memory and gives plugins no
allocator, or a latency-critical loop that forbids cudaMalloc after start-up.
For them the library keeps a fixed 128 MiB device scratch array of its own.
This test calls that entry point through the C ABI twice in a row (different
inputs, so the second call runs on scratch the first one left behind) and
checks each result against zi_block_forward given a freshly allocated
workspace, with the block parity bar used elsewhere (rel-L2 <= 2e-2, cosine
>= 0.999).  The file sorts last so a run that stops at the first failure has
already run every other test.
"""
import ctypes
import dataclasses

import numpy as np
import pytest

from gpu_util import assert_parity, require_gpu, torch
import zimage_inputs as zi

pytestmark = pytest.mark.gpu


def _case(d, prefix, modulated, s_txt, gh, gw, seed):
    from stream_diffusion_transformer_b200 import abi, model
    cfg = model.make_config(d)
    bits = zi.make_weights(d, seed=seed, keys=model.block_keys(prefix, modulated))
    blk = model.DeviceBlock(cfg, prefix, bits, modulated, "cuda")
    pos = model.positions(s_txt, gh, gw)
    S = gh * gw + s_txt
    inputs = []
    for k in range(2):
        x = torch.from_numpy(zi.make_stream(d, 1, S, seed=seed + 10 * k)).cuda()
        c = torch.from_numpy(zi.make_cond(d, 1, seed=seed + 10 * k)).cuda() if modulated else None
        inputs.append((x, c))
    return abi, model, cfg, blk, pos, S, inputs


def _noalloc(abi, model, cfg, blk, c, pos, x, S):
    out = torch.empty_like(x)
    abi.call("zi_block_forward_noalloc", ctypes.byref(cfg), ctypes.byref(blk.struct), model._p(c), model._p(pos),
             1, S, model._p(x), model._p(out), model._stream())
    return out


@pytest.mark.parametrize("width,modulated", [("tiny", True), ("tiny", False), ("full", True)])
def test_noalloc_matches_workspace_entry_point_twice(width, modulated):
    require_gpu()
    if width == "tiny":
        d, s_txt, gh, gw = zi.TINY, 32, 8, 8
    else:
        d, s_txt, gh, gw = dataclasses.replace(zi.FULL, n_noise=0, n_ctx=0, n_main=1), 32, 16, 16
    abi, model, cfg, blk, pos, S, inputs = _case(d, "layers.0", modulated, s_txt, gh, gw, seed=21)
    abi.clear_device_status()
    outs = [_noalloc(abi, model, cfg, blk, c, pos, x, S) for x, c in inputs]   # two calls in a row
    refs = [model.block_forward(cfg, blk, c, pos, x) for x, c in inputs]      # caller-provided workspace
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    for k in range(2):
        got = outs[k].cpu().numpy().astype(np.float64)
        want = refs[k].cpu().numpy().astype(np.float64)
        assert_parity(got, want, rel=2e-2, cos=0.999, what=f"no-alloc call {k + 1}")


def test_noalloc_rejects_sizes_beyond_the_scratch():
    require_gpu()
    from stream_diffusion_transformer_b200 import abi, model
    d = dataclasses.replace(zi.FULL, n_noise=0, n_ctx=0, n_main=1)
    cfg = model.make_config(d)
    assert abi.block_workspace_size(cfg, 1, 2048) > abi.STATIC_SCRATCH_BYTES
    # rejected on sizes alone, before any pointer is looked at or anything is enqueued
    st = abi.lib().zi_block_forward_noalloc(ctypes.byref(cfg), None, None, None, 1, 2048, None, None, None)
    assert st == abi.ZI_ERR_SCRATCH_LIMIT
    assert "fixed scratch" in abi.status_string(st)
