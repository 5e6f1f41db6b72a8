"""GPU parity of zi_block_forward against the CPU oracle's block.

Bars: block output rel-L2 <= 2e-2 and cosine >= 0.999 against the oracle
(fp64, same bf16 weights); the block's update x_out - x_in cosine >= 0.99, so
a broken sublayer cannot hide behind the residual."""
import dataclasses

import numpy as np
import pytest

from gpu_util import assert_parity, require_gpu, torch
import zimage_inputs as zi
from oracle import zimage_ref as ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    from stream_diffusion_transformer_b200 import abi
    abi.lib()
    abi.clear_device_status()
    yield
    assert abi.device_status() == 0


def run_block(d, prefix, modulated, batch, s_txt, gh, gw, seed, in_place=False):
    from stream_diffusion_transformer_b200 import model
    cfg = model.make_config(d)
    keys = model.block_keys(prefix, modulated)
    bits = zi.make_weights(d, seed=seed, keys=keys)
    S = gh * gw + s_txt
    x = zi.make_stream(d, batch, S, seed=seed)
    c = zi.make_cond(d, batch, seed=seed) if modulated else None
    blk = model.DeviceBlock(cfg, prefix, bits, modulated, "cuda")
    pos = model.positions(s_txt, gh, gw)
    xt = torch.from_numpy(x).cuda()
    ct = None if c is None else torch.from_numpy(c).cuda()
    out = model.block_forward(cfg, blk, ct, pos, xt, xt if in_place else None)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    W = ref.Weights(bits)
    ang = ref.rope_angles(ref.position_ids(s_txt, gh, gw), d.rope_axes)
    for b in range(batch):
        want = ref.block_forward(x[b].astype(np.float64), W, prefix, d, ang, None if c is None else c[b].astype(np.float64))
        assert_parity(got[b], want, rel=2e-2, cos=0.999, what=f"{prefix} b={b}")
        assert_parity(got[b] - x[b], want - x[b], rel=1.0, cos=0.99, what=f"{prefix} delta b={b}")


@pytest.mark.parametrize("modulated", [True, False])
def test_tiny_block(modulated):
    """hidden 256 (2 heads), FFN 688 (padded to 768 inside), 64 image + 32 text tokens."""
    run_block(zi.TINY, "layers.0", modulated, 1, 32, 8, 8, seed=1)


def test_tiny_block_batch_ragged_in_place():
    """batch 2, 5 x 7 image tokens + 17 text tokens: ragged query/key tiles, in-place update."""
    run_block(zi.TINY, "layers.0", True, 2, 17, 5, 7, seed=2, in_place=True)


def test_full_width_block_1152_tokens():
    """One main block at full width: 512x512 image (1,024 tokens) + 128 text tokens."""
    run_block(dataclasses.replace(zi.FULL, n_noise=0, n_ctx=0, n_main=1), "layers.0", True, 1, 128, 32, 32, seed=3)


def test_full_width_block_split_tails_deterministic():
    """456 tokens (16 x 16 image + 200 text; 4 row tiles, the last ragged): every GEMM of
    the block ends in a ragged wave cut along K (QKV and FFN-up in 4 pieces, out-proj
    and FFN-down in 2), finished by whichever piece arrives last.  Parity with the
    oracle, and two runs bit-identical (partials are added in a fixed order)."""
    from stream_diffusion_transformer_b200 import model
    d = dataclasses.replace(zi.FULL, n_noise=0, n_ctx=0, n_main=1)
    cfg = model.make_config(d)
    keys = model.block_keys("layers.0", True)
    bits = zi.make_weights(d, seed=8, keys=keys, threads=8)
    s_txt, gh, gw = 200, 16, 16
    S = gh * gw + s_txt
    x = zi.make_stream(d, 1, S, seed=8)
    c = zi.make_cond(d, 1, seed=8)
    blk = model.DeviceBlock(cfg, "layers.0", bits, True, "cuda")
    pos = model.positions(s_txt, gh, gw)
    xt, ct = torch.from_numpy(x).cuda(), torch.from_numpy(c).cuda()
    out1 = model.block_forward(cfg, blk, ct, pos, xt).cpu().numpy()
    out2 = model.block_forward(cfg, blk, ct, pos, xt).cpu().numpy()
    np.testing.assert_array_equal(out1, out2)
    W = ref.Weights(bits)
    ang = ref.rope_angles(ref.position_ids(s_txt, gh, gw), d.rope_axes)
    want = ref.block_forward(x[0].astype(np.float64), W, "layers.0", d, ang, c[0].astype(np.float64))
    assert_parity(out1[0], want, rel=2e-2, cos=0.999, what="split-tail block")
    assert_parity(out1[0] - x[0], want - x[0], rel=1.0, cos=0.99, what="split-tail block delta")


def test_full_width_unmodulated_text_block():
    """A context-refiner-shaped block on 32 text tokens only (a single partial tile)."""
    d = dataclasses.replace(zi.FULL, n_noise=0, n_ctx=1, n_main=1)
    run_block(d, "context_refiner.0", False, 1, 32, 0, 0, seed=4)


@pytest.mark.slow
def test_full_width_block_cfg_batch2_16896_tokens():
    """A main block of the CFG workload: batch 2 x (16,384 image + 512 text) tokens, on
    sampled rows (keys and values over the whole 16,896-token sequence of each element)."""
    from stream_diffusion_transformer_b200 import model
    d = dataclasses.replace(zi.FULL, n_noise=0, n_ctx=0, n_main=1)
    cfg = model.make_config(d)
    keys = model.block_keys("layers.0", True)
    bits = zi.make_weights(d, seed=7, keys=keys, threads=8)
    s_txt, gh, gw = 512, 128, 128
    S = gh * gw + s_txt
    x = zi.make_stream(d, 2, S, seed=7)
    c = zi.make_cond(d, 2, seed=7)
    blk = model.DeviceBlock(cfg, "layers.0", bits, True, "cuda")
    pos = model.positions(s_txt, gh, gw)
    out = model.block_forward(cfg, blk, torch.from_numpy(c).cuda(), pos, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    W = ref.Weights(bits)
    ang = ref.rope_angles(ref.position_ids(s_txt, gh, gw), d.rope_axes)
    rows = np.unique(np.concatenate([[0, 127, 128, 8191, 16383, 16384, S - 1],
                                     np.random.default_rng(7).integers(0, S, 17)]))
    for b in range(2):
        want = ref.block_forward_rows(x[b].astype(np.float64), W, "layers.0", d, ang, c[b].astype(np.float64), rows)
        assert_parity(got[b][rows], want, rel=2e-2, cos=0.999, what=f"CFG-size block b={b}")
        assert_parity(got[b][rows] - x[b][rows], want - x[b][rows], rel=1.0, cos=0.99,
                      what=f"CFG-size block delta b={b}")
