"""GPU parity of the single steps, through the C ABI, against the CPU oracle.

Tolerances: integer outputs (positions, packed weights) bit-exact; fp32
elementwise steps to fp32 rounding; bf16-output GEMM to bf16 rounding of the
output (rel-L2 <= 4e-3, i.e. ~2^-8); attention rel-L2 <= 1e-2 (P is rounded to
bf16 before the PV product, ~2^-9 per weight)."""
import ctypes

import numpy as np
import pytest

from gpu_util import assert_parity, bits_f64, dev_bits, host_f64, rel_l2, require_gpu, torch
import zimage_inputs as zi
from oracle import scheduler_ref as sch, zimage_ref as ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    from stream_diffusion_transformer_b200 import abi
    abi.lib()
    abi.clear_device_status()
    yield
    assert abi.device_status() == 0


@pytest.fixture(scope="module")
def M():
    from stream_diffusion_transformer_b200 import abi, model
    return abi, model


@pytest.mark.parametrize("s_txt,gh,gw", [(32, 64, 64), (128, 32, 32), (512, 128, 128), (1, 1, 1), (7, 3, 5)])
def test_positions_bit_exact(M, s_txt, gh, gw):
    abi, model = M
    got = model.positions(s_txt, gh, gw).cpu().numpy()
    np.testing.assert_array_equal(got, ref.position_ids(s_txt, gh, gw))


def test_rope_table(M):
    abi, model = M
    cfg = abi.config_default()
    pos = model.positions(32, 64, 64)
    tab = model.rope_table(cfg, pos).cpu().numpy().astype(np.float64)
    ang = ref.rope_angles(ref.position_ids(32, 64, 64))
    np.testing.assert_allclose(tab[..., 0], np.cos(ang), rtol=0, atol=2e-7)
    np.testing.assert_allclose(tab[..., 1], np.sin(ang), rtol=0, atol=2e-7)


@pytest.mark.parametrize("cfg_guidance", [None, 4.0])
def test_euler_step(M, cfg_guidance):
    abi, model = M
    rng = np.random.default_rng(0)
    n = 16 * 128 * 128 + 3  # ragged tail
    x = rng.standard_normal(n).astype(np.float32)
    yc = rng.standard_normal(n).astype(np.float32)
    yu = rng.standard_normal(n).astype(np.float32)
    sig = sch.sigmas(8)
    xt = torch.from_numpy(x).cuda()
    model.euler_step(xt, torch.from_numpy(yc).cuda(), None if cfg_guidance is None else torch.from_numpy(yu).cuda(),
                     cfg_guidance or 0.0, sig[2], sig[3])
    y = yc.astype(np.float64) if cfg_guidance is None else sch.cfg_combine(yc.astype(np.float64), yu, cfg_guidance)
    want = sch.euler_step(x.astype(np.float64), y, sig[2], sig[3])
    np.testing.assert_allclose(xt.cpu().numpy(), want, rtol=2e-6, atol=2e-6)


def test_pack_qkv_and_ffn_bit_exact(M):
    abi, model = M
    D, F = 256, 688
    wq, wk, wv = (zi.make_matrix((D, D), 1, i) for i in range(3))
    dq, dk, dv = dev_bits(wq), dev_bits(wk), dev_bits(wv)
    got = model.pack_qkv(dq, dk, dv).view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got, np.concatenate([wq, wk, wv]))
    w1, w3 = zi.make_matrix((F, D), 2, 0), zi.make_matrix((F, D), 2, 1)
    w2 = zi.make_matrix((D, F), 2, 2)
    Fp = abi.ffn_padded(F)
    w13 = torch.empty((2 * Fp, D), dtype=torch.bfloat16, device="cuda")
    w2p = torch.empty((D, Fp), dtype=torch.bfloat16, device="cuda")
    d1, d3, d2 = dev_bits(w1), dev_bits(w3), dev_bits(w2)  # kept alive until the copies ran
    abi.call("zi_pack_ffn", model._p(d1), model._p(d3), model._p(d2), F, D, model._p(w13), model._p(w2p),
             model._stream())
    torch.cuda.synchronize()
    g13 = w13.view(torch.int16).cpu().numpy().view(np.uint16)
    g2 = w2p.view(torch.int16).cpu().numpy().view(np.uint16)
    pad = lambda a: np.concatenate([a, np.zeros((Fp - F, D), np.uint16)])
    want13 = np.stack([pad(w1).reshape(Fp // 128, 128, D), pad(w3).reshape(Fp // 128, 128, D)], 1).reshape(2 * Fp, D)
    np.testing.assert_array_equal(g13, want13)
    np.testing.assert_array_equal(g2, np.concatenate([w2, np.zeros((D, Fp - F), np.uint16)], 1))


@pytest.mark.parametrize("m,n,k", [(1, 256, 64), (96, 768, 256), (127, 256, 128), (129, 512, 192),
                                   (300, 1536, 256), (1152, 3840, 3840), (4128, 1280, 640),
                                   (4128, 3840, 3840), (2000, 2560, 1024), (4128, 3840, 64),
                                   (4128, 11520, 128), (19000, 256, 64), (4128, 3840, 10240),
                                   (8192, 3584, 16384), (32768, 4096, 8192)])
def test_gemm_bf16(M, m, n, k):
    """Covers single tiles, M tails, several waves, and ragged last waves (4128 x 3840:
    495 tiles = 3 x 148 + 51; 19000 x 256: 149 tiles), and the grouped tile walk with a
    partial last group: 4128 x 3840 x 10240 walks groups of 21 and 12 row tiles,
    8192 x 3584 x 16384 groups of 13 row tiles (the last 12), 32768 x 4096 x 8192 groups
    of 13 and 3 column tiles.  The standalone entry point runs
    every tile whole: it has no workspace for the fp32 partials of the K-split tail the
    forward uses, which the block tests cover (test_full_width_block_split_tails_deterministic)."""
    abi, model = M
    a = zi.make_matrix((m, k), 3, 0)
    b = zi.make_matrix((n, k), 3, 1, std=0.05)
    c = model.gemm(dev_bits(a), dev_bits(b))
    torch.cuda.synchronize()
    want = bits_f64(a) @ bits_f64(b).T
    got = host_f64(c)
    assert rel_l2(got, want) <= 4e-3
    assert np.abs(got - want).max() <= 1e-2 * np.abs(want).max() + 1e-6


@pytest.mark.parametrize("m,n,k", [(1, 256, 64), (96, 768, 256), (255, 256, 128), (257, 512, 192),
                                   (300, 1536, 256), (1152, 3840, 3840), (4128, 3840, 3840),
                                   (4128, 20480, 640), (2000, 2560, 1024), (4128, 3840, 64),
                                   (19000, 256, 64), (33792, 768, 128), (4128, 3840, 10240),
                                   (8192, 3584, 16384)])
def test_gemm_bf16_pair(M, m, n, k):
    """The CTA-pair kernel (256 x 256 tiles, B split across the two SMs): single tiles,
    rows past M in either CTA of the last tile pair (255, 257, 4128 rows), fewer tiles than
    pairs, several waves, exact multiples of 256 rows (33,792, the CFG size), and grouped
    tile walks with a partial last group (4128 x 3840 x 10240: 10 + 7 row tiles;
    8192 x 3584 x 16384: 6 + 6 + 2 column tiles)."""
    abi, model = M
    a = zi.make_matrix((m, k), 6, 0)
    b = zi.make_matrix((n, k), 6, 1, std=0.05)
    c = model.gemm(dev_bits(a), dev_bits(b), pair=True)
    torch.cuda.synchronize()
    want = bits_f64(a) @ bits_f64(b).T
    got = host_f64(c)
    assert rel_l2(got, want) <= 4e-3
    assert np.abs(got - want).max() <= 1e-2 * np.abs(want).max() + 1e-6
    # the single-CTA kernel accumulates every output in the same K order: identical bits
    c1 = model.gemm(dev_bits(a), dev_bits(b))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(c.view(torch.int16).cpu().numpy(), c1.view(torch.int16).cpu().numpy())


@pytest.mark.parametrize("batch,seq,heads", [(1, 96, 2), (1, 128, 1), (2, 200, 2), (1, 1152, 4), (1, 33, 3)])
def test_attention(M, batch, seq, heads):
    abi, model = M
    D = heads * 128
    qkv = zi.make_matrix((batch * seq, 3 * D), 4, seq)
    out = model.attention(dev_bits(qkv), batch, seq, heads)
    torch.cuda.synchronize()
    got = host_f64(out).reshape(batch, seq, heads, 128)
    x = bits_f64(qkv).reshape(batch, seq, 3, heads, 128)
    for b in range(batch):
        want = ref.attention(x[b, :, 0], x[b, :, 1], x[b, :, 2])
        assert_parity(got[b], want, rel=1e-2, cos=0.9999, what=f"attention b={b}")


@pytest.mark.parametrize("seq,kv_len", [(300, [1, 77, 300, 129]), (256, [128, 255, 256, 2])])
def test_attention_key_mask(M, seq, kv_len):
    """Per-element key counts (padding masked as keys): one key, a count inside a tile,
    exactly a tile boundary, all keys, one past a boundary; every query row checked."""
    abi, model = M
    heads, batch = 2, len(kv_len)
    D = heads * 128
    qkv = zi.make_matrix((batch * seq, 3 * D), 4, seq + 7)
    lens = torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    out = model.attention(dev_bits(qkv), batch, seq, heads, kv_len=lens)
    torch.cuda.synchronize()
    got = host_f64(out).reshape(batch, seq, heads, 128)
    x = bits_f64(qkv).reshape(batch, seq, 3, heads, 128)
    for b in range(batch):
        valid = np.arange(seq) < kv_len[b]
        want = ref.attention(x[b, :, 0], x[b, :, 1], x[b, :, 2], key_valid=valid)
        assert_parity(got[b], want, rel=1e-2, cos=0.9999, what=f"masked attention b={b} keys={kv_len[b]}")
        if kv_len[b] == 1:  # a single key: every query's output is that key's value row
            np.testing.assert_allclose(got[b], np.broadcast_to(x[b, 0, 2], got[b].shape), rtol=0, atol=0)


def test_attention_sharp_scores(M):
    """Large logits: the running max moves by far more than 2^8 between key tiles."""
    abi, model = M
    seq, heads = 512, 1
    D = 128
    qkv = zi.bf16_bits_to_f32(zi.make_matrix((seq, 3 * D), 5, 0)).reshape(seq, 3, D)
    qkv[:, 0] *= 4.0
    qkv[:, 1] *= np.linspace(0.5, 6.0, seq, dtype=np.float32)[:, None]  # later keys dominate
    bits = zi.f32_to_bf16_bits(qkv.reshape(seq, 3 * D))
    out = model.attention(dev_bits(bits), 1, seq, heads)
    torch.cuda.synchronize()
    x = bits_f64(bits).reshape(seq, 3, 1, 128)
    want = ref.attention(x[:, 0], x[:, 1], x[:, 2])
    assert_parity(host_f64(out).reshape(seq, 1, 128), want, rel=1e-2, cos=0.9999, what="sharp attention")


def test_fma_pipe_exp2_error_bound(M):
    """The softmax's FMA-pipe 2^x (zi_exp2_poly runs the attention kernel's own routine):
    relative error <= 7.5e-5 against fp64 2^x over [-125, 0] on a dense grid plus every
    integer and half-integer (the ends of the Cody-Waite reduction interval) and points
    2^-20 either side of them.  Below -125 (where the reduced result can fall into the
    denormal range) the result is non-negative and at most 2^-124: against a row maximum
    of 2^0 such a probability is zero at the precision P is kept in; a masked key's -inf
    and the -126 clamp are included."""
    abi, model = M
    grid = np.linspace(-125.0, 0.0, 4_000_001)
    ends = -np.arange(0.0, 125.5, 0.5)
    near = np.concatenate([ends + 2.0 ** -20, ends - 2.0 ** -20])
    x = np.concatenate([grid, ends, near[(near >= -125.0) & (near <= 0.0)]]).astype(np.float32)
    low = np.array([-125.25, -125.5, -125.99997, -126.0, -126.5, -127.0, -150.0, -1e4, -np.inf], dtype=np.float32)
    xd = torch.from_numpy(np.concatenate([x, low])).cuda()
    yd = torch.empty_like(xd)
    abi.call("zi_exp2_poly", model._p(xd), model._p(yd), xd.numel(), model._stream())
    torch.cuda.synchronize()
    y = yd.cpu().numpy().astype(np.float64)
    rel = np.abs(y[:len(x)] / np.exp2(x.astype(np.float64)) - 1.0)
    print(f"[exp2] max relative error {rel.max():.3e} at x = {x[np.argmax(rel)]}")
    assert rel.max() <= 7.5e-5
    tail = y[len(x):]
    assert np.all(tail >= 0.0) and np.all(tail <= 2.0 ** -124), tail
    # an odd count exercises the lone last element
    abi.call("zi_exp2_poly", model._p(xd), model._p(yd), 3, model._stream())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(yd[:3].cpu().numpy(), y[:3].astype(np.float32))
