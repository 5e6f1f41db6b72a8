"""GPU parity of the e4m3 path (quantiser, e4m3 GEMM, e4m3 blocks and model) against
the oracle's e4m3 statement (oracle/fp8_ref.py).

Bars.  Quantised codes and scales: bit-exact (both sides decide in fp32 from the
same fp32 input).  e4m3 GEMM: within bf16 output rounding of the exact product
of the decoded operands (rel-L2 <= 4e-3).  e4m3 blocks: rel-L2 <= 3e-2, cosine
>= 0.999, update cosine >= 0.99; e4m3 model: cosine >= 0.995, rel-L2 <= 3e-2.

Why the block bar is looser than the bf16 block's 2e-2: inside a block the GPU's
activations differ from the oracle's by the bf16 path's own error eps (about
5e-3 after attention).  A quantiser turns that into code flips: a fraction of
about eps / 2^-4 of the codes round the other way, each by one step (2^-4
relative), so the quantised activation differs by about sqrt(eps * 2^-4) ~ 1.8e-2
relative, which the projection carries into the block update.  With every
projection in e4m3 ("all") a block has four quantisers (h, attention output,
h2, SwiGLU output), each adding such a term, and the unmodulated block (gate 1)
passes its whole update to the output: rel-L2 <= 6e-2 and cosine >= 0.998 there."""
import dataclasses

import numpy as np
import pytest

from gpu_util import assert_parity, bits_f64, dev_bits, host_f64, require_gpu, torch
import zimage_inputs as zi
from oracle import fp8_ref as f8
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


def _edge_rows(K=256):
    """Rows built to exercise the rounding: amax exactly 448 (so the scaled value is
    the input itself) with entries on e4m3 midpoints, subnormal midpoints, signed
    zeros and saturating neighbours; a zero row; a row of tiny values; a bf16-like row."""
    rng = np.random.default_rng(0)
    r0 = np.zeros(K, np.float32)
    mids = [1.0625, 1.1875, 1.3125, 2.125, 240.0 + 8.0, 1.5 * 2 ** -9, 0.5 * 2 ** -9, 2.5 * 2 ** -9,
            -1.0625, -0.5 * 2 ** -9, -0.0, 0.0, 447.0, 440.0, 1e-12, -1e-12]
    r0[:len(mids)] = mids
    r0[-1] = 448.0
    r1 = np.zeros(K, np.float32)
    r2 = (rng.standard_normal(K) * 1e-30).astype(np.float32)
    r3 = rng.standard_normal(K).astype(np.float32) * np.float32(3.7)
    r4 = (rng.standard_normal(K) * np.exp2(rng.uniform(-20, 20, K))).astype(np.float32)
    return np.stack([r0, r1, r2, r3, r4])


def test_quantizer_bit_exact_fp32_and_bf16():
    from stream_diffusion_transformer_b200 import model
    x = _edge_rows()
    x = np.concatenate([x, zi.bf16_bits_to_f32(zi.make_matrix((37, 256), 4, 11))], axis=0)
    q, s = model.quantize_rows_e4m3(torch.from_numpy(x).cuda())
    want_q, want_s = f8.quantize_rows(x)
    np.testing.assert_array_equal(q.cpu().numpy(), want_q)
    np.testing.assert_array_equal(s.cpu().numpy(), want_s)
    bits = zi.make_matrix((64, 3840), 4, 12)
    q, s = model.quantize_rows_e4m3(dev_bits(bits))
    want_q, want_s = f8.quantize_rows(zi.bf16_bits_to_f32(bits))
    np.testing.assert_array_equal(q.cpu().numpy(), want_q)
    np.testing.assert_array_equal(s.cpu().numpy(), want_s)


@pytest.mark.parametrize("M,N,K", [(1, 256, 128), (300, 512, 384), (129, 768, 3840)])
def test_gemm_e4m3(M, N, K):
    from stream_diffusion_transformer_b200 import model
    rng = np.random.default_rng(M + N + K)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    a = finite[rng.integers(0, len(finite), (M, K))]
    b = finite[rng.integers(0, len(finite), (N, K))]
    sa = (rng.uniform(0.5, 2.0, M) * 2.0 ** -6).astype(np.float32)
    sb = (rng.uniform(0.5, 2.0, N) * 2.0 ** -5).astype(np.float32)
    t = lambda v: torch.from_numpy(v).cuda()
    out = model.gemm_e4m3(t(a), t(sa), t(b), t(sb))
    torch.cuda.synchronize()
    want = f8.dequantize_rows(a, sa) @ f8.dequantize_rows(b, sb).T
    assert_parity(host_f64(out), want, rel=4e-3, cos=0.99999, what=f"e4m3 GEMM {M}x{N}x{K}")


def test_gemm_e4m3_full_projection_sampled_rows():
    """The QKV projection's shape at 4,128 tokens (M=4128, N=11520, K=3840) from
    quantised activations and weights, checked on sampled rows."""
    from stream_diffusion_transformer_b200 import model
    h = zi.make_stream(zi.FULL, 1, 4128, seed=13)[0] * np.float32(6.0)
    w = zi.make_matrix((11520, 3840), 4, 13)
    hq, hs = model.quantize_rows_e4m3(torch.from_numpy(np.ascontiguousarray(h)).cuda())
    wq, ws = model.quantize_rows_e4m3(dev_bits(w))
    out = host_f64(model.gemm_e4m3(hq, hs, wq, ws))
    rows = np.array([0, 1, 127, 128, 2047, 4095, 4096, 4127])
    want_q, want_s = f8.quantize_rows(h[rows])
    wq_o, ws_o = f8.quantize_rows(zi.bf16_bits_to_f32(w))
    want = f8.dequantize_rows(want_q, want_s) @ f8.dequantize_rows(wq_o, ws_o).T
    assert_parity(out[rows], want, rel=4e-3, cos=0.99999, what="e4m3 GEMM 4128x11520x3840 (sampled rows)")


def _run_fp8_block(d, prefix, modulated, s_txt, gh, gw, seed, twice=False, mode=True):
    from stream_diffusion_transformer_b200 import model
    cfg = model.make_config(d)
    bits = zi.make_weights(d, seed=seed, keys=model.block_keys(prefix, modulated), threads=8)
    S = gh * gw + s_txt
    x = zi.make_stream(d, 1, S, seed=seed)
    c = zi.make_cond(d, 1, seed=seed) if modulated else None
    blk = model.DeviceBlock(cfg, prefix, bits, modulated, "cuda", fp8=mode)
    pos = model.positions(s_txt, gh, gw)
    xt = torch.from_numpy(x).cuda()
    ct = None if c is None else torch.from_numpy(c).cuda()
    got = model.block_forward(cfg, blk, ct, pos, xt).cpu().numpy()
    if twice:
        np.testing.assert_array_equal(model.block_forward(cfg, blk, ct, pos, xt).cpu().numpy(), got)
    W = ref.Weights(bits)
    ang = ref.rope_angles(ref.position_ids(s_txt, gh, gw), d.rope_axes)
    x0 = x[0].astype(np.float64)
    cc = None if c is None else c[0].astype(np.float64)
    want = f8.block_forward(x0, W, prefix, d, ang, cc, all=mode == "all")
    tag = "e4m3-all" if mode == "all" else "e4m3"
    rel_bar, cos_bar = (6e-2, 0.998) if mode == "all" else (3e-2, 0.999)
    assert_parity(got[0], want, rel=rel_bar, cos=cos_bar, what=f"{tag} {prefix} {S} tokens")
    assert_parity(got[0] - x0, want - x0, rel=1.0, cos=0.99, what=f"{tag} {prefix} {S} tokens update")
    bf16 = ref.block_forward(x0, W, prefix, d, ang, cc)
    r = np.linalg.norm((want - x0) - (bf16 - x0)) / np.linalg.norm(bf16 - x0)
    print(f"[fp8] oracle e4m3 vs bf16 block update: rel-L2 {r:.3e}")


@pytest.mark.parametrize("modulated", [True, False])
def test_tiny_block_e4m3(modulated):
    _run_fp8_block(zi.TINY, "layers.0", modulated, 32, 8, 8, seed=21)


def test_full_width_block_e4m3_split_tails():
    """456 tokens: every GEMM ends in a K-split ragged wave; run twice, bit-identical."""
    d = dataclasses.replace(zi.FULL, n_noise=0, n_ctx=0, n_main=1)
    _run_fp8_block(d, "layers.0", True, 200, 16, 16, seed=22, twice=True)


def test_full_width_block_e4m3_1152_tokens():
    d = dataclasses.replace(zi.FULL, n_noise=0, n_ctx=0, n_main=1)
    _run_fp8_block(d, "layers.0", True, 128, 32, 32, seed=23)


def test_full_width_model_e4m3():
    """Full width, 1 + 1 + 2 blocks, 256 + 32 tokens, every block in e4m3."""
    from stream_diffusion_transformer_b200 import model
    d = dataclasses.replace(zi.FULL, n_noise=1, n_ctx=1, n_main=2)
    bits = zi.make_weights(d, seed=24, threads=8)
    dit = model.DiT(model.make_config(d), lambda keys: {k: bits[k] for k in keys}, fp8=True)
    lat = zi.make_latent(d, 1, 32, 32, seed=24)
    txt = zi.make_text(d, 1, 32, seed=24)
    t = np.array([0.25], dtype=np.float32)
    out = dit.forward(torch.from_numpy(lat).cuda(), torch.from_numpy(t).cuda(),
                      torch.from_numpy(txt.view(np.int16)).cuda().view(torch.bfloat16))
    torch.cuda.synchronize()
    W = ref.Weights(bits)
    args = (lat.astype(np.float64), t.astype(np.float64), zi.bf16_bits_to_f32(txt).astype(np.float64), W, d)
    want = f8.model_forward(*args)
    assert_parity(out.cpu().numpy(), want, rel=3e-2, cos=0.995, what="e4m3 full-width shallow model")
    bf16 = ref.model_forward(*args)
    r = np.linalg.norm(want - bf16) / np.linalg.norm(bf16)
    print(f"[fp8] oracle e4m3 vs bf16 model output: rel-L2 {r:.3e}")


@pytest.mark.parametrize("modulated", [True, False])
def test_tiny_block_all_e4m3(modulated):
    _run_fp8_block(zi.TINY, "layers.0", modulated, 32, 8, 8, seed=31, mode="all")


def test_full_width_block_all_e4m3_split_tails():
    """Every projection in e4m3 (attention and SwiGLU outputs quantised per row by an
    extra pass); 456 tokens with K-split tails, run twice, bit-identical."""
    d = dataclasses.replace(zi.FULL, n_noise=0, n_ctx=0, n_main=1)
    _run_fp8_block(d, "layers.0", True, 200, 16, 16, seed=32, twice=True, mode="all")


def test_full_width_model_all_e4m3():
    from stream_diffusion_transformer_b200 import model
    d = dataclasses.replace(zi.FULL, n_noise=1, n_ctx=1, n_main=2)
    bits = zi.make_weights(d, seed=34, threads=8)
    dit = model.DiT(model.make_config(d), lambda keys: {k: bits[k] for k in keys}, fp8="all")
    lat = zi.make_latent(d, 1, 32, 32, seed=34)
    txt = zi.make_text(d, 1, 32, seed=34)
    t = np.array([0.6], dtype=np.float32)
    out = dit.forward(torch.from_numpy(lat).cuda(), torch.from_numpy(t).cuda(),
                      torch.from_numpy(txt.view(np.int16)).cuda().view(torch.bfloat16))
    torch.cuda.synchronize()
    W = ref.Weights(bits)
    args = (lat.astype(np.float64), t.astype(np.float64), zi.bf16_bits_to_f32(txt).astype(np.float64), W, d)
    want = f8.model_forward(*args, all=True)
    assert_parity(out.cpu().numpy(), want, rel=3e-2, cos=0.995, what="e4m3-all full-width shallow model")
    bf16 = ref.model_forward(*args)
    r = np.linalg.norm(want - bf16) / np.linalg.norm(bf16)
    print(f"[fp8] oracle e4m3-all vs bf16 model output: rel-L2 {r:.3e}")


@pytest.mark.parametrize("mode", [True, "all"])
def test_with_e4m3_matches_fresh_e4m3_model(mode):
    """DiT.with_e4m3 quantises the resident bf16 weights of a bf16 model; its forward is
    bit-identical to a model built in e4m3 from the same weights, and the bf16 model it
    came from is left as it was."""
    from stream_diffusion_transformer_b200 import model
    d = dataclasses.replace(zi.FULL, n_noise=1, n_ctx=1, n_main=1)
    bits = zi.make_weights(d, seed=35, threads=8)
    fetch = lambda keys: {k: bits[k] for k in keys}
    base = model.DiT(model.make_config(d), fetch)
    fresh = model.DiT(model.make_config(d), fetch, fp8=mode)
    lat = torch.from_numpy(zi.make_latent(d, 1, 16, 16, seed=35)).cuda()
    txt = torch.from_numpy(zi.make_text(d, 1, 32, seed=35).view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.tensor([0.4], dtype=torch.float32, device="cuda")
    y_base = base.forward(lat, t, txt).cpu().numpy()
    derived = base.with_e4m3(mode)
    y_derived = derived.forward(lat, t, txt).cpu().numpy()
    y_fresh = fresh.forward(lat, t, txt).cpu().numpy()
    np.testing.assert_array_equal(y_derived, y_fresh)
    np.testing.assert_array_equal(base.forward(lat, t, txt).cpu().numpy(), y_base)
    assert not np.array_equal(y_derived, y_base)
