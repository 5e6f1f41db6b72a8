"""Pins of the oracle's block, final layer and full forward."""
import dataclasses
import math

import numpy as np
import pytest

import zimage_inputs as zi
from oracle import brute, zimage_ref as ref

# One head of 128 keeps the brute-force block cheap while using the real RoPE axes.
SMALL = zi.Dims(dim=128, heads=1, ffn=64, n_noise=0, n_ctx=0, n_main=1)


def _weights(d, seed=0):
    return zi.make_weights(d, seed=seed)


def _scaled(bits, key, factor):
    """Copy of a bits dict with one tensor multiplied by a power of two (exact in bf16)."""
    out = dict(bits)
    out[key] = zi.f32_to_bf16_bits(zi.bf16_bits_to_f32(bits[key]) * np.float32(factor))
    return out


def _assert_close_to_scale(a, b, tol=1e-5):
    """max |a - b| <= tol * max |b| (an error bound relative to the output's scale)."""
    assert np.abs(a - b).max() <= tol * np.abs(b).max()


def _brute_block(x, W, prefix, d, pos, c):
    """The block restated with scalar loops and explicit rotation matrices."""
    S, D = x.shape
    w = lambda k: W(k).tolist()
    a = f"{prefix}.attention"
    if c is not None:
        m = brute.matmul_bt([list(c)], w(f"{prefix}.adaLN_modulation.weight"))[0]
        b = W(f"{prefix}.adaLN_modulation.bias")
        m = [m[i] + b[i] for i in range(4 * D)]
        sc1, g1 = m[0:D], [math.tanh(v) for v in m[D:2 * D]]
        sc2, g2 = m[2 * D:3 * D], [math.tanh(v) for v in m[3 * D:4 * D]]
    else:
        sc1 = sc2 = [0.0] * D
        g1 = g2 = [1.0] * D
    xs = x.tolist()
    h = [[v * (1 + sc1[i]) for i, v in enumerate(brute.rms_norm_row(r, w(f"{prefix}.attention_norm1.weight"), 1e-5))] for r in xs]
    q = brute.matmul_bt(h, w(f"{a}.to_q.weight"))
    k = brute.matmul_bt(h, w(f"{a}.to_k.weight"))
    v = brute.matmul_bt(h, w(f"{a}.to_v.weight"))
    hd = d.head_dim
    att = [[0.0] * D for _ in range(S)]
    for hh in range(d.heads):
        sl = slice(hh * hd, (hh + 1) * hd)
        qh = [np.array(brute.rms_norm_row(q[s][sl], w(f"{a}.norm_q.weight"), 1e-5)) for s in range(S)]
        kh = [np.array(brute.rms_norm_row(k[s][sl], w(f"{a}.norm_k.weight"), 1e-5)) for s in range(S)]
        qh = [(brute.rope_matrix(list(pos[s])) @ qh[s]).tolist() for s in range(S)]
        kh = [(brute.rope_matrix(list(pos[s])) @ kh[s]).tolist() for s in range(S)]
        vh = [v[s][sl] for s in range(S)]
        oh = brute.attention_head(qh, kh, vh)
        for s in range(S):
            att[s][sl] = oh[s]
    o = brute.matmul_bt(att, w(f"{a}.to_out.weight"))
    on = [brute.rms_norm_row(r, w(f"{prefix}.attention_norm2.weight"), 1e-5) for r in o]
    x1 = [[xs[s][i] + g1[i] * on[s][i] for i in range(D)] for s in range(S)]
    h2 = [[v * (1 + sc2[i]) for i, v in enumerate(brute.rms_norm_row(r, w(f"{prefix}.ffn_norm1.weight"), 1e-5))] for r in x1]
    ff = f"{prefix}.feed_forward"
    u1 = brute.matmul_bt(h2, w(f"{ff}.w1.weight"))
    u3 = brute.matmul_bt(h2, w(f"{ff}.w3.weight"))
    u = [[u1[s][j] / (1 + math.exp(-u1[s][j])) * u3[s][j] for j in range(d.ffn)] for s in range(S)]
    f = brute.matmul_bt(u, w(f"{ff}.w2.weight"))
    fn = [brute.rms_norm_row(r, w(f"{prefix}.ffn_norm2.weight"), 1e-5) for r in f]
    return np.array([[x1[s][i] + g2[i] * fn[s][i] for i in range(D)] for s in range(S)])


@pytest.mark.parametrize("modulated", [True, False])
def test_block_matches_brute_force(modulated):
    d = SMALL
    W = ref.Weights(_weights(d, seed=11))
    rng = np.random.default_rng(11)
    S = 6
    x = rng.standard_normal((S, d.dim)) * 0.3
    c = rng.standard_normal(d.ada_dim) * 0.5 if modulated else None
    pos = np.array(brute.position_ids_loop(2, 2, 2))
    got = ref.block_forward(x, W, "layers.0", d, ref.rope_angles(pos), c)
    want = _brute_block(x, W, "layers.0", d, pos, c)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-11)


def _block_setup(d=zi.TINY, seed=5, S=12):
    bits = _weights(d, seed)
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((S, d.dim)) * 0.16
    c = rng.standard_normal(d.ada_dim) * 0.07
    ang = ref.rope_angles(ref.position_ids(4, 2, 4))
    return bits, x, c, ang


@pytest.mark.parametrize("modulated", [True, False])
def test_block_rows_matches_block(modulated):
    """The sampled-row form used at full size equals the whole block at those rows."""
    d = zi.TINY
    bits, x, c, ang = _block_setup(d, S=12)
    W = ref.Weights(bits)
    cc = c if modulated else None
    rows = np.array([0, 5, 11, 7])
    full = ref.block_forward(x, W, "layers.0", d, ang, cc)
    np.testing.assert_allclose(ref.block_forward_rows(x, W, "layers.0", d, ang, cc, rows), full[rows],
                               rtol=1e-12, atol=1e-14)


def test_zero_modulation_gives_identity_block():
    """tanh(0) = 0 gates both residual updates off."""
    d = zi.TINY
    bits, x, c, ang = _block_setup(d)
    bits = dict(bits)
    for k in ("layers.0.adaLN_modulation.weight", "layers.0.adaLN_modulation.bias"):
        bits[k] = np.zeros_like(bits[k])
    y = ref.block_forward(x, ref.Weights(bits), "layers.0", d, ang, c)
    np.testing.assert_array_equal(y, x)


def test_scale_minus_one_silences_both_sublayers():
    """(1 + scale) = 0 zeroes the sublayer inputs, so the block returns x even with open gates."""
    d = zi.TINY
    D = d.dim
    bits, x, c, ang = _block_setup(d)
    bits = dict(bits)
    bits["layers.0.adaLN_modulation.weight"] = np.zeros_like(bits["layers.0.adaLN_modulation.weight"])
    b = np.zeros(4 * D, dtype=np.float32)
    b[0:D] = -1.0
    b[2 * D:3 * D] = -1.0
    b[D:2 * D] = 0.5
    b[3 * D:] = 0.5
    bits["layers.0.adaLN_modulation.bias"] = zi.f32_to_bf16_bits(b)
    y = ref.block_forward(x, ref.Weights(bits), "layers.0", d, ang, c)
    np.testing.assert_allclose(y, x, rtol=0, atol=1e-12)


@pytest.mark.parametrize("modulated", [True, False])
def test_post_norm_makes_output_rescaling_exact(modulated):
    """z-image-turbo-mnn card, "Conversion details": to_out and w2 outputs feed an
    RMSNorm, so to_out / 64 and (w3 / 64, w2 * 64) leave the block output unchanged.

    The invariance is exact up to the norm's eps, so the base weights put the two
    projections' outputs well above it (x 2^12, exact in bf16), as the real model's
    large activations do.
    """
    d = zi.TINY
    bits, x, c, ang = _block_setup(d)
    bits = _scaled(bits, "layers.0.attention.to_out.weight", 2.0 ** 12)
    bits = _scaled(bits, "layers.0.feed_forward.w2.weight", 2.0 ** 12)
    cc = c if modulated else None
    base = ref.block_forward(x, ref.Weights(bits), "layers.0", d, ang, cc)
    b1 = _scaled(bits, "layers.0.attention.to_out.weight", 1 / 64)
    b1 = _scaled(b1, "layers.0.feed_forward.w3.weight", 1 / 64)
    b1 = _scaled(b1, "layers.0.feed_forward.w2.weight", 64.0)
    _assert_close_to_scale(ref.block_forward(x, ref.Weights(b1), "layers.0", d, ang, cc), base)
    b2 = _scaled(bits, "layers.0.feed_forward.w2.weight", 1 / 64)
    _assert_close_to_scale(ref.block_forward(x, ref.Weights(b2), "layers.0", d, ang, cc), base)
    # to_v acts linearly through attention and to_out, so the same norm absorbs it;
    # w1 feeds the SiLU, so rescaling it changes the output
    for key in ("layers.0.attention.to_v.weight",):
        _assert_close_to_scale(ref.block_forward(x, ref.Weights(_scaled(bits, key, 1 / 64)), "layers.0", d, ang, cc), base)
    b3 = _scaled(bits, "layers.0.feed_forward.w1.weight", 1 / 64)
    assert np.abs(ref.block_forward(x, ref.Weights(b3), "layers.0", d, ang, cc) - base).max() > 1e-3


def test_block_is_permutation_equivariant():
    """Unmasked attention with per-token positions: the order [image; text] is immaterial."""
    d = zi.TINY
    bits, x, c, ang = _block_setup(d)
    W = ref.Weights(bits)
    perm = np.random.default_rng(9).permutation(x.shape[0])
    y = ref.block_forward(x, W, "layers.0", d, ang, c)
    yp = ref.block_forward(x[perm], W, "layers.0", d, ang[perm], c)
    np.testing.assert_allclose(yp, y[perm], rtol=1e-10, atol=1e-12)


def test_final_layer_is_shift_and_scale_invariant():
    d = zi.TINY
    bits = _weights(d, 2)
    W = ref.Weights(bits)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((8, d.dim))
    c = rng.standard_normal(d.ada_dim) * 0.07
    y = ref.final_layer(x, W, c)
    np.testing.assert_allclose(ref.final_layer(3.0 * x + 0.7, W, c), y, rtol=1e-5, atol=1e-6)
    assert y.shape == (8, 64)


def test_text_features_enter_through_rms_norm():
    """cap_embedder starts with RMSNorm: scaling all text features leaves the output unchanged."""
    d = zi.TINY_R
    W = ref.Weights(_weights(d, 4))
    lat = zi.make_latent(d, 1, 4, 4, seed=4)
    txt = zi.bf16_bits_to_f32(zi.make_text(d, 1, 3, seed=4)).astype(np.float64)
    t = np.array([0.3])
    y = ref.model_forward(lat, t, txt, W, d)
    _assert_close_to_scale(ref.model_forward(lat, t, 4.0 * txt, W, d), y)


def test_batch_elements_are_independent():
    d = zi.TINY_R
    W = ref.Weights(_weights(d, 6))
    lat = zi.make_latent(d, 2, 4, 6, seed=6)
    txt = zi.bf16_bits_to_f32(zi.make_text(d, 2, 5, seed=6))
    t = np.array([0.25, 0.8])
    y = ref.model_forward(lat, t, txt, W, d)
    y1 = ref.model_forward(lat[1:], t[1:], txt[1:], W, d)
    np.testing.assert_allclose(y[1:], y1, rtol=1e-12, atol=1e-14)


def test_trace_records_every_block():
    d = zi.TINY_R
    W = ref.Weights(_weights(d, 7))
    lat = zi.make_latent(d, 1, 4, 4, seed=7)
    txt = zi.bf16_bits_to_f32(zi.make_text(d, 1, 3, seed=7))
    tr = []
    ref.model_forward(lat, np.array([0.5]), txt, W, d, trace=tr)
    assert [t.shape for t in tr] == [(4, 256), (3, 256), (7, 256)]


def test_padding_is_invisible_with_the_key_mask():
    """Variable-length text: element 1 padded from 3 to 7 text tokens (pad rows hold
    cap_pad_token, masked as keys) gives the output of running it unpadded."""
    d = zi.TINY_R
    W = ref.Weights(_weights(d, 8))
    lat = zi.make_latent(d, 2, 4, 6, seed=8).astype(np.float64)
    txt = zi.bf16_bits_to_f32(zi.make_text(d, 2, 7, seed=8)).astype(np.float64)
    t = np.array([0.4, 0.7])
    lens = np.array([7, 3])
    padded = ref.model_forward(lat, t, txt, W, d, txt_len=lens)
    full0 = ref.model_forward(lat[:1], t[:1], txt[:1], W, d)
    short1 = ref.model_forward(lat[1:], t[1:], txt[1:, :3], W, d)
    np.testing.assert_allclose(padded[:1], full0, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(padded[1:], short1, rtol=1e-10, atol=1e-12)


def test_pad_token_value_and_pad_features_do_not_leak():
    d = zi.TINY_R
    bits = _weights(d, 9)
    lat = zi.make_latent(d, 1, 4, 4, seed=9).astype(np.float64)
    txt = zi.bf16_bits_to_f32(zi.make_text(d, 1, 6, seed=9)).astype(np.float64)
    t = np.array([0.5])
    lens = np.array([2])
    base = ref.model_forward(lat, t, txt, ref.Weights(bits), d, txt_len=lens)
    txt2 = txt.copy()
    txt2[:, 2:] *= -3.0
    b2 = dict(bits)
    b2["cap_pad_token"] = zi.f32_to_bf16_bits(zi.bf16_bits_to_f32(bits["cap_pad_token"]) * np.float32(5.0))
    np.testing.assert_allclose(ref.model_forward(lat, t, txt2, ref.Weights(b2), d, txt_len=lens), base,
                               rtol=1e-10, atol=1e-12)
    # without the key mask the pads would change the image tokens
    unmasked = ref.model_forward(lat, t, txt, ref.Weights(bits), d)
    assert np.abs(unmasked - base).max() > 1e-4


# ------------------------------------------------------------------ timestep MLP and final layer
# The timestep is passed to the model as 1 - sigma' (z-image-turbo-mnn card, "Scheduler") and
# scaled by 1000 before a [cos, sin] sinusoid and the 256 -> 1024 -> SiLU -> 256 MLP (readings
# of the same card's "Scheduler" and of the parameter count); the final layer is
# LayerNorm(eps 1e-6, no affine) x (1 + Linear(SiLU(c))) -> Linear (H3ddle page, "What was
# changed, and why": two small linears, final_layer.linear [64, 3840]).

def _bits_of(arr):
    """Exact small values (all representable in bf16) as bf16 bits."""
    b = zi.f32_to_bf16_bits(np.asarray(arr, dtype=np.float32))
    assert np.array_equal(zi.bf16_bits_to_f32(b), np.asarray(arr, dtype=np.float32))
    return b


def _silu(v):
    return v / (1.0 + math.exp(-v))


@pytest.mark.parametrize("t", [0.0, 0.3, 0.875])
def test_t_embed_matches_brute_force(t):
    d = zi.TINY
    W = ref.Weights(_weights(d, 12))
    got = ref.t_embed(np.array([t]), W)[0]
    want = brute.t_embed_loop(t, W("t_embedder.linear1.weight").tolist(), W("t_embedder.linear1.bias").tolist(),
                              W("t_embedder.linear2.weight").tolist(), W("t_embedder.linear2.bias").tolist())
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-13)


def test_t_embed_closed_form():
    """Selector weights make each output a hand-computable function of t:
    c0 = 2 SiLU(cos(1000 t)), c1 = 2 SiLU(sin(1000 t)), c2 = 2 SiLU(cos(10 t))
    (f_64 = 10000^(-1/2) = 1/100), c3 = 2 SiLU(sin(10 t)), c4 = SiLU(b1_4) with b1_4 = 0.5,
    c5 = b2_5 = 0.25, every other output 0."""
    d = zi.TINY
    w1 = np.zeros((d.t_mid, d.t_freq), np.float32)
    w1[0, 0] = w1[1, 128] = w1[2, 64] = w1[3, 192] = 1.0
    b1 = np.zeros(d.t_mid, np.float32)
    b1[4] = 0.5
    w2 = np.zeros((d.ada_dim, d.t_mid), np.float32)
    for i in range(4):
        w2[i, i] = 2.0
    w2[4, 4] = 1.0
    b2 = np.zeros(d.ada_dim, np.float32)
    b2[5] = 0.25
    W = ref.Weights({"t_embedder.linear1.weight": _bits_of(w1), "t_embedder.linear1.bias": _bits_of(b1),
                     "t_embedder.linear2.weight": _bits_of(w2), "t_embedder.linear2.bias": _bits_of(b2)})
    for t in (0.0, 0.3, 0.875):
        want = np.zeros(d.ada_dim)
        want[0] = 2 * _silu(math.cos(1000 * t))
        want[1] = 2 * _silu(math.sin(1000 * t))
        want[2] = 2 * _silu(math.cos(10 * t))
        want[3] = 2 * _silu(math.sin(10 * t))
        want[4] = _silu(0.5)
        want[5] = 0.25
        np.testing.assert_allclose(ref.t_embed(np.array([t]), W)[0], want, rtol=1e-12, atol=1e-14)


def test_final_layer_matches_brute_force():
    d = zi.TINY
    W = ref.Weights(_weights(d, 13))
    rng = np.random.default_rng(13)
    x = rng.standard_normal((3, d.dim)) * 0.7 + 0.2
    c = rng.standard_normal(d.ada_dim) * 0.5
    got = ref.final_layer(x, W, c)
    args = [W(k).tolist() for k in ("final_layer.adaLN_modulation.weight", "final_layer.adaLN_modulation.bias",
                                     "final_layer.linear.weight", "final_layer.linear.bias")]
    for r in range(3):
        np.testing.assert_allclose(got[r], brute.final_layer_loop(x[r].tolist(), c.tolist(), *args),
                                   rtol=1e-11, atol=1e-13)


def test_final_layer_closed_form():
    """Row 0 alternates +-1 (mean 0, variance 1), row 1 is 3 +- 2 (mean 3, variance 4), so the
    LayerNorm gives +-1/sqrt(1 + 1e-6) and +-1/sqrt(1 + 0.25e-6).  c = (1, -2, 0, ...) gives
    SiLU(c) = (e/(1+e), -2/(1+e^2), 0, ...); adaLN weights 0.5 and 0.25 on those two inputs and
    bias 0.125 make s = 0.5 SiLU(1) + 0.25 SiLU(-2) + 0.125 for every channel.  The final
    linear picks channel 0 (output 0), channel 1 (output 1), their sum (output 2, which is 0)
    and a bias of 0.75 (output 3)."""
    d = zi.TINY
    D, P = d.dim, d.patch_dim
    sign = np.where(np.arange(D) % 2 == 0, 1.0, -1.0)
    x = np.stack([sign, 3.0 + 2.0 * sign])
    c = np.zeros(d.ada_dim)
    c[0], c[1] = 1.0, -2.0
    wa = np.zeros((D, d.ada_dim), np.float32)
    wa[:, 0], wa[:, 1] = 0.5, 0.25
    ba = np.full(D, 0.125, np.float32)
    wf = np.zeros((P, D), np.float32)
    wf[0, 0] = wf[1, 1] = wf[2, 0] = wf[2, 1] = 1.0
    bf = np.zeros(P, np.float32)
    bf[3] = 0.75
    W = ref.Weights({"final_layer.adaLN_modulation.weight": _bits_of(wa),
                     "final_layer.adaLN_modulation.bias": _bits_of(ba),
                     "final_layer.linear.weight": _bits_of(wf), "final_layer.linear.bias": _bits_of(bf)})
    s = 0.5 * (1.0 / (1.0 + math.exp(-1.0))) + 0.25 * (-2.0 / (1.0 + math.exp(2.0))) + 0.125
    got = ref.final_layer(x, W, c)
    for r, var in enumerate((1.0, 4.0)):
        ln0 = 2.0 ** r / math.sqrt(var + 1e-6)  # |x - mean| is 1 in row 0 and 2 in row 1
        want = np.zeros(P)
        want[0], want[1], want[3] = ln0 * (1 + s), -ln0 * (1 + s), 0.75
        np.testing.assert_allclose(got[r], want, rtol=1e-13, atol=1e-14)
