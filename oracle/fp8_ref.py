"""FP8 (e4m3) projections: CPU statement of the quantised variant of the forward.

TEST INFRASTRUCTURE ONLY: the GPU library never imports this module.

What the pages give (page title, section): the quantised variants are the
pages' main subject -- int8 weights with rotated activations (Z-Image-Turbo
repackaged for H3ddle, "What was changed, and why"), qfloat8 and int8 builds
(ostris "Z-Image", "Specifics"; z-image-turbo-mnn "Conversion details"), and the
observation that the output projection and FFN w2 feed an RMSNorm directly
(z-image-turbo-mnn "Conversion details").  None fixes an fp8 recipe, so this
module states one (a reading, shared with the GPU path):

  * format: OCP e4m3 -- 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits;
    exponent 0 holds the subnormals m * 2^-9; the all-ones pattern S.1111.111 is
    NaN; the largest finite magnitude is 448 (S.1111.110).  Rounding to nearest,
    ties to the even code; magnitudes beyond 448 saturate to 448.
  * which projections: the two whose input is a whole-row RMSNorm output, the
    fused QKV projection and the FFN w1|w3 projection; optionally (all=True)
    also the attention output projection and FFN w2, whose inputs (attention
    output, SwiGLU output) are quantised per row the same way.  The embedders,
    adaLN and the final layer stay bf16.
  * scales: one per row of each operand.  Activations h [M, K]: s_a[m] =
    amax_m / 448, codes = e4m3(h[m, :] * (448 / amax_m)).  Weights [N, K]: the
    same per output channel.  A row of zeros gets scale 1 and zero codes.
    The scale and the scaled value are formed in fp32 (the GPU's precision),
    so both sides take the same rounding decisions from the same fp32 input.
  * the product: y[m, n] = s_a[m] s_w[n] sum_k a[m, k] w[n, k] over the decoded
    codes (exact here in fp64; fp32 accumulation on the GPU).
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from oracle import zimage_ref as ref

E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each e4m3 byte (float64; NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


# the 127 non-negative finite values in code order (code 0x00 .. 0x7E), increasing
_POS_CODES = np.arange(0x7F)
_POS_VALUES = e4m3_decode(_POS_CODES)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Nearest e4m3 code of each value (ties to the even code), saturating at 448; the
    sign bit is the input's (so -0 and negative values that round to zero give 0x80).

    Written as a search over the table of representable magnitudes: the two
    neighbours of |x| are found, the nearer wins, and on an exact tie the code
    with a zero lowest mantissa bit (the even code) wins."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_POS_VALUES, a, side="left")          # first value >= a
    hi = np.minimum(hi, len(_POS_VALUES) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (_POS_CODES[hi] % 2 == 0))
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    code = np.where(a == _POS_VALUES[hi], _POS_CODES[hi], code)
    return (code | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)  # the sign is kept, also on zero


def quantize_rows(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row e4m3 quantisation of x [R, K]: (codes uint8 [R, K], scales fp32 [R]).

    amax, 448 / amax and x * (448 / amax) are each rounded to fp32, as the GPU
    forms them; a zero row gets scale 1 and zero codes."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=1)
    zero = amax == 0
    safe = np.where(zero, np.float32(1.0), amax).astype(np.float32)
    inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    y = (x32 * inv[:, None]).astype(np.float32)
    codes = e4m3_encode(y)
    codes[zero] = 0
    scale = np.where(zero, np.float32(1.0), (safe / np.float32(E4M3_MAX)).astype(np.float32)).astype(np.float32)
    return codes, scale


def dequantize_rows(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[:, None]


def fp8_linear(h: np.ndarray, w: np.ndarray) -> np.ndarray:
    """h [M, K] @ w [N, K]^T with both operands quantised per row (the reading above)."""
    hq, hs = quantize_rows(h)
    wq, ws = quantize_rows(w)
    return dequantize_rows(hq, hs) @ dequantize_rows(wq, ws).T


def block_forward(x: np.ndarray, W: ref.Weights, prefix: str, d, angles: np.ndarray,
                  c: Optional[np.ndarray] = None, key_valid: Optional[np.ndarray] = None,
                  all: bool = False) -> np.ndarray:
    """The block of zimage_ref.block_forward with the QKV and FFN w1|w3 projections in e4m3
    (all=True: the output projection and FFN w2 as well).

    h is quantised once per row and shared by q, k and v (one fused projection);
    every weight row (output channel) has its own scale."""
    S, D = x.shape
    H, hd = d.heads, d.head_dim
    if c is not None:
        scale_msa, gate_msa, scale_mlp, gate_mlp = ref.adaln(c, W, prefix)
    else:
        scale_msa = scale_mlp = 0.0
        gate_msa = gate_mlp = 1.0
    a = f"{prefix}.attention"
    h = ref.rms_norm(x, W(f"{prefix}.attention_norm1.weight")) * (1.0 + scale_msa)
    wqkv = np.concatenate([W(f"{a}.to_q.weight"), W(f"{a}.to_k.weight"), W(f"{a}.to_v.weight")], axis=0)
    qkv = fp8_linear(h, wqkv)
    q, k, v = (qkv[:, i * D:(i + 1) * D].reshape(S, H, hd) for i in range(3))
    q = ref.apply_rope(ref.rms_norm(q, W(f"{a}.norm_q.weight")), angles)
    k = ref.apply_rope(ref.rms_norm(k, W(f"{a}.norm_k.weight")), angles)
    att = ref.attention(q, k, v, key_valid).reshape(S, D)
    o = fp8_linear(att, W(f"{a}.to_out.weight")) if all else ref.linear(att, W(f"{a}.to_out.weight"))
    x1 = x + gate_msa * ref.rms_norm(o, W(f"{prefix}.attention_norm2.weight"))
    h2 = ref.rms_norm(x1, W(f"{prefix}.ffn_norm1.weight")) * (1.0 + scale_mlp)
    ff = f"{prefix}.feed_forward"
    w13 = np.concatenate([W(f"{ff}.w1.weight"), W(f"{ff}.w3.weight")], axis=0)
    g13 = fp8_linear(h2, w13)
    F = d.ffn
    u = ref.silu(g13[:, :F]) * g13[:, F:]
    f = fp8_linear(u, W(f"{ff}.w2.weight")) if all else ref.linear(u, W(f"{ff}.w2.weight"))
    return x1 + gate_mlp * ref.rms_norm(f, W(f"{prefix}.ffn_norm2.weight"))


def block_forward_rows(x: np.ndarray, W: ref.Weights, prefix: str, d, angles: np.ndarray,
                       c: Optional[np.ndarray], rows: np.ndarray, all: bool = False) -> np.ndarray:
    """block_forward(x, ...)[rows] for the selected query rows only (keys and values
    from every row).  Every step but attention is per row, and so is the e4m3
    quantisation (one scale per row), so the selected rows' results are those of
    the whole-sequence block."""
    S, D = x.shape
    H, hd = d.heads, d.head_dim
    if c is not None:
        scale_msa, gate_msa, scale_mlp, gate_mlp = ref.adaln(c, W, prefix)
    else:
        scale_msa = scale_mlp = 0.0
        gate_msa = gate_mlp = 1.0
    a = f"{prefix}.attention"
    h = ref.rms_norm(x, W(f"{prefix}.attention_norm1.weight")) * (1.0 + scale_msa)
    hq, hs = quantize_rows(h)
    hd8 = dequantize_rows(hq, hs)  # the quantised h of every row
    deq = lambda w: dequantize_rows(*quantize_rows(w))
    k = ref.apply_rope(ref.rms_norm((hd8 @ deq(W(f"{a}.to_k.weight")).T).reshape(S, H, hd),
                                    W(f"{a}.norm_k.weight")), angles)
    v = (hd8 @ deq(W(f"{a}.to_v.weight")).T).reshape(S, H, hd)
    q = (hd8[rows] @ deq(W(f"{a}.to_q.weight")).T).reshape(len(rows), H, hd)
    q = ref.apply_rope(ref.rms_norm(q, W(f"{a}.norm_q.weight")), angles[rows])
    att = ref.attention(q, k, v).reshape(len(rows), D)
    o = fp8_linear(att, W(f"{a}.to_out.weight")) if all else ref.linear(att, W(f"{a}.to_out.weight"))
    x1 = x[rows] + gate_msa * ref.rms_norm(o, W(f"{prefix}.attention_norm2.weight"))
    h2 = ref.rms_norm(x1, W(f"{prefix}.ffn_norm1.weight")) * (1.0 + scale_mlp)
    ff = f"{prefix}.feed_forward"
    w13 = np.concatenate([W(f"{ff}.w1.weight"), W(f"{ff}.w3.weight")], axis=0)
    g13 = fp8_linear(h2, w13)
    F = d.ffn
    u = ref.silu(g13[:, :F]) * g13[:, F:]
    f = fp8_linear(u, W(f"{ff}.w2.weight")) if all else ref.linear(u, W(f"{ff}.w2.weight"))
    return x1 + gate_mlp * ref.rms_norm(f, W(f"{prefix}.ffn_norm2.weight"))


def model_forward(latent: np.ndarray, t: np.ndarray, txt: np.ndarray, W: ref.Weights, d,
                  all: bool = False) -> np.ndarray:
    """zimage_ref.model_forward with every block's QKV and FFN w1|w3 projections in e4m3
    (all=True: every block projection)."""
    B, C, Hl, Wl = latent.shape
    p = d.patch
    gh, gw = Hl // p, Wl // p
    s_img = gh * gw
    L = txt.shape[1]
    tokens = ref.patchify(np.asarray(latent, dtype=W.dtype), p)
    c_all = ref.t_embed(t, W)
    ang = ref.rope_angles(ref.position_ids(L, gh, gw), d.rope_axes)
    outs = []
    for b in range(B):
        c = c_all[b]
        xi = ref.linear(tokens[b], W("x_embedder.weight"), W("x_embedder.bias"))
        xt = ref.embed_text(np.asarray(txt[b], dtype=W.dtype), W)
        for i in range(d.n_noise):
            xi = block_forward(xi, W, f"noise_refiner.{i}", d, ang[:s_img], c, all=all)
        for i in range(d.n_ctx):
            xt = block_forward(xt, W, f"context_refiner.{i}", d, ang[s_img:], None, all=all)
        x = np.concatenate([xi, xt], axis=0)
        for i in range(d.n_main):
            x = block_forward(x, W, f"layers.{i}", d, ang, c, all=all)
        y = ref.final_layer(x[:s_img], W, c)
        outs.append(ref.unpatchify(y[None], C, Hl, Wl, p)[0])
    return np.stack(outs, axis=0)
