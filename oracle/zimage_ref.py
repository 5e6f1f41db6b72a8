"""Step-by-step CPU statement of the Z-Image S3-DiT transformer forward.

TEST INFRASTRUCTURE ONLY (see the package docstring): the GPU library never
imports this module.

Sources (page title, section):
  * ostris ai-toolkit docs, "Z-Image" -- "Architecture" (30 single-stream
    blocks + 2 noise-refiner blocks on image tokens + 2 context-refiner blocks
    on text tokens; hidden 3840 = 30 heads x 128; SwiGLU 10240; RMSNorm,
    QK-RMSNorm; 3-axis RoPE [32, 48, 48], theta 256; adaLN from a 256-d
    timestep embedding, context refiner unmodulated; text and image tokens in
    one sequence), "Latent space" (2x2 patch, one token per 16x16 pixels),
    "Specifics" (the model takes t with 1 = clean).
  * z-image-turbo-mnn model card -- "Conversion details" (the attention output
    projection and FFN w2 outputs feed directly into an RMSNorm), "Model files"
    (transformer interface: sample, timestep, text features -> output).
  * Z-Image-Turbo repackaged for H3ddle -- "What was changed" (the final
    layer's two small linears, final_layer.linear [64, 3840]).

Readings where the pages are silent (each is shared by oracle and GPU path):
  eps 1e-5 for every RMSNorm; final LayerNorm without affine, eps 1e-6;
  adaLN output split [scale_msa, gate_msa, scale_mlp, gate_mlp], scale used as
  (1 + s), gate as tanh(g), no activation between c and the block adaLN
  linear; the final layer's adaLN takes SiLU(c); QK-RMSNorm (gains shared by
  heads) before RoPE; RoPE rotates adjacent pairs (2j, 2j+1) as a complex
  product, head dims [0,32) / [32,80) / [80,128) use axes 0 / 1 / 2 with
  omega_j = theta^(-2j/d_axis); position ids: text token j -> (j+1, 0, 0),
  image token (r, c) -> (L_text+1, r, c); timestep scaled by 1000 before a
  [cos, sin] sinusoid with frequencies 10000^(-k/128); patch feature index
  (i*2 + j)*16 + channel, tokens row-major; unified sequence [image; text];
  attention scale 1/sqrt(128), no mask.
"""
from __future__ import annotations

from typing import Dict, Optional, Set

import numpy as np

from zimage_inputs import Dims, bf16_bits_to_f32

NORM_EPS = 1e-5       # every RMSNorm (block, QK, caption)
FINAL_EPS = 1e-6      # final LayerNorm
ROPE_THETA = 256.0    # "3-axis RoPE [32, 48, 48], theta 256"
T_SCALE = 1000.0      # t in [0, 1] is scaled to [0, 1000] before the sinusoid
MAX_PERIOD = 10000.0  # sinusoid base


class Weights:
    """Read-only view of bf16 weight bits, upcast on access; records used keys."""

    def __init__(self, bits: Dict[str, np.ndarray], dtype=np.float64):
        self.bits = bits
        self.dtype = dtype
        self.used: Set[str] = set()

    def __call__(self, key: str) -> np.ndarray:
        self.used.add(key)
        return bf16_bits_to_f32(self.bits[key]).astype(self.dtype)


# ---------------------------------------------------------------- primitives

def rms_norm(x: np.ndarray, gain: np.ndarray, eps: float = NORM_EPS) -> np.ndarray:
    """y = gain * x / sqrt(mean(x^2) + eps) over the last axis."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gain


def layer_norm(x: np.ndarray, eps: float = FINAL_EPS) -> np.ndarray:
    """LayerNorm over the last axis without affine parameters."""
    mu = np.mean(x, axis=-1, keepdims=True)
    xc = x - mu
    var = np.mean(xc * xc, axis=-1, keepdims=True)
    return xc / np.sqrt(var + eps)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def linear(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray] = None) -> np.ndarray:
    """x @ w^T (+ b); w is [out, in] as stored in the checkpoint."""
    y = x @ w.T
    return y if b is None else y + b


# ---------------------------------------------------------------- embeddings

def timestep_embedding(t_in: np.ndarray, width: int = 256, max_period: float = MAX_PERIOD) -> np.ndarray:
    """[cos(t f_k), sin(t f_k)] with f_k = max_period^(-k/(width/2)), k < width/2."""
    half = width // 2
    k = np.arange(half, dtype=np.float64)
    freqs = np.exp(-np.log(max_period) * k / half)
    args = np.asarray(t_in, dtype=np.float64)[:, None] * freqs[None, :]
    return np.concatenate([np.cos(args), np.sin(args)], axis=-1)


def t_embed(t: np.ndarray, W: Weights) -> np.ndarray:
    """Conditioning vector c [B, 256]: sinusoid of 1000 t -> Linear -> SiLU -> Linear."""
    e = timestep_embedding(np.asarray(t, dtype=np.float64) * T_SCALE).astype(W.dtype)
    h = silu(linear(e, W("t_embedder.linear1.weight"), W("t_embedder.linear1.bias")))
    return linear(h, W("t_embedder.linear2.weight"), W("t_embedder.linear2.bias"))


def patchify(latent: np.ndarray, p: int = 2) -> np.ndarray:
    """[B, C, H, W] -> [B, (H/p)(W/p), p*p*C]; token (r, s) row-major, feature (i*p + j)*C + c."""
    B, C, H, Wd = latent.shape
    x = latent.reshape(B, C, H // p, p, Wd // p, p)      # b c r i s j
    x = x.transpose(0, 2, 4, 3, 5, 1)                    # b r s i j c
    return x.reshape(B, (H // p) * (Wd // p), p * p * C)


def unpatchify(tokens: np.ndarray, C: int, H: int, Wd: int, p: int = 2) -> np.ndarray:
    """Inverse of patchify: [B, (H/p)(W/p), p*p*C] -> [B, C, H, W]."""
    B = tokens.shape[0]
    x = tokens.reshape(B, H // p, Wd // p, p, p, C)      # b r s i j c
    x = x.transpose(0, 5, 1, 3, 2, 4)                    # b c r i s j
    return x.reshape(B, C, H, Wd)


def position_ids(s_txt: int, grid_h: int, grid_w: int) -> np.ndarray:
    """int32 [grid_h*grid_w + s_txt, 3] for the sequence [image; text].

    Image token (r, c) -> (s_txt + 1, r, c); text token j -> (j + 1, 0, 0).
    """
    rr, cc = np.meshgrid(np.arange(grid_h), np.arange(grid_w), indexing="ij")
    img = np.stack([np.full(grid_h * grid_w, s_txt + 1), rr.ravel(), cc.ravel()], axis=1)
    j = np.arange(s_txt)
    txt = np.stack([j + 1, np.zeros_like(j), np.zeros_like(j)], axis=1)
    return np.concatenate([img, txt], axis=0).astype(np.int32)


def position_ids_varlen(s_txt: int, txt_len: int, grid_h: int, grid_w: int) -> np.ndarray:
    """Positions of one padded sequence [image; txt_len text tokens; s_txt - txt_len pads].

    Reading for padded batches: positions follow the element's own text length,
    so image token (r, c) -> (txt_len + 1, r, c); text and pad row j -> (j + 1, 0, 0).
    With the pads masked as keys this makes padding invisible to the valid tokens."""
    pos = position_ids(s_txt, grid_h, grid_w)
    pos[:grid_h * grid_w, 0] = txt_len + 1
    return pos


def rope_angles(pos: np.ndarray, axes=(32, 48, 48), theta: float = ROPE_THETA) -> np.ndarray:
    """Rotation angles [S, sum(axes)/2]: axis a, pair j -> pos[:, a] * theta^(-2j/d_a)."""
    cols = []
    for a, d_a in enumerate(axes):
        j = np.arange(d_a // 2, dtype=np.float64)
        omega = theta ** (-2.0 * j / d_a)
        cols.append(pos[:, a:a + 1].astype(np.float64) * omega[None, :])
    return np.concatenate(cols, axis=1)


def apply_rope(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate pairs (2j, 2j+1) of x [S, H, hd] by angles [S, hd/2] (complex product)."""
    S, H, hd = x.shape
    xr = x.reshape(S, H, hd // 2, 2)
    a, b = xr[..., 0], xr[..., 1]
    cs = np.cos(angles)[:, None, :].astype(x.dtype)
    sn = np.sin(angles)[:, None, :].astype(x.dtype)
    return np.stack([a * cs - b * sn, a * sn + b * cs], axis=-1).reshape(S, H, hd)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, key_valid: Optional[np.ndarray] = None) -> np.ndarray:
    """Non-causal softmax(q k^T / sqrt(hd)) v per head; q, k, v [S, H, hd].

    key_valid (bool [T], optional): keys marked False are excluded (an additive
    -inf key mask, FastVideo zimage handoff, "Transformer": the padded
    variable-length stream needs a key mask)."""
    S, H, hd = q.shape
    out = np.empty((q.shape[0], H, hd), dtype=q.dtype)
    scale = 1.0 / np.sqrt(hd)
    for h in range(H):
        s = (q[:, h] @ k[:, h].T) * scale
        if key_valid is not None:
            s = np.where(key_valid[None, :], s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h] = p @ v[:, h]
    return out


# ---------------------------------------------------------------- blocks

def adaln(c: np.ndarray, W: Weights, prefix: str):
    """Block modulation from c [256]: (scale_msa, gate_msa, scale_mlp, gate_mlp), gates tanh'd."""
    m = linear(c, W(f"{prefix}.adaLN_modulation.weight"), W(f"{prefix}.adaLN_modulation.bias"))
    scale_msa, gate_msa, scale_mlp, gate_mlp = np.split(m, 4, axis=-1)
    return scale_msa, np.tanh(gate_msa), scale_mlp, np.tanh(gate_mlp)


def block_forward(x: np.ndarray, W: Weights, prefix: str, d: Dims, angles: np.ndarray,
                  c: Optional[np.ndarray] = None, return_parts: bool = False,
                  key_valid: Optional[np.ndarray] = None):
    """One S3-DiT block on x [S, D].  c=None runs the unmodulated (context-refiner) form.

    attention sublayer: h = RMSNorm1(x)(1 + scale_msa); q, k, v = h Wq, h Wk, h Wv;
      q, k <- RoPE(RMSNorm_head(.)); o = Attn(q, k, v) Wout;
      x <- x + tanh(gate_msa) RMSNorm2(o)
    FFN sublayer: h = RMSNormF1(x)(1 + scale_mlp); f = (SiLU(h W1) * (h W3)) W2;
      x <- x + tanh(gate_mlp) RMSNormF2(f)
    """
    S, D = x.shape
    H, hd = d.heads, d.head_dim
    if c is not None:
        scale_msa, gate_msa, scale_mlp, gate_mlp = adaln(c, W, prefix)
    else:
        scale_msa = scale_mlp = 0.0
        gate_msa = gate_mlp = 1.0
    a = f"{prefix}.attention"
    h = rms_norm(x, W(f"{prefix}.attention_norm1.weight")) * (1.0 + scale_msa)
    q = linear(h, W(f"{a}.to_q.weight")).reshape(S, H, hd)
    k = linear(h, W(f"{a}.to_k.weight")).reshape(S, H, hd)
    v = linear(h, W(f"{a}.to_v.weight")).reshape(S, H, hd)
    q = apply_rope(rms_norm(q, W(f"{a}.norm_q.weight")), angles)
    k = apply_rope(rms_norm(k, W(f"{a}.norm_k.weight")), angles)
    att = attention(q, k, v, key_valid).reshape(S, D)
    o = linear(att, W(f"{a}.to_out.weight"))
    x1 = x + gate_msa * rms_norm(o, W(f"{prefix}.attention_norm2.weight"))
    h2 = rms_norm(x1, W(f"{prefix}.ffn_norm1.weight")) * (1.0 + scale_mlp)
    ff = f"{prefix}.feed_forward"
    u = silu(linear(h2, W(f"{ff}.w1.weight"))) * linear(h2, W(f"{ff}.w3.weight"))
    f = linear(u, W(f"{ff}.w2.weight"))
    x2 = x1 + gate_mlp * rms_norm(f, W(f"{prefix}.ffn_norm2.weight"))
    if return_parts:
        return x2, dict(h=h, q=q, k=k, v=v, att=att, o=o, x1=x1, h2=h2, u=u, f=f)
    return x2


def block_forward_rows(x: np.ndarray, W: Weights, prefix: str, d: Dims, angles: np.ndarray,
                       c: Optional[np.ndarray], rows: np.ndarray,
                       key_valid: Optional[np.ndarray] = None) -> np.ndarray:
    """block_forward(x, ...)[rows], computed for those query rows only.

    Keys and values come from every row of x (the attention is over the whole
    sequence); every other step is per row, so only the selected rows go
    through the query projection, attention, output projection and FFN.
    """
    S, D = x.shape
    H, hd = d.heads, d.head_dim
    if c is not None:
        scale_msa, gate_msa, scale_mlp, gate_mlp = adaln(c, W, prefix)
    else:
        scale_msa = scale_mlp = 0.0
        gate_msa = gate_mlp = 1.0
    a = f"{prefix}.attention"
    h = rms_norm(x, W(f"{prefix}.attention_norm1.weight")) * (1.0 + scale_msa)
    k = apply_rope(rms_norm(linear(h, W(f"{a}.to_k.weight")).reshape(S, H, hd), W(f"{a}.norm_k.weight")), angles)
    v = linear(h, W(f"{a}.to_v.weight")).reshape(S, H, hd)
    hr = h[rows]
    q = linear(hr, W(f"{a}.to_q.weight")).reshape(len(rows), H, hd)
    q = apply_rope(rms_norm(q, W(f"{a}.norm_q.weight")), angles[rows])
    att = attention(q, k, v, key_valid).reshape(len(rows), D)
    o = linear(att, W(f"{a}.to_out.weight"))
    x1 = x[rows] + gate_msa * rms_norm(o, W(f"{prefix}.attention_norm2.weight"))
    h2 = rms_norm(x1, W(f"{prefix}.ffn_norm1.weight")) * (1.0 + scale_mlp)
    ff = f"{prefix}.feed_forward"
    u = silu(linear(h2, W(f"{ff}.w1.weight"))) * linear(h2, W(f"{ff}.w3.weight"))
    f = linear(u, W(f"{ff}.w2.weight"))
    return x1 + gate_mlp * rms_norm(f, W(f"{prefix}.ffn_norm2.weight"))


def final_layer(x_img: np.ndarray, W: Weights, c: np.ndarray) -> np.ndarray:
    """LayerNorm(x) * (1 + Linear(SiLU(c))) -> Linear to p*p*C features."""
    s = linear(silu(c), W("final_layer.adaLN_modulation.weight"), W("final_layer.adaLN_modulation.bias"))
    y = layer_norm(x_img) * (1.0 + s)
    return linear(y, W("final_layer.linear.weight"), W("final_layer.linear.bias"))


def embed_text(txt: np.ndarray, W: Weights) -> np.ndarray:
    """cap_embedder: RMSNorm(cap_dim, gain) then Linear cap_dim -> D (+bias)."""
    t = rms_norm(txt, W("cap_embedder.norm.weight"))
    return linear(t, W("cap_embedder.linear.weight"), W("cap_embedder.linear.bias"))


def model_forward(latent: np.ndarray, t: np.ndarray, txt: np.ndarray, W: Weights, d: Dims,
                  trace: Optional[list] = None, txt_len: Optional[np.ndarray] = None) -> np.ndarray:
    """Full transformer forward.

    latent [B, C, H/8, W/8] (any float), t [B] in [0, 1] (1 = clean),
    txt [B, L, cap_dim] float.  Returns the raw model output [B, C, H/8, W/8]
    (the scheduler negates it).  ``trace``, if given, receives the residual
    stream [S, D] of sample 0 after every block, in execution order.

    txt_len [B] (optional): element b has txt_len[b] valid text tokens; its text
    rows from txt_len[b] on are padding: their embeddings are replaced by the
    cap_pad_token and they are masked as keys in every attention.
    """
    B, C, Hl, Wl = latent.shape
    p = d.patch
    gh, gw = Hl // p, Wl // p
    s_img = gh * gw
    L = txt.shape[1]
    tokens = patchify(np.asarray(latent, dtype=W.dtype), p)
    c_all = t_embed(t, W)
    outs = []
    for b in range(B):
        c = c_all[b]
        lb = L if txt_len is None else int(txt_len[b])
        if txt_len is None:
            ang = rope_angles(position_ids(L, gh, gw), d.rope_axes)
            kv_txt = kv_all = None
        else:
            ang = rope_angles(position_ids_varlen(L, lb, gh, gw), d.rope_axes)
            kv_txt = np.arange(L) < lb
            kv_all = np.concatenate([np.ones(s_img, dtype=bool), kv_txt])
        xi = linear(tokens[b], W("x_embedder.weight"), W("x_embedder.bias"))
        xt = embed_text(np.asarray(txt[b], dtype=W.dtype), W)
        if txt_len is not None and lb < L:
            xt[lb:] = W("cap_pad_token")
        for i in range(d.n_noise):
            xi = block_forward(xi, W, f"noise_refiner.{i}", d, ang[:s_img], c)
            if trace is not None and b == 0:
                trace.append(xi.copy())
        for i in range(d.n_ctx):
            xt = block_forward(xt, W, f"context_refiner.{i}", d, ang[s_img:], None, key_valid=kv_txt)
            if trace is not None and b == 0:
                trace.append(xt.copy())
        x = np.concatenate([xi, xt], axis=0)
        for i in range(d.n_main):
            x = block_forward(x, W, f"layers.{i}", d, ang, c, key_valid=kv_all)
            if trace is not None and b == 0:
                trace.append(x.copy())
        y = final_layer(x[:s_img], W, c)
        outs.append(unpatchify(y[None], C, Hl, Wl, p)[0])
    return np.stack(outs, axis=0)
