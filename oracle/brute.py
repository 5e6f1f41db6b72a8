"""Scalar-loop fp64 restatements used to pin the oracle on tiny inputs.

TEST INFRASTRUCTURE ONLY.  These are written as explicit loops (or, for RoPE,
as an explicit block-diagonal rotation matrix) so that they share no
vectorisation, reshaping or transposition with ``zimage_ref``; a transposed
operand or a wrong index there disagrees with the result here.
"""
from __future__ import annotations

import math
from typing import List, Sequence

import numpy as np


def matmul_bt(a: Sequence[Sequence[float]], b: Sequence[Sequence[float]]) -> List[List[float]]:
    """C[i][j] = sum_k a[i][k] * b[j][k] (b stored [out, in])."""
    n, m, kk = len(a), len(b), len(a[0])
    return [[math.fsum(a[i][k] * b[j][k] for k in range(kk)) for j in range(m)] for i in range(n)]


def rms_norm_row(x: Sequence[float], g: Sequence[float], eps: float) -> List[float]:
    ms = math.fsum(v * v for v in x) / len(x)
    r = 1.0 / math.sqrt(ms + eps)
    return [x[i] * r * g[i] for i in range(len(x))]


def attention_head(q, k, v) -> List[List[float]]:
    """softmax(q k^T / sqrt(d)) v for one head; q [S, d], k [T, d], v [T, dv] as nested lists."""
    S, T, d = len(q), len(k), len(q[0])
    scale = 1.0 / math.sqrt(d)
    out = []
    for i in range(S):
        s = [math.fsum(q[i][c] * k[j][c] for c in range(d)) * scale for j in range(T)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = math.fsum(e)
        out.append([math.fsum(e[j] * v[j][c] for j in range(T)) / z for c in range(len(v[0]))])
    return out


def rope_matrix(pos: Sequence[int], axes=(32, 48, 48), theta: float = 256.0) -> np.ndarray:
    """Explicit [hd, hd] rotation matrix R with RoPE(x) = R x for one token.

    Pair j of axis a occupies dims (off_a + 2j, off_a + 2j + 1) and rotates by
    pos[a] * theta^(-2j/d_a), counter-clockwise.
    """
    hd = sum(axes)
    R = np.zeros((hd, hd))
    off = 0
    for a, d_a in enumerate(axes):
        for j in range(d_a // 2):
            ang = pos[a] * theta ** (-2.0 * j / d_a)
            i0 = off + 2 * j
            R[i0, i0] = math.cos(ang)
            R[i0, i0 + 1] = -math.sin(ang)
            R[i0 + 1, i0] = math.sin(ang)
            R[i0 + 1, i0 + 1] = math.cos(ang)
        off += d_a
    return R


def patchify_loop(latent: np.ndarray, p: int = 2) -> np.ndarray:
    """Token (b, r*(W/p)+s), feature (i*p+j)*C + c <- latent[b, c, p*r+i, p*s+j]."""
    B, C, H, W = latent.shape
    gh, gw = H // p, W // p
    out = np.zeros((B, gh * gw, p * p * C), dtype=latent.dtype)
    for b in range(B):
        for r in range(gh):
            for s in range(gw):
                for i in range(p):
                    for j in range(p):
                        for c in range(C):
                            out[b, r * gw + s, (i * p + j) * C + c] = latent[b, c, p * r + i, p * s + j]
    return out


def position_ids_loop(s_txt: int, grid_h: int, grid_w: int) -> List[List[int]]:
    ids = []
    for r in range(grid_h):
        for c in range(grid_w):
            ids.append([s_txt + 1, r, c])
    for j in range(s_txt):
        ids.append([j + 1, 0, 0])
    return ids


def t_embed_loop(t: float, w1, b1, w2, b2, t_scale: float = 1000.0, max_period: float = 10000.0) -> List[float]:
    """Conditioning vector of one timestep, written out element by element.

    The model timestep t (1 = clean) is scaled by t_scale; entry k < half of the
    sinusoid is cos(t_scale t f_k), entry half + k is sin(t_scale t f_k), with
    f_k = max_period^(-k / half); then hidden unit j = SiLU(sum_k w1[j][k] e_k + b1[j])
    and output i = sum_j w2[i][j] hidden_j + b2[i].  w1, w2 are [out][in] nested lists.
    """
    width = len(w1[0])
    half = width // 2
    e = [0.0] * width
    for k in range(half):
        arg = t * t_scale * math.exp(-math.log(max_period) * k / half)
        e[k] = math.cos(arg)
        e[half + k] = math.sin(arg)
    hid = []
    for j in range(len(w1)):
        z = math.fsum(w1[j][k] * e[k] for k in range(width)) + b1[j]
        hid.append(z / (1.0 + math.exp(-z)))
    return [math.fsum(w2[i][j] * hid[j] for j in range(len(hid))) + b2[i] for i in range(len(w2))]


def final_layer_loop(x_row: Sequence[float], c: Sequence[float], wa, ba, wf, bf, eps: float = 1e-6) -> List[float]:
    """Final layer of one image token, element by element.

    LayerNorm without affine (mean and biased variance over the row, eps inside the
    root), scaled by (1 + s) with s_i = sum_k wa[i][k] SiLU(c_k) + ba[i], then the
    linear map out_j = sum_i wf[j][i] y_i + bf[j].
    """
    n = len(x_row)
    mu = math.fsum(x_row) / n
    var = math.fsum((v - mu) ** 2 for v in x_row) / n
    inv = 1.0 / math.sqrt(var + eps)
    sc = [v / (1.0 + math.exp(-v)) for v in c]
    y = []
    for i in range(n):
        s = math.fsum(wa[i][k] * sc[k] for k in range(len(sc))) + ba[i]
        y.append((x_row[i] - mu) * inv * (1.0 + s))
    return [math.fsum(wf[j][i] * y[i] for i in range(n)) + bf[j] for j in range(len(wf))]
