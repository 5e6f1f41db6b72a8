"""Seeded synthetic inputs for the Z-Image S3-DiT forward: weights, latents, text features.

This module is shared by the CPU oracle (``oracle/``) and by the GPU path's tests
and benchmark.  It holds shapes and random numbers only: none of the method's
arithmetic lives here (no norms, no projections, no RoPE, no schedule).

Shapes follow the architecture summary on the ostris ai-toolkit page "Z-Image"
(sections "Components", "Latent space", "Architecture"): hidden 3840 = 30 heads x
128, SwiGLU FFN 10240, 2 noise-refiner + 2 context-refiner + 30 main blocks,
2560-d text features, 256-d timestep embedding, 16 latent channels, 2x2 patch.
The key list reproduces the 521 checkpoint keys named on the FastVideo page
(section "Transformer") and the 6,154,908,736 parameters of the ostris
"Components" table; the oracle's tests pin both counts.

Random numbers: NumPy PCG64.  Every tensor has its own child seed
``SeedSequence(seed, spawn_key=(stream, index))`` so any one tensor (or block)
can be regenerated alone and tensors can be generated in parallel.
Streams: 0 = weights (index = position in the canonical key order),
1 = latent, 2 = conditional text features, 3 = unconditional text features.

Init recipe (the configs say "random-init N(0, 0.02)"): linear weights and
biases N(0, 0.02); RMSNorm gains 1 + N(0, 0.02) so that a dropped gain is
detectable; pad tokens N(0, 0.02).  Values are drawn in fp32 and rounded to
bf16 (round to nearest even); both sides consume the same bf16 bits.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

WEIGHT_STREAM, LATENT_STREAM, TEXT_STREAM, TEXT_UNCOND_STREAM = 0, 1, 2, 3
INIT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class Dims:
    """Sizes of one S3-DiT variant (shapes only)."""
    dim: int = 3840          # hidden width D
    heads: int = 30          # attention heads (query and key/value)
    head_dim: int = 128
    ffn: int = 10240         # SwiGLU inner width F
    cap_dim: int = 2560      # text-feature width (Qwen3-4B hidden)
    t_freq: int = 256        # sinusoidal timestep-embedding width
    t_mid: int = 1024        # timestep MLP hidden width
    in_ch: int = 16          # latent channels
    patch: int = 2
    n_noise: int = 2         # noise-refiner blocks (image tokens, modulated)
    n_ctx: int = 2           # context-refiner blocks (text tokens, unmodulated)
    n_main: int = 30         # main single-stream blocks
    rope_axes: Tuple[int, int, int] = (32, 48, 48)

    @property
    def ada_dim(self) -> int:
        """Width of the conditioning vector c fed to every adaLN linear."""
        return min(self.dim, 256)

    @property
    def patch_dim(self) -> int:
        return self.patch * self.patch * self.in_ch

    @property
    def n_modulated(self) -> int:
        return self.n_noise + self.n_main


FULL = Dims()
# One modulated main block at hidden 256 (2 heads x 128), FFN 688, no refiners.
TINY = Dims(dim=256, heads=2, ffn=688, n_noise=0, n_ctx=0, n_main=1)
# The same tiny width with one block of each kind, so the refiners are exercised.
TINY_R = Dims(dim=256, heads=2, ffn=688, n_noise=1, n_ctx=1, n_main=1)


def block_specs(prefix: str, d: Dims, modulated: bool) -> List[Tuple[str, Tuple[int, ...], str]]:
    D, F, hd = d.dim, d.ffn, d.head_dim
    s = [
        (f"{prefix}.attention.to_q.weight", (D, D), "linear"),
        (f"{prefix}.attention.to_k.weight", (D, D), "linear"),
        (f"{prefix}.attention.to_v.weight", (D, D), "linear"),
        (f"{prefix}.attention.to_out.weight", (D, D), "linear"),
        (f"{prefix}.attention.norm_q.weight", (hd,), "gain"),
        (f"{prefix}.attention.norm_k.weight", (hd,), "gain"),
        (f"{prefix}.attention_norm1.weight", (D,), "gain"),
        (f"{prefix}.attention_norm2.weight", (D,), "gain"),
        (f"{prefix}.ffn_norm1.weight", (D,), "gain"),
        (f"{prefix}.ffn_norm2.weight", (D,), "gain"),
        (f"{prefix}.feed_forward.w1.weight", (F, D), "linear"),
        (f"{prefix}.feed_forward.w2.weight", (D, F), "linear"),
        (f"{prefix}.feed_forward.w3.weight", (F, D), "linear"),
    ]
    if modulated:
        s += [
            (f"{prefix}.adaLN_modulation.weight", (4 * D, d.ada_dim), "linear"),
            (f"{prefix}.adaLN_modulation.bias", (4 * D,), "linear"),
        ]
    return s


def weight_specs(d: Dims) -> List[Tuple[str, Tuple[int, ...], str]]:
    """Canonical ordered list of (key, shape, init kind)."""
    D = d.dim
    s: List[Tuple[str, Tuple[int, ...], str]] = [
        ("x_embedder.weight", (D, d.patch_dim), "linear"),
        ("x_embedder.bias", (D,), "linear"),
        ("cap_embedder.norm.weight", (d.cap_dim,), "gain"),
        ("cap_embedder.linear.weight", (D, d.cap_dim), "linear"),
        ("cap_embedder.linear.bias", (D,), "linear"),
        ("t_embedder.linear1.weight", (d.t_mid, d.t_freq), "linear"),
        ("t_embedder.linear1.bias", (d.t_mid,), "linear"),
        ("t_embedder.linear2.weight", (d.ada_dim, d.t_mid), "linear"),
        ("t_embedder.linear2.bias", (d.ada_dim,), "linear"),
    ]
    for i in range(d.n_noise):
        s += block_specs(f"noise_refiner.{i}", d, True)
    for i in range(d.n_ctx):
        s += block_specs(f"context_refiner.{i}", d, False)
    for i in range(d.n_main):
        s += block_specs(f"layers.{i}", d, True)
    s += [
        ("final_layer.adaLN_modulation.weight", (D, d.ada_dim), "linear"),
        ("final_layer.adaLN_modulation.bias", (D,), "linear"),
        ("final_layer.linear.weight", (d.patch_dim, D), "linear"),
        ("final_layer.linear.bias", (d.patch_dim,), "linear"),
        ("x_pad_token", (D,), "pad"),
        ("cap_pad_token", (D,), "pad"),
    ]
    return s


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, stream: int, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(stream, index))))


def make_tensor(seed: int, index: int, shape: Sequence[int], kind: str) -> np.ndarray:
    """One weight tensor as bf16 bits (uint16), drawn from its own child seed."""
    v = _rng(seed, WEIGHT_STREAM, index).standard_normal(size=tuple(shape), dtype=np.float32)
    v *= np.float32(INIT_STD)
    if kind == "gain":
        v += np.float32(1.0)
    return f32_to_bf16_bits(v)


def iter_weights(d: Dims, seed: int = 0, keys: Optional[Iterable[str]] = None,
                 threads: int = 1):
    """Yield (key, bf16 bits) in canonical order (restricted to ``keys`` if given)."""
    specs = weight_specs(d)
    want = None if keys is None else set(keys)
    jobs = [(i, k, sh, kind) for i, (k, sh, kind) in enumerate(specs) if want is None or k in want]
    if threads <= 1:
        for i, k, sh, kind in jobs:
            yield k, make_tensor(seed, i, sh, kind)
        return
    with ThreadPoolExecutor(max_workers=threads) as ex:
        window = []
        for job in jobs:
            window.append((job[1], ex.submit(make_tensor, seed, job[0], job[2], job[3])))
            if len(window) >= 2 * threads:
                k, fut = window.pop(0)
                yield k, fut.result()
        for k, fut in window:
            yield k, fut.result()


def make_weights(d: Dims, seed: int = 0, keys: Optional[Iterable[str]] = None,
                 threads: int = 1) -> Dict[str, np.ndarray]:
    """All (or the selected) weights as a dict of bf16 bit arrays."""
    return dict(iter_weights(d, seed, keys, threads))


def make_latent(d: Dims, batch: int, lat_h: int, lat_w: int, seed: int = 0) -> np.ndarray:
    """Latent N(0, 1), fp32 [B, C, lat_h, lat_w] (lat = image size / 8)."""
    return _rng(seed, LATENT_STREAM).standard_normal(size=(batch, d.in_ch, lat_h, lat_w), dtype=np.float32)


def make_text(d: Dims, batch: int, length: int, seed: int = 0, uncond: bool = False) -> np.ndarray:
    """Text features N(0, 1) rounded to bf16, returned as bits [B, L, cap_dim]."""
    stream = TEXT_UNCOND_STREAM if uncond else TEXT_STREAM
    v = _rng(seed, stream).standard_normal(size=(batch, length, d.cap_dim), dtype=np.float32)
    return f32_to_bf16_bits(v)


def make_stream(d: Dims, batch: int, seq: int, seed: int = 0, std: float = 0.16) -> np.ndarray:
    """A residual stream N(0, std^2), fp32 [B, S, D], for single-block workloads."""
    return (_rng(seed, LATENT_STREAM, 1).standard_normal(size=(batch, seq, d.dim), dtype=np.float32)
            * np.float32(std))


def make_cond(d: Dims, batch: int, seed: int = 0, std: float = 0.07) -> np.ndarray:
    """A conditioning vector c N(0, std^2), fp32 [B, ada_dim], for single-block workloads."""
    return (_rng(seed, LATENT_STREAM, 2).standard_normal(size=(batch, d.ada_dim), dtype=np.float32)
            * np.float32(std))


MATRIX_STREAM = 4


def make_matrix(shape: Sequence[int], seed: int = 0, index: int = 0, std: float = 1.0) -> np.ndarray:
    """A generic N(0, std^2) tensor rounded to bf16 (bits), for single-kernel checks."""
    v = _rng(seed, MATRIX_STREAM, index).standard_normal(size=tuple(shape), dtype=np.float32)
    if std != 1.0:
        v *= np.float32(std)
    return f32_to_bf16_bits(v)
