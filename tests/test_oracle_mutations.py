"""Planted mistakes in the oracle must trip at least one pin.

Each case patches one plausible mistake into ``oracle.zimage_ref`` (on the CPU,
inside the test only) and re-runs the pins that should catch it.
"""
import numpy as np
import pytest

from oracle import zimage_ref as ref
import test_oracle_block as tb
import test_oracle_primitives as tp
import test_oracle_structure as ts


def _rope_half_split(x, angles):
    S, H, hd = x.shape
    a, b = x[..., :hd // 2], x[..., hd // 2:]
    cs, sn = np.cos(angles)[:, None, :], np.sin(angles)[:, None, :]
    return np.concatenate([a * cs - b * sn, a * sn + b * cs], axis=-1)


def _rope_clockwise(x, angles):
    return ref.__dict__["_orig_apply_rope"](x, -angles)


def _angles_wrong_exponent(pos, axes=(32, 48, 48), theta=256.0):
    cols = []
    for a, d_a in enumerate(axes):
        j = np.arange(d_a // 2, dtype=np.float64)
        cols.append(pos[:, a:a + 1] * (theta ** (-1.0 * j / d_a))[None, :])
    return np.concatenate(cols, axis=1)


def _attention_keys_softmax(q, k, v):
    S, H, hd = q.shape
    out = np.empty_like(q)
    for h in range(H):
        s = (q[:, h] @ k[:, h].T) / np.sqrt(hd)
        p = np.exp(s - s.max(axis=0, keepdims=True))
        p = p / p.sum(axis=0, keepdims=True)          # normalised over queries
        out[:, h] = p @ v[:, h]
    return out


def _attention_no_scale(q, k, v):
    return ref.__dict__["_orig_attention"](q * np.sqrt(q.shape[-1]), k, v)


def _rms_no_eps_sqrt(x, gain, eps=1e-5):
    return x / (np.mean(x * x, axis=-1, keepdims=True) + eps) * gain


def _patchify_channel_slowest(latent, p=2):
    B, C, H, W = latent.shape
    x = latent.reshape(B, C, H // p, p, W // p, p).transpose(0, 2, 4, 1, 3, 5)
    return x.reshape(B, (H // p) * (W // p), p * p * C)


def _block_without_post_norm(x, W, prefix, d, angles, c=None, return_parts=False):
    saved = ref.rms_norm
    calls = {"n": 0}

    def rms(xx, g, eps=ref.NORM_EPS):
        calls["n"] += 1
        # the 2nd and 5th norms of the block are the post-norms (after to_out, after w2)
        if xx.shape[-1] == d.dim and calls["n"] in (4, 6):
            return xx * g
        return saved(xx, g, eps)

    ref.rms_norm = rms
    try:
        return ref.__dict__["_orig_block_forward"](x, W, prefix, d, angles, c, return_parts)
    finally:
        ref.rms_norm = saved


def _t_embed_no_scale(t, W):
    e = ref.timestep_embedding(np.asarray(t, dtype=np.float64)).astype(W.dtype)  # t, not 1000 t
    h = ref.silu(ref.linear(e, W("t_embedder.linear1.weight"), W("t_embedder.linear1.bias")))
    return ref.linear(h, W("t_embedder.linear2.weight"), W("t_embedder.linear2.bias"))


def _t_embed_silu_last(t, W):
    e = ref.timestep_embedding(np.asarray(t, dtype=np.float64) * ref.T_SCALE).astype(W.dtype)
    h = ref.linear(e, W("t_embedder.linear1.weight"), W("t_embedder.linear1.bias"))
    return ref.silu(ref.linear(h, W("t_embedder.linear2.weight"), W("t_embedder.linear2.bias")))


def _sinusoid_sin_first(t_in, width=256, max_period=10000.0):
    e = ref.__dict__["_orig_timestep_embedding"](t_in, width, max_period)
    return np.concatenate([e[:, width // 2:], e[:, :width // 2]], axis=-1)


def _sinusoid_full_width_exponent(t_in, width=256, max_period=10000.0):
    k = np.arange(width // 2, dtype=np.float64)
    args = np.asarray(t_in, dtype=np.float64)[:, None] * np.exp(-np.log(max_period) * k / width)[None, :]
    return np.concatenate([np.cos(args), np.sin(args)], axis=-1)


def _final_layer_raw_c(x_img, W, c):
    s = ref.linear(c, W("final_layer.adaLN_modulation.weight"), W("final_layer.adaLN_modulation.bias"))
    return ref.linear(ref.layer_norm(x_img) * (1.0 + s), W("final_layer.linear.weight"), W("final_layer.linear.bias"))


def _final_layer_scale_without_one(x_img, W, c):
    s = ref.linear(ref.silu(c), W("final_layer.adaLN_modulation.weight"), W("final_layer.adaLN_modulation.bias"))
    return ref.linear(ref.layer_norm(x_img) * s, W("final_layer.linear.weight"), W("final_layer.linear.bias"))


def _final_layer_uncentred(x_img, W, c):
    s = ref.linear(ref.silu(c), W("final_layer.adaLN_modulation.weight"), W("final_layer.adaLN_modulation.bias"))
    y = x_img / np.sqrt(np.mean(x_img * x_img, axis=-1, keepdims=True) + ref.FINAL_EPS) * (1.0 + s)
    return ref.linear(y, W("final_layer.linear.weight"), W("final_layer.linear.bias"))


T_PINS = [tb.test_t_embed_closed_form, lambda: [tb.test_t_embed_matches_brute_force(t) for t in (0.3, 0.875)]]
F_PINS = [tb.test_final_layer_closed_form, tb.test_final_layer_matches_brute_force]

MUTATIONS = [
    ("apply_rope", _rope_half_split, [tp.test_rope_matches_explicit_rotation_matrix]),
    ("apply_rope", _rope_clockwise, [tp.test_rope_complex_product_convention]),
    ("rope_angles", _angles_wrong_exponent, [tp.test_rope_frequencies_closed_form]),
    ("attention", _attention_keys_softmax, [tp.test_attention_matches_brute_force]),
    ("attention", _attention_no_scale, [tp.test_attention_matches_brute_force]),
    ("rms_norm", _rms_no_eps_sqrt, [tp.test_rms_norm_closed_form]),
    ("patchify", _patchify_channel_slowest, [ts.test_patchify_matches_index_loop_and_roundtrips]),
    ("block_forward", _block_without_post_norm,
     [lambda: tb.test_post_norm_makes_output_rescaling_exact(True)]),
    ("t_embed", _t_embed_no_scale, T_PINS),
    ("t_embed", _t_embed_silu_last, T_PINS),
    ("timestep_embedding", _sinusoid_sin_first, T_PINS + [tp.test_timestep_embedding_values]),
    ("timestep_embedding", _sinusoid_full_width_exponent, T_PINS + [tp.test_timestep_embedding_values]),
    ("final_layer", _final_layer_raw_c, F_PINS),
    ("final_layer", _final_layer_scale_without_one, F_PINS),
    ("final_layer", _final_layer_uncentred, F_PINS),
]


@pytest.mark.parametrize("name,bad,pins", MUTATIONS, ids=[f"{m[0]}:{m[1].__name__}" for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, bad, pins):
    monkeypatch.setitem(ref.__dict__, f"_orig_{name}", getattr(ref, name))
    monkeypatch.setattr(ref, name, bad)
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed == len(pins), f"planted {bad.__name__} in {name} was not caught"
