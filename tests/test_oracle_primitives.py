"""Pins of the oracle's primitives: closed forms, invariants and brute force."""
import math

import numpy as np
import pytest

from oracle import brute, zimage_ref as ref


# ------------------------------------------------------------------ RMSNorm

def test_rms_norm_closed_form():
    # x = [3, 4]: mean square 12.5, so y = g * x / sqrt(12.5 + eps)
    x = np.array([3.0, 4.0])
    g = np.array([2.0, 0.5])
    y = ref.rms_norm(x, g, eps=0.0)
    assert y == pytest.approx([2 * 3 / math.sqrt(12.5), 0.5 * 4 / math.sqrt(12.5)], rel=1e-15)


def test_rms_norm_scale_invariance_and_brute():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 64)) * 3.0
    g = 1 + 0.02 * rng.standard_normal(64)
    for alpha in (0.5, 7.0, 1e3):
        np.testing.assert_allclose(ref.rms_norm(alpha * x, g), ref.rms_norm(x, g), rtol=2e-5)
    for r in range(5):
        np.testing.assert_allclose(ref.rms_norm(x[r], g), brute.rms_norm_row(list(x[r]), list(g), 1e-5), rtol=1e-13)


def test_layer_norm_shift_and_scale_invariance():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((4, 48))
    y = ref.layer_norm(x)
    np.testing.assert_allclose(y.mean(axis=-1), 0, atol=1e-13)
    np.testing.assert_allclose((y * y).mean(axis=-1), 1, rtol=1e-5)
    np.testing.assert_allclose(ref.layer_norm(5.0 * x + 3.0), y, rtol=1e-6, atol=1e-6)


# ------------------------------------------------------------------ RoPE

def test_rope_frequencies_closed_form():
    # theta = 256 = 2^8, so omega_j = 2^(-16 j / d_axis): 2^(-j/2) on the 32-wide
    # axis and 2^(-j/3) on the 48-wide axes.
    ang = ref.rope_angles(np.array([[1, 0, 0]]))[0]
    assert ang[2] == pytest.approx(0.5, rel=1e-15)     # axis 0, j = 2
    assert ang[1] == pytest.approx(2 ** -0.5, rel=1e-15)
    assert np.all(ang[16:] == 0)
    ang = ref.rope_angles(np.array([[0, 1, 0]]))[0]
    assert ang[16 + 3] == pytest.approx(0.5, rel=1e-15)  # axis 1, j = 3
    assert np.all(ang[:16] == 0) and np.all(ang[40:] == 0)
    ang = ref.rope_angles(np.array([[0, 0, 5]]))[0]
    assert ang[40 + 6] == pytest.approx(5 * 0.25, rel=1e-15)  # axis 2, j = 6
    assert np.all(ang[:40] == 0)


def test_rope_complex_product_convention():
    # pair (1, 0) rotated by +pi/2 becomes (0, 1): counter-clockwise, i.e. (a + ib) e^{i angle}
    x = np.zeros((1, 1, 128))
    x[0, 0, 0] = 1.0
    ang = np.zeros((1, 64))
    ang[0, 0] = math.pi / 2
    y = ref.apply_rope(x, ang)
    assert y[0, 0, 0] == pytest.approx(0.0, abs=1e-15)
    assert y[0, 0, 1] == pytest.approx(1.0, abs=1e-15)


def test_rope_matches_explicit_rotation_matrix():
    rng = np.random.default_rng(2)
    pos = np.array([[3, 7, 11], [33, 0, 0], [0, 127, 5]])
    x = rng.standard_normal((3, 2, 128))
    y = ref.apply_rope(x, ref.rope_angles(pos))
    for s in range(3):
        R = brute.rope_matrix(list(pos[s]))
        for h in range(2):
            np.testing.assert_allclose(y[s, h], R @ x[s, h], rtol=1e-12, atol=1e-12)


def test_rope_norm_identity_and_relative_position():
    rng = np.random.default_rng(3)
    pos = rng.integers(0, 200, size=(6, 3))
    q = rng.standard_normal((6, 3, 128))
    k = rng.standard_normal((6, 3, 128))
    ang = ref.rope_angles(pos)
    rq, rk = ref.apply_rope(q, ang), ref.apply_rope(k, ang)
    # norm preserved per pair
    np.testing.assert_allclose((rq.reshape(6, 3, 64, 2) ** 2).sum(-1), (q.reshape(6, 3, 64, 2) ** 2).sum(-1), rtol=1e-12)
    # position 0 is the identity
    np.testing.assert_array_equal(ref.apply_rope(q, ref.rope_angles(np.zeros((6, 3), int))), q)
    # scores depend on position differences only
    shift = np.array([[17, 4, 9]])
    ang2 = ref.rope_angles(pos + shift)
    s1 = np.einsum("shd,thd->hst", rq, rk)
    s2 = np.einsum("shd,thd->hst", ref.apply_rope(q, ang2), ref.apply_rope(k, ang2))
    np.testing.assert_allclose(s1, s2, rtol=1e-9, atol=1e-9)


# ------------------------------------------------------------------ attention

def test_attention_matches_brute_force():
    rng = np.random.default_rng(4)
    S, H, hd = 24, 2, 128
    q, k, v = (rng.standard_normal((S, H, hd)) for _ in range(3))
    out = ref.attention(q, k, v)
    for h in range(H):
        bf = np.array(brute.attention_head(q[:, h].tolist(), k[:, h].tolist(), v[:, h].tolist()))
        np.testing.assert_allclose(out[:, h], bf, rtol=1e-11, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(5)
    S, hd = 10, 128
    q = rng.standard_normal((S, 1, hd))
    v = rng.standard_normal((S, 1, hd))
    # identical keys: uniform weights, output = mean of V
    k = np.tile(rng.standard_normal((1, 1, hd)), (S, 1, 1))
    np.testing.assert_allclose(ref.attention(q, k, v)[:, 0], np.tile(v[:, 0].mean(0), (S, 1)), rtol=1e-12)
    # one key aligned with every query and very large: output = that key's value
    k = np.zeros((S, 1, hd))
    q = np.ones((S, 1, hd))
    k[3, 0, :] = 50.0
    np.testing.assert_allclose(ref.attention(q, k, v)[:, 0], np.tile(v[3, 0], (S, 1)), rtol=1e-12)


# ------------------------------------------------------------------ timestep embedding

def test_timestep_embedding_values():
    e = ref.timestep_embedding(np.array([0.0, 100.0]))
    np.testing.assert_array_equal(e[0, :128], 1.0)
    np.testing.assert_array_equal(e[0, 128:], 0.0)
    # f_0 = 1, f_64 = 10000^(-1/2) = 0.01
    assert e[1, 0] == pytest.approx(math.cos(100.0), abs=1e-12)
    assert e[1, 64] == pytest.approx(math.cos(1.0), abs=1e-12)
    assert e[1, 128 + 64] == pytest.approx(math.sin(1.0), abs=1e-12)


def test_silu_closed_form():
    assert ref.silu(np.array([0.0]))[0] == 0.0
    assert ref.silu(np.array([1.0]))[0] == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
