"""Pins of the e4m3 oracle (oracle/fp8_ref.py) against the format's definition and
against properties the quantised product must have; no GPU."""
import numpy as np
import pytest

import zimage_inputs as zi
from oracle import fp8_ref as f8
from oracle import zimage_ref as ref


def test_decode_closed_forms():
    """Values fixed by the e4m3 layout (bias 7, 3 mantissa bits, subnormals m 2^-9)."""
    cases = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x3C: 1.5,
             0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0x77: 240.0, 0xB8: -1.0, 0xFE: -448.0}
    for code, want in cases.items():
        assert f8.e4m3_decode(np.array([code]))[0] == want, hex(code)
    assert np.isnan(f8.e4m3_decode(np.array([0x7F, 0xFF]))).all()
    pos = f8.e4m3_decode(np.arange(0x7F))
    assert np.all(np.diff(pos) > 0) and len(np.unique(pos)) == 127


def test_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    assert np.array_equal(f8.e4m3_encode(f8.e4m3_decode(codes)), codes)


def test_round_to_nearest_even_and_saturation():
    # midpoints go to the code with an even mantissa
    assert f8.e4m3_encode(np.array([1.0625]))[0] == 0x38      # between 1.0 (0x38) and 1.125 (0x39)
    assert f8.e4m3_encode(np.array([1.1875]))[0] == 0x3A      # between 1.125 and 1.25 (0x3A)
    assert f8.e4m3_encode(np.array([1.5 * 2.0 ** -9]))[0] == 0x02
    assert f8.e4m3_encode(np.array([0.5 * 2.0 ** -9]))[0] == 0x00
    assert f8.e4m3_encode(np.array([0.50001 * 2.0 ** -9]))[0] == 0x01
    # just off a midpoint goes to the nearer value
    assert f8.e4m3_encode(np.array([1.0626]))[0] == 0x39
    # beyond the largest finite value: saturate
    assert f8.e4m3_encode(np.array([464.0, 1000.0, -1e6]))[:].tolist() == [0x7E, 0x7E, 0xFE]
    assert f8.e4m3_encode(np.array([-0.0, -1e-12]))[:].tolist() == [0x80, 0x80]


def test_encode_is_nearest_by_brute_force():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(4000) * np.exp2(rng.uniform(-12, 9, 4000))
    codes = f8.e4m3_encode(x)
    table = f8.e4m3_decode(np.arange(0x7F))
    for v, c in zip(x, codes):
        err = abs(min(abs(v), 448.0) - table)
        assert abs(abs(f8.e4m3_decode(np.array([c]))[0]) - min(abs(v), 448.0)) == err.min()


def test_quantize_rows_properties():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((6, 300)).astype(np.float32)
    x[2] = 0.0
    codes, scale = f8.quantize_rows(x)
    assert scale.dtype == np.float32 and codes.dtype == np.uint8
    assert scale[2] == 1.0 and not codes[2].any()
    for r in (0, 1, 3):
        i = np.argmax(np.abs(x[r]))
        assert codes[r, i] & 0x7F == 0x7E                   # the row's largest magnitude maps to 448
        assert scale[r] == np.float32(np.abs(x[r]).max() / np.float32(448.0))
    # a power-of-two rescaling of a row changes only its scale
    c2, s2 = f8.quantize_rows(x * np.float32(8.0))
    assert np.array_equal(c2, codes) and np.allclose(s2[[0, 1, 3]], 8 * scale[[0, 1, 3]], rtol=0)
    # quantise-dequantise error: half a step of 3 mantissa bits, relative, for normal values
    back = f8.dequantize_rows(codes, scale)
    y = x.astype(np.float64)
    normal = np.abs(y) >= 2.0 ** -6 * scale[:, None]
    assert np.all(np.abs(back - y)[normal] <= 2.0 ** -4 * np.abs(y)[normal] * (1 + 1e-6))


def test_fp8_linear_is_exact_on_representable_operands():
    """Operands already on the e4m3 grid with a 448 entry in every row: scales are 1
    and the quantised product is the plain product."""
    rng = np.random.default_rng(2)
    a = f8.e4m3_decode(rng.integers(0, 0x7E, (5, 64)))
    w = f8.e4m3_decode(rng.integers(0, 0x7E, (7, 64)))
    a[:, 0] = 448.0
    w[:, 3] = -448.0
    np.testing.assert_array_equal(f8.fp8_linear(a, w), a @ w.T)


def test_fp8_block_tracks_the_bf16_block():
    """The e4m3 block stays close to the bf16 block (rel-L2 of the block update a few
    percent: 3 mantissa bits) but is not identical to it."""
    d = zi.TINY_R
    bits = zi.make_weights(d, seed=3)
    W = ref.Weights(bits)
    x = zi.make_stream(d, 1, 40, seed=3)[0].astype(np.float64)
    c = zi.make_cond(d, 1, seed=3)[0].astype(np.float64)
    ang = ref.rope_angles(ref.position_ids(8, 4, 8), d.rope_axes)
    y16 = ref.block_forward(x, W, "layers.0", d, ang, c)
    y8 = f8.block_forward(x, W, "layers.0", d, ang, c)
    rel = np.linalg.norm((y8 - x) - (y16 - x)) / np.linalg.norm(y16 - x)
    assert 1e-4 < rel < 0.1


def test_all_projection_block_moves_further_from_bf16():
    """all=True also quantises the output projection and FFN w2: the block's update moves
    further from the bf16 block than with two e4m3 projections, and stays within 20%."""
    d = zi.TINY_R
    bits = zi.make_weights(d, seed=5)
    W = ref.Weights(bits)
    x = zi.make_stream(d, 1, 24, seed=5)[0].astype(np.float64)
    c = zi.make_cond(d, 1, seed=5)[0].astype(np.float64)
    ang = ref.rope_angles(ref.position_ids(8, 4, 4), d.rope_axes)
    y16 = ref.block_forward(x, W, "layers.0", d, ang, c)
    y8 = f8.block_forward(x, W, "layers.0", d, ang, c)
    y8a = f8.block_forward(x, W, "layers.0", d, ang, c, all=True)
    e = lambda y: np.linalg.norm((y - x) - (y16 - x)) / np.linalg.norm(y16 - x)
    assert 0 < e(y8) < e(y8a) < 0.2


@pytest.mark.parametrize("all_", [False, True])
def test_block_forward_rows_equals_whole_block(all_):
    """Selecting query rows gives exactly those rows of the whole-sequence e4m3 block
    (quantisation is per row, attention takes keys and values from every row)."""
    d = zi.TINY_R
    W = ref.Weights(zi.make_weights(d, seed=6))
    x = zi.make_stream(d, 1, 40, seed=6)[0].astype(np.float64)
    c = zi.make_cond(d, 1, seed=6)[0].astype(np.float64)
    ang = ref.rope_angles(ref.position_ids(8, 4, 8), d.rope_axes)
    rows = np.array([0, 3, 17, 31, 39])
    whole = f8.block_forward(x, W, "layers.0", d, ang, c, all=all_)
    np.testing.assert_allclose(f8.block_forward_rows(x, W, "layers.0", d, ang, c, rows, all=all_), whole[rows],
                               rtol=1e-12, atol=1e-12)
