"""Pins of the oracle's structure against the sizes the pages print."""
import numpy as np
import pytest

from conftest import read_golden
import zimage_inputs as zi
from oracle import brute, zimage_ref as ref


def _golden_dict(name):
    return {r[0]: r[1:] for r in read_golden(name)}


def test_key_and_parameter_count():
    g = _golden_dict("param_counts.txt")
    specs = zi.weight_specs(zi.FULL)
    assert len(specs) == int(g["keys"][0])
    n = sum(int(np.prod(s)) for _, s, _ in specs)
    assert n == int(g["params"][0])
    # 12.31 GB in bf16 (2 bytes per parameter), as printed (decimal GB, 2 places)
    assert round(2 * n / 1e9, 2) == float(g["bf16_gigabytes"][0])


def test_final_layer_size():
    g = _golden_dict("param_counts.txt")
    specs = {k: s for k, s, _ in zi.weight_specs(zi.FULL)}
    fl = [k for k in specs if k.startswith("final_layer.")]
    n = sum(int(np.prod(specs[k])) for k in fl)
    assert round(n / 1e6, 1) == float(g["final_layer_params_millions"][0])
    assert list(specs["final_layer.linear.weight"]) == [int(v) for v in g["final_layer_linear_shape"]]


def test_context_refiner_has_no_modulation():
    specs = [k for k, _, _ in zi.weight_specs(zi.FULL)]
    ctx = [k for k in specs if k.startswith("context_refiner.0.")]
    main = [k for k in specs if k.startswith("layers.0.")]
    assert len(ctx) == 13 and len(main) == 15
    assert not any("adaLN" in k for k in ctx)


@pytest.mark.parametrize("row", read_golden("token_counts.txt"))
def test_token_counts(row):
    side, ch, lh, lw, tokens = (int(v) for v in row)
    assert side // 8 == lh == lw
    lat = np.zeros((1, ch, lh, lw), dtype=np.float32)
    tok = ref.patchify(lat, 2)
    assert tok.shape == (1, tokens, 4 * ch)


def test_patchify_matches_index_loop_and_roundtrips():
    rng = np.random.default_rng(1)
    lat = rng.standard_normal((2, 16, 6, 8))
    tok = ref.patchify(lat)
    np.testing.assert_array_equal(tok, brute.patchify_loop(lat))
    np.testing.assert_array_equal(ref.unpatchify(tok, 16, 6, 8), lat)


def test_position_ids_match_loop():
    for s_txt, gh, gw in [(32, 64, 64), (1, 1, 1), (7, 3, 5), (512, 128, 128)]:
        got = ref.position_ids(s_txt, gh, gw)
        assert got.dtype == np.int32
        np.testing.assert_array_equal(got, np.array(brute.position_ids_loop(s_txt, gh, gw), dtype=np.int32))
    ids = ref.position_ids(512, 128, 128)
    assert ids[:, 0].max() == 513 and ids[:, 1].max() == 127 and ids[:, 2].max() == 127


def test_every_key_is_consumed_by_the_forward():
    d = zi.TINY_R
    W = ref.Weights(zi.make_weights(d, seed=3))
    lat = zi.make_latent(d, 1, 4, 4, seed=3)
    txt = zi.bf16_bits_to_f32(zi.make_text(d, 1, 3, seed=3))
    out = ref.model_forward(lat, np.array([0.5]), txt, W, d)
    assert out.shape == lat.shape
    unused = set(W.bits) - W.used
    # pad tokens only fill padding, which no configuration here needs
    assert unused == {"x_pad_token", "cap_pad_token"}
