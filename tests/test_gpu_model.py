"""GPU parity of zi_model_forward (the full transformer) against the CPU oracle.

Bar: full-stack output cosine >= 0.995 against the fp64 oracle on the same
bf16 weights and inputs; rel-L2 <= 3e-2 is also checked."""
import dataclasses

import numpy as np
import pytest

from gpu_util import assert_parity, require_gpu, torch
import zimage_inputs as zi
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


def run_model(d, batch, lat_h, lat_w, s_txt, t, seed):
    from stream_diffusion_transformer_b200 import model
    bits = zi.make_weights(d, seed=seed)
    dit = model.DiT(model.make_config(d), lambda keys: {k: bits[k] for k in keys})
    lat = zi.make_latent(d, batch, lat_h, lat_w, seed=seed)
    txt = zi.make_text(d, batch, s_txt, seed=seed)
    tt = np.asarray(t, dtype=np.float32)
    out = dit.forward(torch.from_numpy(lat).cuda(), torch.from_numpy(tt).cuda(),
                      torch.from_numpy(txt.view(np.int16)).cuda().view(torch.bfloat16))
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    want = ref.model_forward(lat.astype(np.float64), tt.astype(np.float64), zi.bf16_bits_to_f32(txt).astype(np.float64),
                             ref.Weights(bits), d)
    return got, want


def test_tiny_model():
    """The tiny configuration: 1 modulated block, hidden 256, 16x16x16 latent -> 64 + 32 tokens, t = 0.5."""
    got, want = run_model(zi.TINY, 1, 16, 16, 32, [0.5], seed=0)
    assert_parity(got, want, rel=3e-2, cos=0.995, what="tiny model")


def test_tiny_model_with_refiners_batch2_ragged():
    """One block of each kind, batch 2, 5 x 6 image tokens and 20 text tokens per element."""
    got, want = run_model(zi.TINY_R, 2, 10, 12, 20, [0.3, 0.8], seed=1)
    for b in range(2):
        assert_parity(got[b], want[b], rel=3e-2, cos=0.995, what=f"tiny+refiners b={b}")


def test_full_width_shallow_model():
    """Full width (3840, 30 heads, FFN 10240, text 2560) with 1 + 1 + 2 blocks, 256 + 32 tokens."""
    d = dataclasses.replace(zi.FULL, n_noise=1, n_ctx=1, n_main=2)
    got, want = run_model(d, 1, 32, 32, 32, [0.25], seed=2)
    assert_parity(got, want, rel=3e-2, cos=0.995, what="full-width shallow model")
