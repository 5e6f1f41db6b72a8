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


def _denoise_case(d, lat_hw, s_txt, n_steps, seed, guidance=None):
    from stream_diffusion_transformer_b200 import model
    from oracle import scheduler_ref as sch
    bits = zi.make_weights(d, seed=seed)
    dit = model.DiT(model.make_config(d), lambda keys: {k: bits[k] for k in keys})
    lat = zi.make_latent(d, 1, lat_hw, lat_hw, seed=seed)
    txt = zi.make_text(d, 1, s_txt, seed=seed)
    txt_u = zi.make_text(d, 1, s_txt, seed=seed, uncond=True)
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    got = dit.denoise(torch.from_numpy(lat).cuda(), dev(txt), n_steps=n_steps, shift=3.0, guidance=guidance,
                      txt_uncond=dev(txt_u) if guidance is not None else None)
    torch.cuda.synchronize()
    W = ref.Weights(bits)
    tc = zi.bf16_bits_to_f32(txt).astype(np.float64)
    tu = zi.bf16_bits_to_f32(txt_u).astype(np.float64)

    def model_fn(x, t, uncond):
        return ref.model_forward(x, t, tu if uncond else tc, W, d)

    want = sch.denoise(lat.astype(np.float64), model_fn, n_steps, 3.0, guidance)
    return got.cpu().numpy().astype(np.float64), want, lat.astype(np.float64)


def test_turbo_loop_8_steps():
    """8-step FlowMatch-Euler loop (shift 3, t = 1 - sigma', output negated) at full width,
    1 + 1 + 2 blocks, 256 image + 128 text tokens; final latent against the oracle's loop."""
    d = dataclasses.replace(zi.FULL, n_noise=1, n_ctx=1, n_main=2)
    got, want, x0 = _denoise_case(d, 32, 128, 8, seed=3)
    assert_parity(got, want, rel=3e-2, cos=0.995, what="8-step loop final latent")
    assert_parity(got - x0, want - x0, rel=3e-2, cos=0.995, what="8-step loop latent change")


def test_cfg_loop_batch2():
    """Guidance 4: conditional and unconditional texts as one batch-2 forward per step."""
    got, want, x0 = _denoise_case(zi.TINY_R, 8, 16, 4, seed=4, guidance=4.0)
    assert_parity(got, want, rel=3e-2, cos=0.995, what="CFG loop final latent")
    assert_parity(got - x0, want - x0, rel=3e-2, cos=0.995, what="CFG loop latent change")


def test_variable_length_text_batch():
    """Prompts of 20 and 7 tokens padded to 20 (cap_pad_token rows, masked as keys):
    each element against the oracle's padded batch, and element 1 against the
    oracle run on its unpadded 7-token prompt alone."""
    from stream_diffusion_transformer_b200 import model
    d = zi.TINY_R
    bits = zi.make_weights(d, seed=5)
    dit = model.DiT(model.make_config(d), lambda keys: {k: bits[k] for k in keys})
    lat = zi.make_latent(d, 2, 10, 12, seed=5)
    txt = zi.make_text(d, 2, 20, seed=5)
    txt[1, 7:] = 0x7F80  # +inf bits in the padding rows: they must not reach the output
    tt = np.array([0.35, 0.6], dtype=np.float32)
    lens = [20, 7]
    out = dit.forward(torch.from_numpy(lat).cuda(), torch.from_numpy(tt).cuda(),
                      torch.from_numpy(txt.view(np.int16)).cuda().view(torch.bfloat16), txt_len=lens)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    W = ref.Weights(bits)
    tf = zi.bf16_bits_to_f32(txt).astype(np.float64)
    tf[1, 7:] = 0.0
    want = ref.model_forward(lat.astype(np.float64), tt.astype(np.float64), tf, W, d, txt_len=np.array(lens))
    for b in range(2):
        assert_parity(got[b], want[b], rel=3e-2, cos=0.995, what=f"varlen b={b} len={lens[b]}")
    alone = ref.model_forward(lat[1:].astype(np.float64), tt[1:].astype(np.float64), tf[1:, :7], W, d)
    assert_parity(got[1:], alone, rel=3e-2, cos=0.995, what="varlen b=1 vs unpadded alone")


def test_variable_length_cfg_loop_full_width():
    """CFG loop at full width (1 + 1 + 2 blocks, 256 image tokens): a 96-token prompt and
    a 9-token negative prompt padded to one 96-row batch-2 forward per step, against the
    oracle's loop that runs each branch on its own unpadded text."""
    from oracle import scheduler_ref as sch
    from stream_diffusion_transformer_b200 import model
    d = dataclasses.replace(zi.FULL, n_noise=1, n_ctx=1, n_main=2)
    bits = zi.make_weights(d, seed=6, threads=8)
    dit = model.DiT(model.make_config(d), lambda keys: {k: bits[k] for k in keys})
    lat = zi.make_latent(d, 1, 32, 32, seed=6)
    txt = zi.make_text(d, 1, 96, seed=6)
    txt_u = zi.make_text(d, 1, 9, seed=6, uncond=True)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    got = dit.denoise(torch.from_numpy(lat).cuda(), dev(txt), n_steps=3, shift=3.0, guidance=4.0,
                      txt_uncond=dev(txt_u))
    torch.cuda.synchronize()
    W = ref.Weights(bits)
    tc = zi.bf16_bits_to_f32(txt).astype(np.float64)
    tu = zi.bf16_bits_to_f32(txt_u).astype(np.float64)

    def model_fn(x, t, uncond):
        return ref.model_forward(x, t, tu if uncond else tc, W, d)

    x0 = lat.astype(np.float64)
    want = sch.denoise(x0, model_fn, 3, 3.0, 4.0)
    g = got.cpu().numpy().astype(np.float64)
    assert_parity(g, want, rel=3e-2, cos=0.995, what="varlen CFG loop final latent")
    assert_parity(g - x0, want - x0, rel=3e-2, cos=0.995, what="varlen CFG loop latent change")


def test_graph_captured_loop_matches_eager():
    """The 8-step loop captured as one CUDA graph (CFG with a padded short negative
    prompt) gives bit-identical latents to the eager loop, on two different inputs."""
    from stream_diffusion_transformer_b200 import model
    d = zi.TINY_R
    bits = zi.make_weights(d, seed=9)
    dit = model.DiT(model.make_config(d), lambda keys: {k: bits[k] for k in keys})
    txt = zi.make_text(d, 1, 24, seed=9)
    txt_u = zi.make_text(d, 1, 5, seed=9, uncond=True)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    g = model.DenoiseGraph(dit, (1, d.in_ch, 12, 10), dev(txt), n_steps=8, guidance=4.0, txt_uncond=dev(txt_u))
    for seed in (10, 11):
        lat = torch.from_numpy(zi.make_latent(d, 1, 12, 10, seed=seed)).cuda()
        eager = dit.denoise(lat, dev(txt), n_steps=8, guidance=4.0, txt_uncond=dev(txt_u))
        got = g.run(lat)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        assert torch.equal(got, eager)


@pytest.mark.parametrize("t", [0.0, 1.0])
def test_degenerate_one_image_token_one_text_token(t):
    """The smallest sequence: a 2x2 latent (one image token) and one text token, at the
    timestep's end points t = 0 and t = 1; batch 2 with identical elements gives
    identical outputs."""
    from stream_diffusion_transformer_b200 import model
    d = zi.TINY_R
    bits = zi.make_weights(d, seed=12)
    dit = model.DiT(model.make_config(d), lambda keys: {k: bits[k] for k in keys})
    lat = np.repeat(zi.make_latent(d, 1, 2, 2, seed=12), 2, axis=0)
    txt = np.repeat(zi.make_text(d, 1, 1, seed=12), 2, axis=0)
    tt = np.array([t, t], dtype=np.float32)
    out = dit.forward(torch.from_numpy(np.ascontiguousarray(lat)).cuda(), torch.from_numpy(tt).cuda(),
                      torch.from_numpy(np.ascontiguousarray(txt).view(np.int16)).cuda().view(torch.bfloat16))
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    np.testing.assert_array_equal(got[0], got[1])
    want = ref.model_forward(lat[:1].astype(np.float64), tt[:1].astype(np.float64),
                             zi.bf16_bits_to_f32(txt[:1]).astype(np.float64), ref.Weights(bits), d)
    assert_parity(got[:1].astype(np.float64), want, rel=3e-2, cos=0.995, what=f"1 + 1 tokens, t={t}")


def test_empty_calls_enqueue_nothing():
    """Zero-sized work is accepted and launches nothing (no kernel, no error)."""
    from stream_diffusion_transformer_b200 import abi, model
    a = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")  # real buffers; M = 0 rows are used
    b = torch.zeros((256, 64), dtype=torch.bfloat16, device="cuda")
    c = torch.zeros((1, 256), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros(16, device="cuda")
    with abi.Profile(capacity=8) as prof:
        abi.call("zi_gemm_bf16", model._p(a), model._p(b), model._p(c), 0, 256, 64, model._stream())
        model.euler_step(x[:0], x[:0], None, 0.0, 1.0, 0.5)
    torch.cuda.synchronize()
    assert prof.kinds == []
