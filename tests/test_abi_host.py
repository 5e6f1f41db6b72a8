"""The C-ABI library loads, exports every declared entry point, and its host-only
logic (status strings, defaults, workspace sizes, sigma schedule, argument
checks) behaves -- all without a GPU."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from conftest import ROOT
from oracle import scheduler_ref as sch

HEADER = os.path.join(ROOT, "include", "zimage_dit.h")


@pytest.fixture(scope="module")
def abi():
    from stream_diffusion_transformer_b200 import abi as a, build
    build.build()
    a.lib()
    return a


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^ZI_API\s+[\w\s\*]+?\b(zi_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("zi_block_forward", "zi_model_forward", "zi_euler_step"):
        assert required in names
    assert len(names) >= 20


def test_library_exports_every_declared_symbol(abi):
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (zi_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    assert set(names) == set(abi.exported_symbols())
    for n in names:
        assert hasattr(abi.lib(), n)


def test_status_strings_and_version(abi):
    for s in range(-7, 1):
        assert abi.status_string(s) not in ("", "unknown status")
    assert abi.status_string(-99) == "unknown status"
    assert abi.lib().zi_version() >= 100


def test_default_config_is_zimage(abi):
    c = abi.config_default()
    assert (c.dim, c.heads, c.head_dim, c.ffn, c.cap_dim) == (3840, 30, 128, 10240, 2560)
    assert (c.t_freq, c.t_mid, c.in_ch, c.patch) == (256, 1024, 16, 2)
    assert (c.n_noise, c.n_ctx, c.n_main) == (2, 2, 30)
    assert list(c.rope_axes) == [32, 48, 48]
    assert (c.rope_theta, c.t_scale) == (256.0, 1000.0)
    assert c.norm_eps == pytest.approx(1e-5) and c.final_eps == pytest.approx(1e-6)


def test_ffn_padding(abi):
    assert abi.ffn_padded(10240) == 10240
    assert abi.ffn_padded(688) == 768
    assert abi.ffn_padded(1) == 128


def test_sigmas_match_oracle(abi):
    for n, shift in ((8, 3.0), (1, 3.0), (30, 6.0), (4, 1.0)):
        np.testing.assert_allclose(abi.sigmas(n, shift), sch.sigmas(n, shift), rtol=0, atol=1e-15)


def test_timesteps_match_oracle(abi):
    """zi_timesteps gives the model timestep of every call, 1 - sigma'_i rounded to fp32 once
    (z-image-turbo-mnn card, "Scheduler"), and nothing for the zero-sigma end point."""
    for n, shift in ((8, 3.0), (1, 3.0), (30, 6.0), (4, 1.0)):
        got = abi.timesteps(n, shift)
        want = sch.timesteps(sch.sigmas(n, shift)).astype(np.float32)
        assert len(got) == n
        np.testing.assert_array_equal(np.array(got, dtype=np.float32), want)
    # the 8-step Turbo schedule: t = 1 - 3k/(8 + 2k) for k = 8 .. 1, starting at 0 (pure noise)
    got = abi.timesteps(8, 3.0)
    assert got[0] == 0.0
    np.testing.assert_allclose(got, [1.0 - 3.0 * k / (8.0 + 2.0 * k) for k in range(8, 0, -1)], rtol=0, atol=6e-8)
    L = abi.lib()
    assert L.zi_timesteps(0, 3.0, (ctypes.c_float * 1)()) == abi.ZI_ERR_ARG
    assert L.zi_timesteps(4, 0.0, (ctypes.c_float * 4)()) == abi.ZI_ERR_ARG
    assert L.zi_timesteps(4, 3.0, None) == abi.ZI_ERR_ARG


def test_workspace_sizes(abi):
    c = abi.config_default()
    ws_block = abi.block_workspace_size(c, 1, 1152)
    ws_model = abi.model_workspace_size(c, 1, 128, 128, 32)
    S = 4128
    # at least the activations the forward keeps (x fp32, h/att/o bf16, qkv, u)
    assert ws_model >= S * 3840 * (4 + 2 * 3 + 2 * 3) + S * 10240 * 2
    assert ws_model < 2 * S * 3840 * (4 + 2 * 3 + 2 * 3) + 2 * S * 10240 * 2 + (64 << 20)
    assert ws_block >= 1152 * 3840 * 2 * 6
    assert abi.model_workspace_size(c, 2, 256, 256, 512) > ws_model


def test_argument_checks_need_no_gpu(abi):
    """Every call below is rejected by the host-side checks before any device work
    (fake pointers are only ever paired with a shape or alignment that fails)."""
    c = abi.config_default()
    bad = abi.config_default()
    bad.head_dim = 64
    with pytest.raises(abi.ZiError) as e:
        abi.block_workspace_size(bad, 1, 16)
    assert e.value.status == abi.ZI_ERR_SHAPE
    bad = abi.config_default()
    bad.rope_axes[0] = 30
    with pytest.raises(abi.ZiError):
        abi.block_workspace_size(bad, 1, 16)
    with pytest.raises(abi.ZiError) as e:
        abi.model_workspace_size(c, 1, 127, 128, 32)
    assert e.value.status == abi.ZI_ERR_SHAPE
    L = abi.lib()
    assert L.zi_gemm_bf16(None, None, None, 128, 256, 64, None) == abi.ZI_ERR_ARG
    assert L.zi_gemm_bf16(ctypes.c_void_p(8), ctypes.c_void_p(32), ctypes.c_void_p(48), 128, 256, 64,
                          None) == abi.ZI_ERR_ALIGN
    assert L.zi_gemm_bf16(ctypes.c_void_p(16), ctypes.c_void_p(32), ctypes.c_void_p(48), 128, 200, 64,
                          None) == abi.ZI_ERR_SHAPE
    assert L.zi_attention(None, None, 1, 16, 2, None) == abi.ZI_ERR_ARG
    assert L.zi_euler_step(None, None, None, 0.0, 1.0, 0.5, 4, None) == abi.ZI_ERR_ARG
    huge = 1 << 40  # more than 2^31 - 1 blocks of 256 threads
    assert L.zi_euler_step(ctypes.c_void_p(16), ctypes.c_void_p(32), None, 0.0, 1.0, 0.5, huge,
                           None) == abi.ZI_ERR_SHAPE
    assert L.zi_exp2_poly(ctypes.c_void_p(16), ctypes.c_void_p(32), 2 * huge, None) == abi.ZI_ERR_SHAPE
    assert L.zi_exp2_poly(None, None, 0, None) == abi.ZI_OK
    assert L.zi_timesteps(0, 3.0, None) == abi.ZI_ERR_ARG
    assert L.zi_timesteps(8, 0.0, (ctypes.c_float * 8)()) == abi.ZI_ERR_ARG
    assert L.zi_block_forward(ctypes.byref(c), None, None, None, 1, 16, None, None, None, 0, None) == abi.ZI_ERR_ARG
    assert L.zi_sigmas(0, 3.0, None) == abi.ZI_ERR_ARG
    assert L.zi_watchdog_selftest(0, None) == abi.ZI_ERR_ARG
    assert L.zi_watchdog_selftest(3000000, None) == abi.ZI_ERR_ARG


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    from stream_diffusion_transformer_b200 import abi as a
    monkeypatch.setattr(a, "_lib", None)
    monkeypatch.setattr(a, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        a.lib()
