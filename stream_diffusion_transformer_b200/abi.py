"""ctypes binding of libzimage_dit.so (argument marshalling only).

Every function here forwards to the C entry point of the same name declared in
include/zimage_dit.h; a non-zero status raises ZiError.  There is no fallback:
if the shared library is missing or a call fails, the error propagates.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int, c_size_t, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libzimage_dit.so")

ZI_OK, ZI_ERR_ARG, ZI_ERR_SHAPE, ZI_ERR_ALIGN, ZI_ERR_WORKSPACE, ZI_ERR_CUDA, ZI_ERR_TIMEOUT, ZI_ERR_DEVICE = (
    0, -1, -2, -3, -4, -5, -6, -7)
ZI_ERR_SCRATCH_LIMIT = -8
STATIC_SCRATCH_BYTES = 128 * 1024 * 1024


class ZiError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed: {text} (status {status})")
        self.status = status


class ZiConfig(ctypes.Structure):
    _fields_ = [
        ("dim", c_int), ("heads", c_int), ("head_dim", c_int), ("ffn", c_int), ("cap_dim", c_int),
        ("t_freq", c_int), ("t_mid", c_int), ("in_ch", c_int), ("patch", c_int),
        ("n_noise", c_int), ("n_ctx", c_int), ("n_main", c_int), ("rope_axes", c_int * 3),
        ("rope_theta", c_float), ("norm_eps", c_float), ("final_eps", c_float), ("t_scale", c_float),
    ]


BLOCK_FIELDS = ("w_qkv", "w_out", "w13", "w2", "g_attn1", "g_attn2", "g_ffn1", "g_ffn2", "g_q", "g_k",
                "w_ada", "b_ada", "w_qkv8", "s_qkv", "w13_8", "s_13", "w_out8", "s_out", "w2_8", "s_2")


class ZiBlockWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in BLOCK_FIELDS]


MODEL_FIELDS = ("x_emb_w", "x_emb_b", "cap_norm", "cap_w", "cap_b", "t_w1", "t_b1", "t_w2", "t_b2",
                "final_ada_w", "final_ada_b", "final_w", "final_b")


class ZiModelWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in MODEL_FIELDS] + [
        ("noise", POINTER(ZiBlockWeights)), ("ctx", POINTER(ZiBlockWeights)), ("main", POINTER(ZiBlockWeights)),
        ("cap_pad", c_void_p)]


_SIGS = {
    "zi_status_string": (c_char_p, [c_int]),
    "zi_version": (c_int, []),
    "zi_config_default": (c_int, [POINTER(ZiConfig)]),
    "zi_ffn_padded": (c_int, [c_int]),
    "zi_pack_qkv": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p]),
    "zi_pack_ffn": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "zi_block_workspace_size": (c_int, [POINTER(ZiConfig), c_int, c_int, POINTER(c_size_t)]),
    "zi_model_workspace_size": (c_int, [POINTER(ZiConfig), c_int, c_int, c_int, c_int, POINTER(c_size_t)]),
    "zi_block_forward": (c_int, [POINTER(ZiConfig), POINTER(ZiBlockWeights), c_void_p, c_void_p, c_int, c_int,
                                 c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "zi_block_forward_noalloc": (c_int, [POINTER(ZiConfig), POINTER(ZiBlockWeights), c_void_p, c_void_p, c_int,
                                         c_int, c_void_p, c_void_p, c_void_p]),
    "zi_model_forward": (c_int, [POINTER(ZiConfig), POINTER(ZiModelWeights), c_int, c_int, c_int, c_int,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "zi_model_forward_varlen": (c_int, [POINTER(ZiConfig), POINTER(ZiModelWeights), c_int, c_int, c_int, c_int,
                                        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                        c_void_p]),
    "zi_model_forward_trace": (c_int, [POINTER(ZiConfig), POINTER(ZiModelWeights), c_int, c_int, c_int, c_int,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                       c_void_p]),
    "zi_euler_step": (c_int, [c_void_p, c_void_p, c_void_p, c_float, c_double, c_double, c_size_t, c_void_p]),
    "zi_sigmas": (c_int, [c_int, c_double, POINTER(c_double)]),
    "zi_timesteps": (c_int, [c_int, c_double, POINTER(c_float)]),
    "zi_positions": (c_int, [c_int, c_int, c_int, c_void_p, c_void_p]),
    "zi_rope_table": (c_int, [POINTER(ZiConfig), c_void_p, c_int, c_void_p, c_void_p]),
    "zi_gemm_bf16": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p]),
    "zi_gemm_bf16_pair": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p]),
    "zi_attention": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p]),
    "zi_quantize_rows_e4m3": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "zi_gemm_e4m3": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p]),
    "zi_attention_varlen": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_void_p]),
    "zi_profile_begin": (c_int, [c_int]),
    "zi_profile_end": (c_int, [POINTER(c_float), POINTER(c_int), c_int, POINTER(c_int)]),
    "zi_watchdog_selftest": (c_int, [c_int, c_void_p]),
    "zi_exp2_poly": (c_int, [c_void_p, c_void_p, c_size_t, c_void_p]),
    "zi_device_status": (c_int, [POINTER(c_int)]),
    "zi_clear_device_status": (c_int, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m stream_diffusion_transformer_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().zi_status_string(status).decode()


def _check(fn: str, status: int) -> None:
    if status != ZI_OK:
        raise ZiError(fn, status, status_string(status))


def call(fn: str, *args) -> None:
    """Call a status-returning entry point and raise on error."""
    _check(fn, getattr(lib(), fn)(*args))


def config_default() -> ZiConfig:
    c = ZiConfig()
    call("zi_config_default", ctypes.byref(c))
    return c


def ffn_padded(ffn: int) -> int:
    return lib().zi_ffn_padded(ffn)


def block_workspace_size(cfg: ZiConfig, batch: int, seq: int) -> int:
    n = c_size_t(0)
    call("zi_block_workspace_size", ctypes.byref(cfg), batch, seq, ctypes.byref(n))
    return n.value


def model_workspace_size(cfg: ZiConfig, batch: int, lat_h: int, lat_w: int, s_txt: int) -> int:
    n = c_size_t(0)
    call("zi_model_workspace_size", ctypes.byref(cfg), batch, lat_h, lat_w, s_txt, ctypes.byref(n))
    return n.value


def sigmas(n_steps: int, shift: float = 3.0):
    out = (c_double * (n_steps + 1))()
    call("zi_sigmas", n_steps, shift, out)
    return list(out)


def timesteps(n_steps: int, shift: float = 3.0):
    """Model timestep of each transformer call of the schedule (zi_timesteps), as Python floats
    holding the exact fp32 values."""
    out = (c_float * n_steps)()
    call("zi_timesteps", n_steps, shift, out)
    return list(out)


def device_status() -> int:
    code = c_int(0)
    st = lib().zi_device_status(ctypes.byref(code))
    if st not in (ZI_OK, ZI_ERR_TIMEOUT):
        _check("zi_device_status", st)
    return code.value


def clear_device_status() -> None:
    call("zi_clear_device_status")


KERNEL_NAMES = {
    1: "gemm_qkv_qknorm_rope", 2: "attention", 3: "gemm_out_proj", 4: "gemm_ffn_up_swiglu",
    5: "gemm_ffn_down", 6: "post_norm_residual", 7: "pre_norm", 8: "adaln_gemv", 9: "timestep_mlp",
    10: "rope_table", 11: "positions", 12: "patchify", 13: "gemm_embed", 14: "gemm_final_unpatchify",
    15: "euler", 16: "gemm", 17: "text_pad", 18: "split_clear", 19: "quantize_e4m3", 20: "watchdog_selftest",
    21: "exp2_poly_test",
}


class Profile:
    """Context manager recording the duration of every library kernel launched inside it."""

    def __init__(self, capacity: int = 4096):
        self.capacity = capacity
        self.ms = []
        self.kinds = []

    def __enter__(self):
        call("zi_profile_begin", self.capacity)
        return self

    def __exit__(self, *exc):
        ms = (c_float * self.capacity)()
        kinds = (c_int * self.capacity)()
        n = c_int(0)
        call("zi_profile_end", ms, kinds, self.capacity, ctypes.byref(n))
        if n.value < 0:
            raise RuntimeError("profile capacity exceeded")
        self.ms = list(ms[:n.value])
        self.kinds = [KERNEL_NAMES.get(k, str(k)) for k in kinds[:n.value]]
        return False

    def by_kernel(self):
        out = {}
        for k, m in zip(self.kinds, self.ms):
            e = out.setdefault(k, [0, 0.0])
            e[0] += 1
            e[1] += m
        return out


def exported_symbols():
    """Names of every entry point this binding declares."""
    return list(_SIGS)
