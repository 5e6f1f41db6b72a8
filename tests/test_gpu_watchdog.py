"""Failure detection on the GPU without a fault: a wait that nothing completes runs
out, the kernel records a timeout in the device error word and returns, the host
reads it, pipeline kernels refuse to run while it is set, and after clearing it
the context works normally."""
import ctypes

import numpy as np
import pytest

from gpu_util import host_f64, require_gpu, torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_stays_usable():
    require_gpu()
    from stream_diffusion_transformer_b200 import abi, model
    abi.clear_device_status()
    abi.call("zi_watchdog_selftest", 50000, model._stream())  # 50 ms limit
    torch.cuda.synchronize()
    assert abi.device_status() == 6
    code = ctypes.c_int(0)
    assert abi.lib().zi_device_status(ctypes.byref(code)) == abi.ZI_ERR_TIMEOUT and code.value == 6

    g = torch.Generator(device="cuda").manual_seed(0)
    a = torch.randn((256, 128), device="cuda", generator=g).to(torch.bfloat16)
    b = torch.randn((256, 128), device="cuda", generator=g).to(torch.bfloat16)
    c = torch.full((256, 256), 7.0, device="cuda", dtype=torch.bfloat16)
    model.gemm(a, b, out=c)  # the error word is set: the kernel exits without writing
    torch.cuda.synchronize()
    assert torch.all(c == 7.0)

    abi.clear_device_status()
    assert abi.device_status() == 0
    model.gemm(a, b, out=c)
    torch.cuda.synchronize()
    want = a.float() @ b.float().T
    err = np.linalg.norm(host_f64(c) - host_f64(want)) / np.linalg.norm(host_f64(want))
    assert err < 4e-3 and abi.device_status() == 0
