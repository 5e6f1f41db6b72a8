"""Helpers shared by the GPU parity tests: tensor transfer and the parity metrics."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import zimage_inputs as zi


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip("needs an sm_100 GPU")


def dev_bits(bits: np.ndarray) -> "torch.Tensor":
    """bf16 bit patterns -> device bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_f64(t: "torch.Tensor") -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits_f64(bits: np.ndarray) -> np.ndarray:
    return zi.bf16_bits_to_f32(bits).astype(np.float64)


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64).ravel()
    want = np.asarray(want, dtype=np.float64).ravel()
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


def cosine(got, want) -> float:
    got = np.asarray(got, dtype=np.float64).ravel()
    want = np.asarray(want, dtype=np.float64).ravel()
    return float(got @ want / (np.linalg.norm(got) * np.linalg.norm(want)))


def assert_parity(got, want, rel=2e-2, cos=0.999, what=""):
    r, c = rel_l2(got, want), cosine(got, want)
    print(f"[parity] {what}: rel-L2 {r:.3e} cos {c:.7f}")
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert r <= rel and c >= cos, f"{what}: rel-L2 {r:.3e} (<= {rel}), cos {c:.6f} (>= {cos})"
    return r, c
