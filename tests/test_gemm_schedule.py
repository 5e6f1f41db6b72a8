"""Host-side check of the GEMM work schedule (no GPU): tests/schedule_check.cu is built
with nvcc and runs the kernels' own schedule functions (tile_origin, WorkWalker,
make_tail_sched, choose_raster, sched_units from zi_gemm.cuh) over the single-CTA and
CTA-pair tilings for a grid of shapes, with and without the K-split tail: every
(m, n) tile is walked once, every k-block of every tile is computed once, split
pieces are well formed and their partial slots and counters stay inside the
scratch."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _nvcc():
    for p in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if p and os.path.exists(p):
            return p
    return None


def test_gemm_schedule_covers_every_tile_and_k_block(tmp_path):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not found")
    exe = tmp_path / "schedule_check"
    cmd = [nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(ROOT, "stream_diffusion_transformer_b200", "csrc"),
           os.path.join(ROOT, "tests", "schedule_check.cu"), "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True, timeout=300)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip().startswith("schedule ok"), out.stdout
    assert int(out.stdout.split()[-1]) >= 700
