"""FlowMatch-Euler schedule, update and CFG combine (CPU oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (page title, section):
  * z-image-turbo-mnn model card, "Scheduler": shift 3.0; sigmas
    linspace(1, 1/N, N) mapped through sigma' = shift*sigma / (1 + (shift-1)*sigma);
    the transformer receives (1000 - 1000 sigma')/1000 = 1 - sigma'; its output
    is negated before the Euler step.
  * FastVideo zimage handoff, "Pinned official pipeline context" / "Scheduler":
    sigma_min = 0 and a num_steps + 1 point schedule whose final zero-sigma
    transformer call is skipped.
  * ostris ai-toolkit "Z-Image", "Specifics": t = 1 is clean; output negated to
    match the noise - latents flow target; the UI guidance 4 becomes 3 before
    the pipeline.

Readings: the Euler update is x <- x + (sigma'_{i+1} - sigma'_i) * v with
v = -model_output; CFG is y = y_u + g (y_c - y_u) (equivalently y_c + (g-1)(y_c - y_u)),
no truncation or renormalisation.
"""
from __future__ import annotations

from typing import Callable, Optional

import numpy as np


def shift_sigma(sigma, shift: float = 3.0):
    """sigma' = shift * sigma / (1 + (shift - 1) * sigma)."""
    sigma = np.asarray(sigma, dtype=np.float64)
    return shift * sigma / (1.0 + (shift - 1.0) * sigma)


def sigmas(n_steps: int, shift: float = 3.0) -> np.ndarray:
    """n_steps + 1 shifted sigmas: linspace(1, 1/N, N) through the shift, then 0."""
    base = np.linspace(1.0, 1.0 / n_steps, n_steps)
    return np.append(shift_sigma(base, shift), 0.0)


def timesteps(sig: np.ndarray) -> np.ndarray:
    """Model timestep per call, t_i = 1 - sigma'_i (1 = clean); the zero-sigma call is skipped."""
    return 1.0 - np.asarray(sig[:-1], dtype=np.float64)


def cfg_combine(y_cond: np.ndarray, y_uncond: np.ndarray, guidance: float) -> np.ndarray:
    return y_uncond + guidance * (y_cond - y_uncond)


def euler_step(x: np.ndarray, model_out: np.ndarray, sigma: float, sigma_next: float) -> np.ndarray:
    """One Euler step of the flow ODE with velocity v = -model_out."""
    return x + (sigma_next - sigma) * (-model_out)


def denoise(x0: np.ndarray, model: Callable[[np.ndarray, np.ndarray, bool], np.ndarray],
            n_steps: int, shift: float = 3.0, guidance: Optional[float] = None) -> np.ndarray:
    """Run the N-step loop.  model(x, t[B], uncond) -> raw output of x's shape.

    With guidance None only the conditional branch runs (Turbo default).
    """
    sig = sigmas(n_steps, shift)
    x = np.asarray(x0, dtype=np.float64).copy()
    B = x.shape[0]
    for i in range(n_steps):
        t = np.full(B, 1.0 - sig[i])
        y = model(x, t, False)
        if guidance is not None:
            y = cfg_combine(y, model(x, t, True), guidance)
        x = euler_step(x, y, sig[i], sig[i + 1])
    return x
