"""Z-Image S3-DiT forward on B200 (sm_100a): a C-ABI CUDA library and its Python front end.

    from stream_diffusion_transformer_b200 import abi, model
    cfg = abi.config_default()            # Z-Image sizes
    dit = model.DiT(cfg, fetch)           # weights resident on the GPU
    y = dit.forward(latent, t, txt)       # raw transformer output

The kernels live in libzimage_dit.so (built by ``python -m
stream_diffusion_transformer_b200.build``); this package only marshals
arguments.  Importing it does not load the library; the first call does, and
raises if it is missing.
"""
from . import abi  # noqa: F401

__all__ = ["abi"]
