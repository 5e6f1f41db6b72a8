"""Python front end of the C ABI: device-resident weights, workspaces and calls.

PyTorch is used only to own device memory and streams; every step of the
forward runs in libzimage_dit.so.  bf16 tensors are handed over as raw bits.
"""
from __future__ import annotations

import ctypes
from typing import Callable, Dict, Iterable, List, Optional, Sequence

import numpy as np
import torch

from . import abi

Bits = np.ndarray  # uint16 bf16 bit patterns


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def upload_bits(bits: Bits, device) -> torch.Tensor:
    """bf16 bit patterns (uint16 numpy) -> a bf16 tensor on `device`."""
    host = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return host.to(device).view(torch.bfloat16)


def make_config(dims) -> abi.ZiConfig:
    """ZiConfig from any object with the model's size attributes (dim, heads, ...)."""
    c = abi.config_default()
    for name in ("dim", "heads", "head_dim", "ffn", "cap_dim", "t_freq", "t_mid", "in_ch", "patch",
                 "n_noise", "n_ctx", "n_main"):
        setattr(c, name, int(getattr(dims, name)))
    axes = getattr(dims, "rope_axes", (32, 48, 48))
    for i in range(3):
        c.rope_axes[i] = int(axes[i])
    return c


def block_keys(prefix: str, modulated: bool) -> List[str]:
    a = f"{prefix}.attention"
    k = [f"{a}.to_q.weight", f"{a}.to_k.weight", f"{a}.to_v.weight", f"{a}.to_out.weight",
         f"{a}.norm_q.weight", f"{a}.norm_k.weight", f"{prefix}.attention_norm1.weight",
         f"{prefix}.attention_norm2.weight", f"{prefix}.ffn_norm1.weight", f"{prefix}.ffn_norm2.weight",
         f"{prefix}.feed_forward.w1.weight", f"{prefix}.feed_forward.w2.weight", f"{prefix}.feed_forward.w3.weight"]
    if modulated:
        k += [f"{prefix}.adaLN_modulation.weight", f"{prefix}.adaLN_modulation.bias"]
    return k


TOP_KEYS = {
    "x_emb_w": "x_embedder.weight", "x_emb_b": "x_embedder.bias",
    "cap_norm": "cap_embedder.norm.weight", "cap_w": "cap_embedder.linear.weight",
    "cap_b": "cap_embedder.linear.bias",
    "t_w1": "t_embedder.linear1.weight", "t_b1": "t_embedder.linear1.bias",
    "t_w2": "t_embedder.linear2.weight", "t_b2": "t_embedder.linear2.bias",
    "final_ada_w": "final_layer.adaLN_modulation.weight", "final_ada_b": "final_layer.adaLN_modulation.bias",
    "final_w": "final_layer.linear.weight", "final_b": "final_layer.linear.bias",
    "cap_pad": "cap_pad_token",
}


class DeviceBlock:
    """One block's weights in the library's layout (fused qkv, interleaved w13, padded w2).

    fp8=True also stores e4m3 codes of the fused qkv and w13 with one scale per
    output channel (zi_quantize_rows_e4m3); the block then runs those two
    projections in e4m3.  fp8="all" does the same for w_out and w2, so every
    projection of the block runs in e4m3."""

    def __init__(self, cfg: abi.ZiConfig, prefix: str, bits: Dict[str, Bits], modulated: bool, device,
                 fp8=False):
        D, F = cfg.dim, cfg.ffn
        Fp = abi.ffn_padded(F)
        a = f"{prefix}.attention"
        self.t: Dict[str, torch.Tensor] = {}
        w_qkv = torch.empty((3 * D, D), dtype=torch.bfloat16, device=device)
        for i, nm in enumerate(("to_q", "to_k", "to_v")):
            w_qkv[i * D:(i + 1) * D].copy_(upload_bits(bits[f"{a}.{nm}.weight"], "cpu"))
        self.t["w_qkv"] = w_qkv
        self.t["w_out"] = upload_bits(bits[f"{a}.to_out.weight"], device)
        ff = f"{prefix}.feed_forward"
        w1 = upload_bits(bits[f"{ff}.w1.weight"], device)
        w3 = upload_bits(bits[f"{ff}.w3.weight"], device)
        w2 = upload_bits(bits[f"{ff}.w2.weight"], device)
        self.t["w13"] = torch.empty((2 * Fp, D), dtype=torch.bfloat16, device=device)
        self.t["w2"] = torch.empty((D, Fp), dtype=torch.bfloat16, device=device)
        abi.call("zi_pack_ffn", _p(w1), _p(w3), _p(w2), F, D, _p(self.t["w13"]), _p(self.t["w2"]), _stream())
        torch.cuda.current_stream().synchronize()  # the temporaries w1, w3, w2 are freed on return
        for fld, key in (("g_attn1", f"{prefix}.attention_norm1.weight"),
                         ("g_attn2", f"{prefix}.attention_norm2.weight"),
                         ("g_ffn1", f"{prefix}.ffn_norm1.weight"), ("g_ffn2", f"{prefix}.ffn_norm2.weight"),
                         ("g_q", f"{a}.norm_q.weight"), ("g_k", f"{a}.norm_k.weight")):
            self.t[fld] = upload_bits(bits[key], device)
        if modulated:
            self.t["w_ada"] = upload_bits(bits[f"{prefix}.adaLN_modulation.weight"], device)
            self.t["b_ada"] = upload_bits(bits[f"{prefix}.adaLN_modulation.bias"], device)
        self.modulated = modulated
        self._finish(fp8)

    BF16_FIELDS = ("w_qkv", "w_out", "w13", "w2", "g_attn1", "g_attn2", "g_ffn1", "g_ffn2", "g_q", "g_k",
                   "w_ada", "b_ada")

    def _finish(self, fp8):
        if fp8:
            groups = [("w_qkv", "w_qkv8", "s_qkv"), ("w13", "w13_8", "s_13")]
            if fp8 == "all":
                groups += [("w_out", "w_out8", "s_out"), ("w2", "w2_8", "s_2")]
            for src, q, sc in groups:
                self.t[q], self.t[sc] = quantize_rows_e4m3(self.t[src])
        self.fp8 = fp8
        self.struct = abi.ZiBlockWeights(**{f: (self.t[f].data_ptr() if f in self.t else None)
                                            for f in abi.BLOCK_FIELDS})

    def with_e4m3(self, fp8=True) -> "DeviceBlock":
        """The same block sharing these bf16 tensors, with e4m3 codes made from them (see the
        class docstring for fp8)."""
        b = DeviceBlock.__new__(DeviceBlock)
        b.t = {k: v for k, v in self.t.items() if k in self.BF16_FIELDS}
        b.modulated = self.modulated
        b._finish(fp8)
        return b

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.t.values())


class DiT:
    """The S3-DiT transformer on one GPU, weights resident in HBM."""

    def __init__(self, cfg: abi.ZiConfig, fetch: Callable[[Sequence[str]], Dict[str, Bits]], device="cuda",
                 fp8=False):
        """fetch(keys) -> {key: bf16 bits} is called once per block and once for the rest,
        so a 12 GB model never has to sit in host memory at once.  fp8=True runs every
        block's QKV and FFN w1|w3 projections in e4m3, fp8="all" every block
        projection (see DeviceBlock)."""
        self.cfg = cfg
        self.device = torch.device(device)
        abi.lib()
        top = fetch(list(TOP_KEYS.values()))
        self.top = {f: upload_bits(top[k], self.device) for f, k in TOP_KEYS.items()}
        self.fp8 = fp8
        self.noise = [DeviceBlock(cfg, f"noise_refiner.{i}", fetch(block_keys(f"noise_refiner.{i}", True)), True,
                                  self.device, fp8) for i in range(cfg.n_noise)]
        self.ctx = [DeviceBlock(cfg, f"context_refiner.{i}", fetch(block_keys(f"context_refiner.{i}", False)),
                                False, self.device, fp8) for i in range(cfg.n_ctx)]
        self.main = [DeviceBlock(cfg, f"layers.{i}", fetch(block_keys(f"layers.{i}", True)), True, self.device, fp8)
                     for i in range(cfg.n_main)]
        self._bind()

    def _bind(self):
        self._noise_arr = (abi.ZiBlockWeights * max(1, len(self.noise)))(*[b.struct for b in self.noise])
        self._ctx_arr = (abi.ZiBlockWeights * max(1, len(self.ctx)))(*[b.struct for b in self.ctx])
        self._main_arr = (abi.ZiBlockWeights * len(self.main))(*[b.struct for b in self.main])
        kw = {f: self.top[f].data_ptr() for f in abi.MODEL_FIELDS}
        self.weights = abi.ZiModelWeights(**kw)
        self.weights.cap_pad = self.top["cap_pad"].data_ptr()
        self.weights.noise = ctypes.cast(self._noise_arr, ctypes.POINTER(abi.ZiBlockWeights))
        self.weights.ctx = ctypes.cast(self._ctx_arr, ctypes.POINTER(abi.ZiBlockWeights))
        self.weights.main = ctypes.cast(self._main_arr, ctypes.POINTER(abi.ZiBlockWeights))
        self._ws: Dict[tuple, torch.Tensor] = {}

    def with_e4m3(self, fp8=True) -> "DiT":
        """This transformer with its block projections in e4m3 (fp8=True: QKV and FFN w1|w3;
        "all": every block projection), sharing the resident bf16 weights: only the e4m3
        codes and their per-row scales are new (zi_quantize_rows_e4m3 on the device)."""
        other = DiT.__new__(DiT)
        other.cfg, other.device, other.top, other.fp8 = self.cfg, self.device, self.top, fp8
        other.noise = [b.with_e4m3(fp8) for b in self.noise]
        other.ctx = [b.with_e4m3(fp8) for b in self.ctx]
        other.main = [b.with_e4m3(fp8) for b in self.main]
        other._bind()
        return other

    def nbytes(self) -> int:
        n = sum(t.numel() * t.element_size() for t in self.top.values())
        return n + sum(b.nbytes() for b in self.noise + self.ctx + self.main)

    def workspace(self, batch: int, lat_h: int, lat_w: int, s_txt: int) -> torch.Tensor:
        key = (batch, lat_h, lat_w, s_txt)
        if key not in self._ws:
            n = abi.model_workspace_size(self.cfg, batch, lat_h, lat_w, s_txt)
            self._ws[key] = torch.empty(n, dtype=torch.uint8, device=self.device)
        return self._ws[key]

    def denoise(self, latent: torch.Tensor, txt: torch.Tensor, n_steps: int = 8, shift: float = 3.0,
                guidance: Optional[float] = None, txt_uncond: Optional[torch.Tensor] = None,
                txt_len: Optional[Sequence[int]] = None,
                txt_uncond_len: Optional[Sequence[int]] = None) -> torch.Tensor:
        """FlowMatch-Euler loop (z-image-turbo-mnn "Scheduler"): n_steps forwards at the
        library's timesteps (zi_timesteps: t_i = 1 - sigma'_i), each followed by
        zi_euler_step with sigma'_i -> sigma'_{i+1}; with guidance and txt_uncond, the conditional and unconditional branches run
        as one batch-2 forward and are combined y_u + g (y_c - y_u).  txt_len /
        txt_uncond_len give the real lengths of padded prompts (see forward); the
        two branches' texts are padded to one length.  Returns the final latent (a
        new tensor; `latent` is left unchanged)."""
        sig = abi.sigmas(n_steps, shift)
        ts = abi.timesteps(n_steps, shift)
        x = latent.clone()
        B = x.shape[0]
        cfg_mode = guidance is not None and txt_uncond is not None
        out = torch.empty((2 * B,) + tuple(x.shape[1:]) if cfg_mode else x.shape, dtype=torch.float32,
                          device=x.device)
        tt = torch.empty(2 * B if cfg_mode else B, dtype=torch.float32, device=x.device)
        lens = None if txt_len is None else list(txt_len)
        if cfg_mode:
            L = max(txt.shape[1], txt_uncond.shape[1])
            if txt.shape[1] != txt_uncond.shape[1] or txt_len is not None or txt_uncond_len is not None:
                lc = list(txt_len) if txt_len is not None else [txt.shape[1]] * B
                lu = list(txt_uncond_len) if txt_uncond_len is not None else [txt_uncond.shape[1]] * B
                lens = lc + lu
            txt_all = torch.zeros((2 * B, L, txt.shape[2]), dtype=txt.dtype, device=txt.device)
            txt_all[:B, :txt.shape[1]].copy_(txt)
            txt_all[B:, :txt_uncond.shape[1]].copy_(txt_uncond)
        else:
            txt_all = txt
        x_in = torch.empty((2 * B,) + tuple(x.shape[1:]), dtype=torch.float32, device=x.device) if cfg_mode else x
        for i in range(n_steps):
            tt.fill_(ts[i])
            if cfg_mode:
                x_in[:B].copy_(x)
                x_in[B:].copy_(x)
            self.forward(x_in, tt, txt_all, out, txt_len=lens)
            if cfg_mode:
                abi.call("zi_euler_step", _p(x), _p(out[:B]), _p(out[B:]), float(guidance), sig[i], sig[i + 1],
                         x.numel(), _stream())
            else:
                abi.call("zi_euler_step", _p(x), _p(out), None, 0.0, sig[i], sig[i + 1], x.numel(), _stream())
        return x

    def forward(self, latent: torch.Tensor, t: torch.Tensor, txt: torch.Tensor,
                out: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                txt_len: Optional[Sequence[int]] = None) -> torch.Tensor:
        """latent fp32 [B, C, H/8, W/8], t fp32 [B] (1 = clean), txt bf16 [B, L, cap_dim] -> raw output.

        txt_len (host ints, one per element, each in [1, L]): element b's prompt is
        its first txt_len[b] text rows, the rest padding (zi_model_forward_varlen)."""
        B, C, Hl, Wl = latent.shape
        L = txt.shape[1]
        assert latent.dtype == torch.float32 and t.dtype == torch.float32 and txt.dtype == torch.bfloat16
        assert latent.is_contiguous() and txt.is_contiguous() and t.is_contiguous()
        if out is None:
            out = torch.empty_like(latent)
        ws = self.workspace(B, Hl, Wl, L)
        if txt_len is None:
            abi.call("zi_model_forward", ctypes.byref(self.cfg), ctypes.byref(self.weights), B, Hl, Wl, L,
                     _p(latent), _p(t), _p(txt), _p(out), _p(ws), ws.numel(), _stream(stream))
        else:
            lens = (ctypes.c_int32 * B)(*[int(v) for v in txt_len])
            abi.call("zi_model_forward_varlen", ctypes.byref(self.cfg), ctypes.byref(self.weights), B, Hl, Wl, L,
                     lens, _p(latent), _p(t), _p(txt), _p(out), _p(ws), ws.numel(), _stream(stream))
        return out


def denoise_cfg_split(latent: torch.Tensor, n_steps: int, shift: float, guidance: float,
                      forward: Callable[[torch.Tensor, torch.Tensor], torch.Tensor],
                      euler: Optional[Callable] = None, group=None) -> torch.Tensor:
    """Classifier-free guidance with the two branches on two ranks (one GPU each):
    rank 0 runs the conditional forward, rank 1 the unconditional one, each on its
    own full replica of the weights; after every forward the two raw outputs are
    exchanged with one all-gather (torch.distributed over NCCL on GPUs; 4 MB per
    step at 2048x2048) and both ranks apply the same guided Euler step, so their
    latents stay identical.

    forward(x, t) -> raw output of x's shape, for this rank's branch (for example
    lambda x, t: dit.forward(x, t, txt_of_this_branch)).  euler(x, y_cond, y_uncond,
    guidance, sigma, sigma_next) updates x in place; by default zi_euler_step.
    Returns the final latent (a new tensor)."""
    import torch.distributed as dist
    if dist.get_world_size(group) != 2:
        raise ValueError("the CFG split runs on exactly two ranks")
    if euler is None:
        euler = lambda x, yc, yu, g, s0, s1: euler_step(x, yc, yu, g, s0, s1)
    sig = abi.sigmas(n_steps, shift)
    ts = abi.timesteps(n_steps, shift)
    x = latent.clone()
    t = torch.empty(x.shape[0], dtype=torch.float32, device=x.device)
    both = [torch.empty_like(x), torch.empty_like(x)]
    for i in range(n_steps):
        t.fill_(ts[i])
        y = forward(x, t)
        dist.all_gather(both, y.contiguous(), group=group)  # [conditional, unconditional]
        euler(x, both[0], both[1], float(guidance), sig[i], sig[i + 1])
    return x


class DenoiseGraph:
    """DiT.denoise captured once as a CUDA graph and replayed: all n_steps forwards,
    their Euler steps (sigmas baked in) and, with guidance, the CFG combines, for
    one fixed latent shape and fixed text features (read in place by every replay:
    change them with copy_() to condition on other text).  run(latent) copies the latent
    into the graph's input buffer, replays, and returns the graph's output tensor
    (overwritten by the next run)."""

    def __init__(self, dit: "DiT", latent_shape, txt: torch.Tensor, n_steps: int = 8, shift: float = 3.0,
                 guidance: Optional[float] = None, txt_uncond: Optional[torch.Tensor] = None,
                 txt_len: Optional[Sequence[int]] = None, txt_uncond_len: Optional[Sequence[int]] = None):
        self.x0 = torch.zeros(tuple(latent_shape), dtype=torch.float32, device=dit.device)
        # the graph reads the text features by address: hold them for its lifetime
        self.txt, self.txt_uncond = txt, txt_uncond
        kw = dict(n_steps=n_steps, shift=shift, guidance=guidance, txt_uncond=txt_uncond, txt_len=txt_len,
                  txt_uncond_len=txt_uncond_len)
        # one eager run first: kernel attributes are set and the workspace exists
        # before capture (neither may happen while the stream is being captured)
        dit.denoise(self.x0, txt, **kw)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.out = dit.denoise(self.x0, txt, **kw)
        torch.cuda.synchronize()

    def run(self, latent: torch.Tensor) -> torch.Tensor:
        self.x0.copy_(latent)
        self.graph.replay()
        return self.out


def forward_trace(dit: "DiT", latent: torch.Tensor, t: torch.Tensor, txt: torch.Tensor):
    """DiT.forward that also returns the residual stream after every block:
    (out, trace fp32 [n_blocks, rows, dim]) with rows = image rows then text rows."""
    B, C, Hl, Wl = latent.shape
    L = txt.shape[1]
    cfg = dit.cfg
    rows = B * ((Hl // 2) * (Wl // 2) + L)
    n_blocks = cfg.n_noise + cfg.n_ctx + cfg.n_main
    trace = torch.empty((n_blocks, rows, cfg.dim), dtype=torch.float32, device=latent.device)
    out = torch.empty_like(latent)
    ws = dit.workspace(B, Hl, Wl, L)
    abi.call("zi_model_forward_trace", ctypes.byref(cfg), ctypes.byref(dit.weights), B, Hl, Wl, L, _p(latent), _p(t),
             _p(txt), _p(out), _p(trace), _p(ws), ws.numel(), _stream())
    return out, trace


def block_forward(cfg: abi.ZiConfig, blk: DeviceBlock, c: Optional[torch.Tensor], pos: torch.Tensor,
                  x_in: torch.Tensor, x_out: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One block on x_in fp32 [B, S, D]; pos int32 [S, 3]; c fp32 [B, 256] (or None if unmodulated)."""
    B, S, D = x_in.shape
    if x_out is None:
        x_out = torch.empty_like(x_in)
    need = abi.block_workspace_size(cfg, B, S)
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=x_in.device)
    abi.call("zi_block_forward", ctypes.byref(cfg), ctypes.byref(blk.struct), _p(c), _p(pos), B, S,
             _p(x_in), _p(x_out), _p(ws), ws.numel(), _stream())
    return x_out


# ------------------------------------------------------------------ single steps

def positions(s_txt: int, grid_h: int, grid_w: int, device="cuda") -> torch.Tensor:
    pos = torch.empty((grid_h * grid_w + s_txt, 3), dtype=torch.int32, device=device)
    abi.call("zi_positions", s_txt, grid_h, grid_w, _p(pos), _stream())
    return pos


def rope_table(cfg: abi.ZiConfig, pos: torch.Tensor) -> torch.Tensor:
    out = torch.empty((pos.shape[0], cfg.head_dim // 2, 2), dtype=torch.float32, device=pos.device)
    abi.call("zi_rope_table", ctypes.byref(cfg), _p(pos), pos.shape[0], _p(out), _stream())
    return out


def gemm(a: torch.Tensor, b: torch.Tensor, out: Optional[torch.Tensor] = None, pair: bool = False) -> torch.Tensor:
    """a bf16 [M, K] @ b bf16 [N, K]^T -> bf16 [M, N]; pair=True runs it on CTA pairs (zi_gemm_bf16_pair)."""
    M, K = a.shape
    N = b.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    abi.call("zi_gemm_bf16_pair" if pair else "zi_gemm_bf16", _p(a), _p(b), _p(out), M, N, K, _stream())
    return out


def attention(qkv: torch.Tensor, batch: int, seq: int, heads: int,
              out: Optional[torch.Tensor] = None, kv_len: Optional[torch.Tensor] = None) -> torch.Tensor:
    """kv_len: device int32 [batch] of valid keys per element (the rest masked), or None."""
    if out is None:
        out = torch.empty((batch * seq, heads * 128), dtype=torch.bfloat16, device=qkv.device)
    if kv_len is None:
        abi.call("zi_attention", _p(qkv), _p(out), batch, seq, heads, _stream())
    else:
        abi.call("zi_attention_varlen", _p(qkv), _p(out), batch, seq, heads, _p(kv_len), _stream())
    return out


def quantize_rows_e4m3(x: torch.Tensor):
    """Per-row e4m3 codes (uint8, x's shape) and fp32 scales [rows] of a 2-D fp32 or bf16 tensor."""
    assert x.dim() == 2 and x.is_contiguous() and x.dtype in (torch.float32, torch.bfloat16)
    q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    sc = torch.empty(x.shape[0], dtype=torch.float32, device=x.device)
    abi.call("zi_quantize_rows_e4m3", _p(x), 1 if x.dtype == torch.bfloat16 else 0, x.shape[0], x.shape[1], _p(q),
             _p(sc), _stream())
    return q, sc


def gemm_e4m3(a: torch.Tensor, sa: torch.Tensor, b: torch.Tensor, sb: torch.Tensor,
              out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """bf16 [M, N] = sa[m] sb[n] (a e4m3 [M, K]) (b e4m3 [N, K])^T."""
    M, K = a.shape
    N = b.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    abi.call("zi_gemm_e4m3", _p(a), _p(sa), _p(b), _p(sb), _p(out), M, N, K, _stream())
    return out


def euler_step(x: torch.Tensor, out_cond: torch.Tensor, out_uncond: Optional[torch.Tensor], guidance: float,
               sigma: float, sigma_next: float) -> torch.Tensor:
    abi.call("zi_euler_step", _p(x), _p(out_cond), _p(out_uncond), float(guidance), float(sigma),
             float(sigma_next), x.numel(), _stream())
    return x


def pack_qkv(wq: torch.Tensor, wk: torch.Tensor, wv: torch.Tensor) -> torch.Tensor:
    D = wq.shape[0]
    out = torch.empty((3 * D, D), dtype=torch.bfloat16, device=wq.device)
    abi.call("zi_pack_qkv", _p(wq), _p(wk), _p(wv), D, _p(out), _stream())
    return out
