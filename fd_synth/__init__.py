"""Seeded synthetic inputs for the FlashDecoder streaming step.

This module is shared by the CPU oracle's tests and by the CUDA path's
tests and benchmark. It holds workload shapes and random-number recipes
only: none of the decoder's arithmetic lives here.

Shapes follow the FlashDecoder paper (academ.us/article/2607.14898):
latent frames z_t of shape [C'][H'][W'] (Sec. 3.1), an optional
PixelUnshuffle x2 of the Wan2.1 latent (Sec. 4.3, "Generalization Across
Latent Spaces"), L_frm tokens per frame (Sec. 3.2, Eq. 1), a Transformer of
width D with N heads of size D_h and G key/value groups (Sec. 3.2, 4.5).

Recipe (stands in for UltraVideo clips encoded by the Wan encoders and for
trained weights, neither of which is available):
  * weights of every Linear ~ N(0,1)/sqrt(fan_in), biases likewise;
  * RMSNorm / KV-norm gains = 1 + 0.1 N(0,1);
  * latents ~ N(0,1);
  * torch CPU generator, seed 0 for weights, seed 1 for latents;
  * bf16 configurations round weights and latents to bf16 (nearest even)
    before anyone sees them, so the oracle and the CUDA path read identical
    values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class FDConfig:
    """One decoder configuration (paper notation in comments)."""
    name: str
    latent_ch: int        # C'
    grid_h: int           # H' (latent grid)
    grid_w: int           # W'
    patch: int            # PixelUnshuffle factor p (1 or 2)
    d_model: int          # D
    n_heads: int          # N (query heads)
    n_kv_heads: int       # G (key/value groups)
    head_dim: int         # D_h
    n_blocks: int
    mlp_ratio: int
    window: int           # W = number of PAST latent frames kept; ring has W+1 slots
    out_ch: int           # C (pixel channels)
    r_t: int              # temporal upsampling factor
    px_per_token: int     # P: pixels per token side
    kv_norm: int          # 1 = KV-norm on
    dtype: str            # "f32" or "bf16" (compute/storage of the CUDA path)
    frames: int           # T' of the workload
    norm_eps: float = 1e-6
    rope_theta: float = 10000.0
    # output head: "linear" = final RMSNorm + one Linear D -> C r_t P^2 +
    # unpatchify; "paper" = temporal upsample Linear D -> r_t D (Eq. 3),
    # n_refine streaming refinement blocks over the r_t sub-frames (window of
    # r_t (W+1) sub-frames), RMSNorm + 2-layer MLP D -> D -> C P^2 and
    # PixelShuffle per sub-frame (paper Sec. 3.4)
    head: str = "linear"
    n_refine: int = 2
    # 1: the MLP sublayer of every Transformer block runs on FP8 E4M3 operands
    # with static per-tensor scales (paper Sec. 4.6); bf16 configurations only
    mlp_fp8: int = 0
    # video streams decoded together per step (each its own video and cache)
    batch: int = 1
    # bf16 attention key splitting: 0 = automatic, 1..4 forced
    attn_splits: int = 0
    # bf16 attention MMA issue: 0 = automatic, 1 = two threads, 2 = one thread
    attn_issuer: int = 0

    # ---- derived shapes (no arithmetic of the method) ----
    @property
    def tok_h(self) -> int:
        return self.grid_h // self.patch

    @property
    def tok_w(self) -> int:
        return self.grid_w // self.patch

    @property
    def L_frm(self) -> int:
        return self.tok_h * self.tok_w

    @property
    def c_in(self) -> int:
        return self.latent_ch * self.patch * self.patch

    @property
    def qkv_dim(self) -> int:
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim

    @property
    def d_ff(self) -> int:
        return self.mlp_ratio * self.d_model

    @property
    def c_out(self) -> int:
        return self.out_ch * self.r_t * self.px_per_token * self.px_per_token

    @property
    def c_px(self) -> int:
        """Columns of one sub-frame's spatial MLP output: C P^2."""
        return self.out_ch * self.px_per_token * self.px_per_token

    @property
    def out_shape(self):
        return (self.out_ch, self.r_t, self.tok_h * self.px_per_token,
                self.tok_w * self.px_per_token)

    def replace(self, **kw) -> "FDConfig":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, FDConfig] = {
    # tiny fp32: 16ch latent, 8x8 grid, patch 1 (64 tokens), 3 frames, d=64,
    # 2 heads x 32, 2 blocks, W=2, 3ch x 4 frames x 8x8 px per token.
    "tiny_fp32": FDConfig("tiny_fp32", 16, 8, 8, 1, 64, 2, 2, 32, 2, 4, 2,
                          3, 4, 8, 1, "f32", 3),
    # Wan2.1-shaped 480p: 16ch, 60x104 grid, patch 2 (1560 tokens), 21 frames.
    "480p_wan21": FDConfig("480p_wan21", 16, 60, 104, 2, 1024, 16, 16, 64, 12,
                           4, 2, 3, 4, 16, 1, "bf16", 21),
    # Wan2.1-shaped 720p: 16ch, 90x160 grid, patch 2 (3600 tokens), 21 frames.
    "720p_wan21": FDConfig("720p_wan21", 16, 90, 160, 2, 1024, 16, 16, 64, 12,
                           4, 2, 3, 4, 16, 1, "bf16", 21),
    # Wan2.2-shaped 1080p: 48ch, 68x120 grid (1088x1920 px), patch 1
    # (8160 tokens), 7 frames, 16 blocks.
    "1080p_wan22": FDConfig("1080p_wan22", 48, 68, 120, 1, 1024, 16, 16, 64,
                            16, 4, 2, 3, 4, 16, 1, "bf16", 7),
    # the same 1080p decoder with W = 1 (the paper's deployed W_frm = 2: the
    # current latent frame plus one previous frame, Sec. 4.4 "Window Size
    # Ablation"), a context row beside the W = 2 workload
    "1080p_wan22_w1": FDConfig("1080p_wan22_w1", 48, 68, 120, 1, 1024, 16, 16, 64,
                               16, 4, 1, 3, 4, 16, 1, "bf16", 7),
    # long-stream Wan2.2-shaped 720p: 48ch, 45x80 grid, patch 1 (3600 tokens),
    # 200 frames, 16 blocks.
    "long720p_wan22": FDConfig("long720p_wan22", 48, 45, 80, 1, 1024, 16, 16,
                               64, 16, 4, 2, 3, 4, 16, 1, "bf16", 200),
    # FlashDecoder-XL backbone shape (D=1536, 24 heads, 3 KV groups, 20 blocks;
    # the paper's W_frm=2 window = 1 past frame) on the Wan2.2 480p latent
    # (48ch, 30x52 grid, 1560 tokens), 7 latent frames.
    "xl_480p_wan22": FDConfig("xl_480p_wan22", 48, 30, 52, 1, 1536, 24, 3, 64,
                              20, 4, 1, 3, 4, 16, 1, "bf16", 7),
    # FlashDecoder-XL with the paper's own head (Sec. 3.4): the XL backbone
    # above, temporal upsampling by r_t = 4, 2 refinement blocks over a window
    # of r_t (W+1) = 8 sub-frames, RMSNorm + MLP 1536 -> 1536 -> 3*16*16 and
    # PixelShuffle; 480p and 720p Wan2.2 latents.
    "xl_480p_wan22_paper": FDConfig("xl_480p_wan22_paper", 48, 30, 52, 1, 1536, 24, 3,
                                    64, 20, 4, 1, 3, 4, 16, 1, "bf16", 7,
                                    head="paper", n_refine=2),
    "xl_720p_wan22_paper": FDConfig("xl_720p_wan22_paper", 48, 45, 80, 1, 1536, 24, 3,
                                    64, 20, 4, 1, 3, 4, 16, 1, "bf16", 7,
                                    head="paper", n_refine=2),
}


BLOCK_KEYS = ("norm1_g", "wqkv", "bqkv", "knorm_g", "vnorm_g", "wo", "bo", "norm2_g",
              "w1", "b1", "w2", "b2")


def weight_names(cfg: FDConfig) -> List[str]:
    """Flat list of weight tensor names in generation order. Backbone blocks
    are "b{l}.*"; with the paper head, refinement blocks are "r{l}.*"."""
    names = ["embed_w", "embed_b"]
    for l in range(cfg.n_blocks):
        names += [f"b{l}.{k}" for k in BLOCK_KEYS]
    if cfg.head == "paper":
        names += ["up_w", "up_b"]
        for l in range(cfg.n_refine):
            names += [f"r{l}.{k}" for k in BLOCK_KEYS]
        names += ["final_g", "sp1_w", "sp1_b", "out_w", "out_b"]
    else:
        names += ["final_g", "out_w", "out_b"]
    return names


def weight_shapes(cfg: FDConfig) -> Dict[str, tuple]:
    """Shapes in PyTorch Linear layout ([out][in]) and the fan_in of each."""
    D, Dh, H = cfg.d_model, cfg.head_dim, cfg.n_heads
    s = {"embed_w": ((D, cfg.c_in), cfg.c_in), "embed_b": ((D,), cfg.c_in)}
    prefixes = [f"b{l}." for l in range(cfg.n_blocks)]
    if cfg.head == "paper":
        prefixes += [f"r{l}." for l in range(cfg.n_refine)]
    for p in prefixes:
        s[p + "norm1_g"] = ((D,), None)
        s[p + "wqkv"] = ((cfg.qkv_dim, D), D)
        s[p + "bqkv"] = ((cfg.qkv_dim,), D)
        s[p + "knorm_g"] = ((Dh,), None)
        s[p + "vnorm_g"] = ((Dh,), None)
        s[p + "wo"] = ((D, H * Dh), H * Dh)
        s[p + "bo"] = ((D,), H * Dh)
        s[p + "norm2_g"] = ((D,), None)
        s[p + "w1"] = ((cfg.d_ff, D), D)
        s[p + "b1"] = ((cfg.d_ff,), D)
        s[p + "w2"] = ((D, cfg.d_ff), cfg.d_ff)
        s[p + "b2"] = ((D,), cfg.d_ff)
    s["final_g"] = ((D,), None)
    if cfg.head == "paper":
        s["up_w"] = ((cfg.r_t * D, D), D)
        s["up_b"] = ((cfg.r_t * D,), D)
        s["sp1_w"] = ((D, D), D)
        s["sp1_b"] = ((D,), D)
        s["out_w"] = ((cfg.c_px, D), D)
        s["out_b"] = ((cfg.c_px,), D)
    else:
        s["out_w"] = ((cfg.c_out, D), D)
        s["out_b"] = ((cfg.c_out,), D)
    return s


def _round(t: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return t.to(torch.bfloat16).to(torch.float32)
    return t


def make_weights(cfg: FDConfig, seed: int = 0) -> Dict[str, np.ndarray]:
    """Random-init weights (float32 numpy, bf16-representable for bf16 configs)."""
    g = torch.Generator().manual_seed(seed)
    shapes = weight_shapes(cfg)
    out = {}
    for name in weight_names(cfg):
        shape, fan_in = shapes[name]
        r = torch.randn(shape, generator=g, dtype=torch.float32)
        if fan_in is None:          # a norm gain
            t = 1.0 + 0.1 * r
        else:
            t = r / math.sqrt(fan_in)
        out[name] = _round(t, cfg.dtype).numpy()
    return out


def make_latents(cfg: FDConfig, frames: int | None = None,
                 seed: int = 1) -> np.ndarray:
    """Latent video z[t][C'][H'][W'] (float32 numpy), N(0,1)."""
    T = cfg.frames if frames is None else frames
    g = torch.Generator().manual_seed(seed)
    z = torch.randn((T, cfg.latent_ch, cfg.grid_h, cfg.grid_w), generator=g,
                    dtype=torch.float32)
    return _round(z, cfg.dtype).numpy()


def perturb_frame(z: np.ndarray, t: int, seed: int = 7,
                  dtype: str = "f32") -> np.ndarray:
    """Copy of z with frame t replaced by fresh N(0,1) values."""
    g = torch.Generator().manual_seed(seed)
    out = z.copy()
    r = torch.randn(z.shape[1:], generator=g, dtype=torch.float32)
    out[t] = _round(r, dtype).numpy()
    return out
