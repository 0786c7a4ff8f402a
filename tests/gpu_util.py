"""Shared helpers of the GPU tests: run the CUDA path through the C ABI and
compare it with the CPU oracle."""
import numpy as np

import fd_synth
import oracle

# Tolerances (fixed by the decoder's specification):
#   fp32 configuration: max abs error <= 1e-4
#   bf16 configurations: output relative L2 error <= 2e-2 and max abs <= 5e-2
FP32_MAX_ABS = 1e-4
BF16_REL_L2 = 2e-2
BF16_MAX_ABS = 5e-2


def torch_dtype(name):
    import torch
    return torch.bfloat16 if name == "bf16" else torch.float32


def gpu_decode(cfg, weights, z, io_dtype=None, frames=None, dec=None, keep=False):
    """Decode z[0..T-1] on the GPU; returns float64 numpy [T][C][r_t][H][W]."""
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    io = io_dtype or cfg.dtype
    T = z.shape[0] if frames is None else frames
    own = dec is None
    if own:
        dec = FlashDecoder(cfg, weights, io_dtype=io)
    dec.reset()
    td = torch_dtype(io)
    outs = []
    for t in range(T):
        lat = torch.from_numpy(np.ascontiguousarray(z[t])).to(td).cuda()
        out = torch.empty(cfg.out_shape, dtype=td, device="cuda")
        dec.decode_frame(lat, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert dec.status() == 0
    res = np.stack([o.float().cpu().numpy().astype(np.float64) for o in outs])
    if own and not keep:
        dec.close()
    return (res, dec) if keep else res


def oracle_decode(cfg, weights, z, frames=None):
    return oracle.decode_video(cfg, weights, z, frames)


def errors(got, ref):
    d = got - ref
    return float(np.linalg.norm(d) / np.linalg.norm(ref)), float(np.abs(d).max())


def assert_close(cfg, got, ref, io_dtype=None):
    rel, mx = errors(got, ref)
    if cfg.dtype == "f32":
        assert mx <= FP32_MAX_ABS, f"max abs {mx:.3e} > {FP32_MAX_ABS}"
    else:
        assert rel <= BF16_REL_L2 and mx <= BF16_MAX_ABS, \
            f"rel L2 {rel:.3e} (<= {BF16_REL_L2}), max abs {mx:.3e} (<= {BF16_MAX_ABS})"
    return rel, mx


def small_bf16(**kw):
    """A bf16 configuration with several GEMM/attention tiles and a ragged tail
    (10 x 13 = 130 tokens = one full 128-row tile plus 2 rows)."""
    base = fd_synth.CONFIGS["480p_wan21"].replace(
        name="small_bf16", latent_ch=16, grid_h=10, grid_w=13, patch=1, d_model=256,
        n_heads=4, n_kv_heads=4, head_dim=64, n_blocks=2, window=2, frames=5)
    return base.replace(**kw)
