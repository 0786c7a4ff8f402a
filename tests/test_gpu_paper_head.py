"""Parity of the CUDA path with the CPU oracle for the paper's output head
(FlashDecoder paper, Sec. 3.4): temporal upsampling (Eq. 3), refinement
blocks streaming r_t sub-frames per latent frame, each attending to the last
r_t (W+1) sub-frames, RMSNorm + 2-layer spatial MLP + PixelShuffle per
sub-frame.

The bf16 path runs the r_t sub-frames of a latent frame through each
refinement block in one launch per kernel when L_frm is a multiple of 8
(a mirrored ring of r_t (W+2) - 1 sub-frames), else one sub-frame at a time;
both are checked here (BATCHED: 12 x 14 = 168 tokens, two query tiles, the
second ragged).

Tolerances as for the linear head: fp32 max abs <= 1e-4; bf16 rel L2 <= 2e-2
and max abs <= 5e-2. Causality, the dependence bound and reset are checked
bit-exactly on the GPU's own outputs.
"""
import numpy as np
import pytest

import fd_synth

from gpu_util import assert_close, gpu_decode, oracle_decode, small_bf16

pytestmark = pytest.mark.gpu

TINY_PAPER = fd_synth.CONFIGS["tiny_fp32"].replace(head="paper", n_refine=2)


def small_bf16_paper(**kw):
    return small_bf16(head="paper", n_refine=2).replace(**kw)


BATCHED = dict(grid_h=12, grid_w=14)      # 168 tokens, a multiple of 8


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from streaming_transformer_video_b200 import lib
    lib()


@pytest.mark.parametrize("kw", [
    dict(),
    dict(frames=7),                                    # refinement ring of 12 wraps twice
    dict(n_refine=1, frames=4),
    dict(window=0, frames=4),                          # ring of r_t sub-frames
    dict(window=1, r_t=2, frames=5),
    dict(r_t=1, frames=4),                             # no upsampling: one sub-frame
    dict(n_heads=4, n_kv_heads=2, frames=4),           # GQA in every block
    dict(grid_h=5, grid_w=7, frames=4),                # 35 tokens: ragged tiles
    dict(px_per_token=16, out_ch=3, frames=3),
    dict(kv_norm=0, frames=4),
])
def test_tiny_fp32_paper_head_matches_oracle(kw):
    cfg = TINY_PAPER.replace(**kw)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    assert_close(cfg, gpu_decode(cfg, w, z), oracle_decode(cfg, w, z))


@pytest.mark.parametrize("kw", [
    dict(),
    dict(window=1, frames=4),
    dict(n_refine=1, frames=4),
    dict(n_heads=8, n_kv_heads=1, d_model=512, frames=4),   # GQA ratio 8
    dict(grid_h=17, grid_w=23, frames=4),                   # 391 tokens, ragged
    dict(px_per_token=8, frames=4),
    # FlashDecoder-XL block shape (D=1536, 24 heads, 3 KV groups) with its
    # two refinement blocks and the W_frm = 2 window
    dict(d_model=1536, n_heads=24, n_kv_heads=3, n_blocks=1, window=1, frames=3),
    # all sub-frames of a refinement block in one launch
    dict(BATCHED, frames=5),
    dict(BATCHED, window=1, frames=7),                      # ring of 11 wraps twice
    dict(BATCHED, window=0, frames=4),                      # 7 slots, windows of 4
    dict(BATCHED, r_t=2, window=1, frames=6),
    dict(BATCHED, r_t=1, frames=4),                         # one sub-frame: W+1 slots, mirrored
    dict(BATCHED, n_refine=1, frames=4),
    dict(BATCHED, attn_splits=3, frames=5),                 # split combine over sub-frames
    dict(grid_h=8, grid_w=16, n_heads=8, n_kv_heads=2, d_model=512, frames=4),   # 128 tokens, GQA
    dict(BATCHED, d_model=1536, n_heads=24, n_kv_heads=3, n_blocks=1, window=1, frames=3),
])
def test_small_bf16_paper_head_matches_oracle(kw):
    cfg = small_bf16_paper(**kw)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    assert_close(cfg, gpu_decode(cfg, w, z), oracle_decode(cfg, w, z))


def test_paper_head_causality_bit_exact():
    cfg = TINY_PAPER.replace(frames=6)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    base = gpu_decode(cfg, w, z)
    pert = gpu_decode(cfg, w, fd_synth.perturb_frame(z, 4))
    np.testing.assert_array_equal(pert[:4], base[:4])
    assert not np.array_equal(pert[4], base[4])


@pytest.mark.parametrize("cfg", [TINY_PAPER.replace(n_blocks=1, n_refine=1, window=1, frames=5),
                                 small_bf16_paper(n_blocks=1, n_refine=1, window=1, frames=5)])
def test_paper_head_dependence_bound_bit_exact(cfg):
    # one backbone block sees latent frames t-W..t; sub-frame 0 of frame t sees
    # sub-frames back to (t-W-1) r_t + 1, i.e. part of frame t-W-1, whose
    # backbone output saw latents back to t-2W-1. So frame t depends on
    # latent t-2W-1 and on nothing older.
    W = cfg.window
    t = cfg.frames - 1
    assert t - 2 * W - 2 >= 0
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    base = gpu_decode(cfg, w, z)
    pert = gpu_decode(cfg, w, fd_synth.perturb_frame(z, t - 2 * W - 2, dtype=cfg.dtype))
    np.testing.assert_array_equal(pert[t], base[t])
    pert = gpu_decode(cfg, w, fd_synth.perturb_frame(z, t - 2 * W - 1, dtype=cfg.dtype))
    assert not np.array_equal(pert[t], base[t])


def test_paper_head_reset_and_host_entry_point():
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    cfg = small_bf16_paper(frames=4)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    z2 = fd_synth.make_latents(cfg, seed=5)
    first, dec = gpu_decode(cfg, w, z, keep=True)
    gpu_decode(cfg, w, z2, dec=dec)                 # another video on the same handle
    np.testing.assert_array_equal(gpu_decode(cfg, w, z, dec=dec), first)
    dec.reset()
    outs = []
    for t in range(z.shape[0]):
        lat = torch.from_numpy(z[t]).to(torch.bfloat16).pin_memory()
        out = torch.empty(cfg.out_shape, dtype=torch.bfloat16).pin_memory()
        dec.decode_frame_host(lat, out)
        torch.cuda.synchronize()
        outs.append(out.float().numpy().astype(np.float64))
    assert dec.status() == 0
    dec.close()
    np.testing.assert_array_equal(np.stack(outs), first)


def test_paper_head_memory_is_constant_over_200_frames():
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    cfg = TINY_PAPER.replace(grid_h=4, grid_w=4)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=200)
    dec = FlashDecoder(cfg, w)
    dec.reset()
    lat = torch.from_numpy(z).cuda()
    out = torch.empty(cfg.out_shape, device="cuda")
    before = (dec.device_bytes(), torch.cuda.memory_allocated())
    free0 = torch.cuda.mem_get_info()[0]
    for t in range(200):
        dec.decode_frame(lat[t], out)
    torch.cuda.synchronize()
    assert dec.status() == 0
    assert dec.frame_index() == 200
    assert (dec.device_bytes(), torch.cuda.memory_allocated()) == before
    assert abs(torch.cuda.mem_get_info()[0] - free0) < (4 << 20)
    kv = 2 * cfg.n_kv_heads * cfg.L_frm * cfg.head_dim * 4
    expect = cfg.n_blocks * (cfg.window + 1) * kv + \
        cfg.n_refine * cfg.r_t * (cfg.window + 1) * kv
    assert dec.cache_bytes() >= expect
    dec.close()


@pytest.mark.parametrize("batched", [False, True])
def test_paper_head_kernel_sequence(batched):
    import torch
    import bench
    from streaming_transformer_video_b200 import FlashDecoder
    cfg = small_bf16_paper(frames=2, **(BATCHED if batched else {}))
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    dec = FlashDecoder(cfg, w, kernel_timing=1)
    dec.reset()
    lat = torch.from_numpy(z).to(torch.bfloat16).cuda()
    out = torch.empty(cfg.out_shape, dtype=torch.bfloat16, device="cuda")
    for t in range(2):
        dec.decode_frame(lat[t], out)
    kinds = [k for k, _ in dec.kernel_ms()]
    slots, copies = dec.ring_layout(cfg.n_blocks)
    dec.close()
    block = ["qkv", "attn", "oproj", "mlp_up", "mlp_down"]
    launches = 1 if batched else cfg.r_t          # launches of each refinement kernel
    assert (copies == 2) == batched == bench.refine_batched(cfg)
    assert kinds == ["step_begin", "embed"] + block * cfg.n_blocks + ["upsample"] + \
        (block * cfg.n_refine + ["spatial", "final"]) * launches
    assert len(kinds) == bench.kernels_per_frame(cfg)


@pytest.mark.parametrize("cfg,layout", [
    (small_bf16_paper(**BATCHED), (4 * 4 - 1, 2)),                 # r_t (W+2) - 1, mirrored
    (small_bf16_paper(**BATCHED, window=1, r_t=2), (2 * 3 - 1, 2)),
    (small_bf16_paper(), (4 * 3, 1)),                               # 130 tokens: r_t (W+1)
    (TINY_PAPER, (TINY_PAPER.r_t * (TINY_PAPER.window + 1), 1)),    # fp32 path
])
def test_refinement_ring_layout(cfg, layout):
    from streaming_transformer_video_b200 import FlashDecoder
    w = fd_synth.make_weights(cfg)
    dec = FlashDecoder(cfg, w)
    try:
        assert dec.ring_layout(0) == (cfg.window + 1, 1)
        for l in range(cfg.n_refine):
            assert dec.ring_layout(cfg.n_blocks + l) == layout
        # the cache holds every slot and copy
        kv = 2 * cfg.n_kv_heads * cfg.L_frm * cfg.head_dim * (2 if cfg.dtype == "bf16" else 4)
        assert dec.cache_bytes() >= (cfg.n_blocks * (cfg.window + 1) +
                                     cfg.n_refine * layout[0] * layout[1]) * kv
    finally:
        dec.close()


def test_xl_480p_paper_head_frames_0_to_2_match_oracle():
    # FlashDecoder-XL as the paper describes it: D=1536, 24 query heads in 3
    # key/value groups, 20 backbone blocks + 2 refinement blocks, W_frm = 2,
    # on the 480p Wan2.2 latent (1560 tokens), full size
    cfg = fd_synth.CONFIGS["xl_480p_wan22_paper"]
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=3)
    assert_close(cfg, gpu_decode(cfg, w, z), oracle_decode(cfg, w, z))
