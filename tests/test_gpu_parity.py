"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Tolerances: fp32 max abs <= 1e-4; bf16 rel L2 <= 2e-2 and max abs <= 5e-2.
Ring-slot indexing is checked exactly; causality and the window bound are
checked bit-exactly on the GPU's own outputs.
"""
import numpy as np
import pytest

import fd_synth
import oracle
from oracle import flashdec_oracle as fo

from gpu_util import (assert_close, errors, gpu_decode, oracle_decode, small_bf16,
                      FP32_MAX_ABS)

pytestmark = pytest.mark.gpu

TINY = fd_synth.CONFIGS["tiny_fp32"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from streaming_transformer_video_b200 import lib
    lib()


# ---------------------------------------------------------------- fp32 tiny
@pytest.mark.parametrize("kw", [
    dict(),                                            # the tiny config itself
    dict(frames=7),                                    # ring wrap-around twice
    dict(kv_norm=0, frames=5),
    dict(n_heads=4, n_kv_heads=2, frames=5),           # GQA
    dict(patch=2, grid_h=16, grid_w=16, frames=5),     # PixelUnshuffle x2
    dict(grid_h=5, grid_w=7, frames=5),                # 35 tokens: ragged tiles
    dict(window=0, frames=4),
    dict(window=1, frames=5),
    dict(window=3, frames=6),
    dict(head_dim=64, n_heads=1, n_kv_heads=1, frames=4),
    dict(px_per_token=16, frames=3),
])
def test_tiny_fp32_matches_oracle(kw):
    cfg = TINY.replace(**kw)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    got = gpu_decode(cfg, w, z)
    ref = oracle_decode(cfg, w, z)
    assert_close(cfg, got, ref)


def test_tiny_fp32_io_bf16():
    cfg = TINY
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    zb = fd_synth.make_latents(cfg.replace(dtype="bf16"))   # bf16-representable latents
    got = gpu_decode(cfg, w, zb, io_dtype="bf16")
    ref = oracle_decode(cfg, w, zb)
    rel, mx = errors(got, ref)
    assert mx <= 2.0 ** -8 * np.abs(ref).max() + FP32_MAX_ABS   # output rounding only
    del z


def test_slot_indexing_is_exact():
    # frame t' lives in slot t' mod (W+1), stored after KV-norm and RoPE at its
    # absolute temporal index; each slot must match exactly one window frame.
    cfg = TINY.replace(frames=5)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    _, dec = gpu_decode(cfg, w, z, keep=True)
    ora = oracle.OracleDecoder(cfg, w)
    for t in range(cfg.frames):
        ora.decode_frame(z[t])
    n = np.arange(cfg.L_frm)
    row, col = (n // cfg.tok_w).astype(float), (n % cfg.tok_w).astype(float)
    S = cfg.window + 1
    try:
        for l in range(cfg.n_blocks):
            frames = ora.window_frames(l)
            assert frames == list(range(cfg.frames - S, cfg.frames))
            for slot in range(S):
                k_gpu, v_gpu = dec.read_slot(l, slot, 0), dec.read_slot(l, slot, 1)
                dist = {}
                for f in frames:
                    k, v = ora.cached_kv(l, f)
                    kr = np.stack([fo.rope_3d(k[:, g], np.full(cfg.L_frm, float(f)), row, col,
                                              cfg.rope_theta) for g in range(cfg.n_kv_heads)])
                    vv = np.stack([v[:, g] for g in range(cfg.n_kv_heads)])
                    dist[f] = max(np.abs(k_gpu - kr).max(), np.abs(v_gpu - vv).max())
                best = min(dist, key=dist.get)
                assert best % S == slot, (l, slot, dist)
                assert dist[best] <= FP32_MAX_ABS
    finally:
        dec.close()


# ---------------------------------------------------------------- invariants
def test_gpu_causality_bit_exact():
    cfg = TINY.replace(frames=6)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    base = gpu_decode(cfg, w, z)
    pert = gpu_decode(cfg, w, fd_synth.perturb_frame(z, 4))
    np.testing.assert_array_equal(pert[:4], base[:4])
    assert not np.array_equal(pert[4], base[4])


@pytest.mark.parametrize("cfg", [TINY.replace(n_blocks=1, frames=7),
                                 small_bf16(n_blocks=1, frames=6)])
def test_gpu_window_bound_bit_exact(cfg):
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    base = gpu_decode(cfg, w, z)
    t = cfg.frames - 1
    pert = gpu_decode(cfg, w, fd_synth.perturb_frame(z, t - cfg.window - 1, dtype=cfg.dtype))
    np.testing.assert_array_equal(pert[t], base[t])
    pert = gpu_decode(cfg, w, fd_synth.perturb_frame(z, t - cfg.window, dtype=cfg.dtype))
    assert not np.array_equal(pert[t], base[t])


def test_memory_is_constant_over_200_frames():
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    cfg = TINY.replace(grid_h=4, grid_w=4)
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
    S = cfg.window + 1
    expect = cfg.n_blocks * 2 * cfg.n_kv_heads * S * cfg.L_frm * cfg.head_dim * 4
    assert dec.cache_bytes() >= expect
    dec.close()


def test_reset_restarts_the_video_bit_exact():
    cfg = TINY.replace(frames=5)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    z2 = fd_synth.make_latents(cfg, seed=5)
    first, dec = gpu_decode(cfg, w, z, keep=True)
    gpu_decode(cfg, w, z2, dec=dec)                  # another video on the same handle
    again = gpu_decode(cfg, w, z, dec=dec)           # reset + the first video again
    dec.close()
    np.testing.assert_array_equal(again, first)


@pytest.mark.parametrize("cfg", [TINY, small_bf16(frames=3)])
def test_host_entry_point_matches_device_entry_point(cfg):
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    dev_out = gpu_decode(cfg, w, z)
    td = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    dec = FlashDecoder(cfg, w)
    dec.reset()
    outs = []
    for t in range(z.shape[0]):
        lat = torch.from_numpy(z[t]).to(td).pin_memory()
        out = torch.empty(cfg.out_shape, dtype=td).pin_memory()
        dec.decode_frame_host(lat, out)
        torch.cuda.synchronize()
        outs.append(out.float().numpy().astype(np.float64))
    assert dec.status() == 0
    dec.close()
    np.testing.assert_array_equal(np.stack(outs), dev_out)


def test_nan_latent_propagates_without_failure():
    import torch
    cfg = TINY
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    z[1, 0, 0, 0] = np.nan
    got = gpu_decode(cfg, w, z)
    assert np.isfinite(got[0]).all()
    assert np.isnan(got[1]).any()


# ---------------------------------------------------------------- bf16 (tcgen05)
@pytest.mark.parametrize("kw", [
    dict(),
    dict(kv_norm=0),
    dict(n_heads=4, n_kv_heads=2),
    dict(n_heads=8, n_kv_heads=8, d_model=512),
    dict(patch=2, grid_h=20, grid_w=26),
    dict(window=0, frames=3),
    dict(window=1, frames=5),
    dict(window=3, frames=6),
    dict(grid_h=17, grid_w=23, frames=4),            # 391 tokens: 4 tiles, ragged
    dict(px_per_token=8),
    dict(n_heads=8, n_kv_heads=1, d_model=512),      # GQA, 8 query heads per group
    # FlashDecoder-XL block shape: D=1536, 24 heads, 3 KV groups (GQA ratio 8)
    dict(d_model=1536, n_heads=24, n_kv_heads=3, n_blocks=1, window=1, frames=4),
])
def test_small_bf16_matches_oracle(kw):
    cfg = small_bf16(**kw)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    got = gpu_decode(cfg, w, z)
    ref = oracle_decode(cfg, w, z)
    assert_close(cfg, got, ref)


def test_small_bf16_io_f32():
    cfg = small_bf16()
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    got = gpu_decode(cfg, w, z, io_dtype="f32")
    ref = oracle_decode(cfg, w, z)
    assert_close(cfg, got, ref)


def test_480p_full_size_frames_0_to_3_match_oracle():
    # the full Wan2.1-shaped 480p decoder (1560 tokens, 12 blocks, W=2), in the
    # launch configuration the benchmark times; 4 frames cover the warm-up of
    # the ring and its first wrap-around
    cfg = fd_synth.CONFIGS["480p_wan21"]
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=4)
    got = gpu_decode(cfg, w, z)
    ref = oracle_decode(cfg, w, z)
    assert_close(cfg, got, ref)


@pytest.mark.parametrize("mode", [1, 2])
def test_kernel_timing_modes(mode):
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    cfg = small_bf16(frames=3)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    dec = FlashDecoder(cfg, w, kernel_timing=mode)
    dec.reset()
    lat = torch.from_numpy(z).to(torch.bfloat16).cuda()
    out = torch.empty(cfg.out_shape, dtype=torch.bfloat16, device="cuda")
    for t in range(3):
        dec.decode_frame(lat[t], out)
    times = dec.kernel_ms()
    dec.close()
    kinds = [k for k, _ in times]
    if mode == 1:                       # every kernel of the frame, in launch order
        assert kinds == ["step_begin", "embed"] + \
            ["qkv", "attn", "oproj", "mlp_up", "mlp_down"] * cfg.n_blocks + ["final"]
    else:                               # the attention launches only
        assert kinds == ["attn"] * cfg.n_blocks
    assert all(ms > 0 for _, ms in times)


def test_xl_gqa_480p_full_depth_frames_0_to_2_match_oracle():
    # the FlashDecoder-XL backbone shape (D=1536, 24 query heads sharing 3
    # key/value groups, 20 blocks, one past frame) on the 480p Wan2.2 latent
    cfg = fd_synth.CONFIGS["xl_480p_wan22"]
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=3)
    got = gpu_decode(cfg, w, z)
    ref = oracle_decode(cfg, w, z)
    assert_close(cfg, got, ref)


# ---------------------------------------------------------------- key splitting
@pytest.mark.parametrize("kw", [
    dict(attn_splits=1),
    dict(attn_splits=2),
    dict(attn_splits=4, window=3, frames=6),
    dict(attn_splits=3, grid_h=1, grid_w=1),                  # 1 key tile: empty ranges
    dict(attn_splits=3, n_heads=8, n_kv_heads=1, d_model=512),
    dict(attn_splits=2, head="paper", n_refine=2, window=1, frames=3),
    dict(attn_splits=4, head="paper", n_refine=1, window=1, frames=3, grid_h=12, grid_w=14),
    # one thread issuing both MMA streams (the form large launches take)
    dict(attn_issuer=2),
    dict(attn_issuer=2, attn_splits=3, grid_h=1, grid_w=1),   # empty key ranges
    dict(attn_issuer=2, attn_splits=4, window=3, frames=6),
    dict(attn_issuer=2, head="paper", n_refine=2, window=1, frames=3, grid_h=12, grid_w=14),
])
def test_attention_key_splitting_matches_oracle(kw):
    # each (query tile, head) split over several CTAs, partial results
    # combined by the last one (flash-decoding style), against the oracle
    cfg = small_bf16(**kw)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    assert_close(cfg, gpu_decode(cfg, w, z), oracle_decode(cfg, w, z))


@pytest.mark.parametrize("cfg", [
    small_bf16(attn_splits=2, frames=4),
    small_bf16(head="paper", n_refine=2, window=1, frames=3, grid_h=12, grid_w=14),
    # the 480p workload at full width (its launches take two issuing threads)
    fd_synth.CONFIGS["480p_wan21"].replace(n_blocks=2, frames=4),
])
def test_both_mma_issuer_forms_give_identical_bits(cfg):
    # the same products in the same order per accumulator, whichever threads
    # issue them
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    np.testing.assert_array_equal(gpu_decode(cfg.replace(attn_issuer=1), w, z),
                                  gpu_decode(cfg.replace(attn_issuer=2), w, z))


def test_attention_key_splitting_is_deterministic():
    cfg = small_bf16(attn_splits=3, frames=4)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    a, dec = gpu_decode(cfg, w, z, keep=True)
    b = gpu_decode(cfg, w, z, dec=dec)                      # same handle, reset, again
    dec.close()
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(gpu_decode(cfg, w, z), a)  # a fresh handle

