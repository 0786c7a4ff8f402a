"""The rolling KV cache on the GPU, checked against the oracle.

FlashDecoder paper, Sec. 3.3 "Frame-by-Frame Processing" (Eq. 2): frame t's
keys and values go into the cache, the oldest frame is evicted beyond W+1
frames, and the queries attend to the frames that exist. Sec. 3.4, Step 2:
the refinement blocks stream r_t sub-frames per latent frame through a cache
of r_t (W+1) sub-frames. Sec. 4.3 "Long Video Decoding": positions are
relative to the current window, so videos of any length decode the same way.

Checked here:
  * slot indexing, exactly: ring slot s of the tcgen05 path (bf16), of every
    video stream of a batch and of the refinement ring holds the frame (or
    sub-frame) f with f = s mod capacity, post-RoPE at its absolute index; a
    mirrored refinement ring (all r_t sub-frames through a block in one
    launch) holds f in both copies, slots s and s + capacity;
  * a ring filled with NaN right after the reset never reaches an output:
    a frame reads only slots written since the reset;
  * a stream restarted after a video whose cache holds NaN decodes its new
    video exactly like a fresh handle;
  * long videos: frames 318-319 of a 320-frame video, and frames at absolute
    index 10^9 and 2^40, match the oracle (whose positions are window-relative).
"""
import numpy as np
import pytest

import fd_synth
import oracle
from oracle import flashdec_oracle as fo

from gpu_util import (BF16_MAX_ABS, BF16_REL_L2, FP32_MAX_ABS, assert_close, gpu_decode,
                      small_bf16, torch_dtype)

pytestmark = pytest.mark.gpu

TINY = fd_synth.CONFIGS["tiny_fp32"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from streaming_transformer_video_b200 import lib
    lib()


def _rotated(cfg, k, pos):
    """Oracle keys [L][G][Dh] rotated at absolute temporal index pos -> [G][L][Dh]."""
    n = np.arange(cfg.L_frm)
    row, col = (n // cfg.tok_w).astype(float), (n % cfg.tok_w).astype(float)
    return np.stack([fo.rope_3d(k[:, g], np.full(cfg.L_frm, float(pos)), row, col,
                                cfg.rope_theta) for g in range(cfg.n_kv_heads)])


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _check_ring(cfg, read, candidates, capacity, copies=1):
    """read(slot, kv) -> GPU slot [G][L][Dh]; candidates: {index: (k_rot, v)},
    the frames the window attends to. Frame f must sit in slot f mod capacity
    (and, with two copies, also in that slot + capacity), matching its
    candidate within the value tolerance and every other one by far less.
    Without copies the window fills the ring, so every slot is checked."""
    tol = 2e-2 if cfg.dtype == "bf16" else 1e-4
    assert len(candidates) == capacity if copies == 1 else len(candidates) < capacity
    for f in sorted(candidates):
        for c in range(copies):
            slot = f % capacity + c * capacity
            k_gpu, v_gpu = read(slot, 0), read(slot, 1)
            dist = {g: max(_rel(k_gpu, kr), _rel(v_gpu, vv)) for g, (kr, vv) in candidates.items()}
            best = min(dist, key=dist.get)
            assert best == f, (slot, dist)
            assert dist[best] <= tol, (slot, dist)
            others = [d for g, d in dist.items() if g != best]
            assert not others or min(others) > 10 * tol, (slot, dist)


def _backbone_candidates(cfg, ora, l):
    out = {}
    for f in ora.window_frames(l):
        k, v = ora.cached_kv(l, f)
        out[f] = (_rotated(cfg, k, f), np.stack([v[:, g] for g in range(cfg.n_kv_heads)]))
    return out


def _decode_keep(cfg, w, z, frames):
    got, dec = gpu_decode(cfg, w, z, frames=frames, keep=True)
    return got, dec


@pytest.mark.parametrize("cfg", [
    small_bf16(window=2, frames=6),                     # wraps: frames 3..5 in slots 0..2
    small_bf16(window=3, frames=7, grid_h=17, grid_w=23),   # 391 tokens, 4 slots
    small_bf16(window=1, n_heads=8, n_kv_heads=2, d_model=512, frames=5),   # GQA
])
def test_bf16_ring_slots_hold_their_frames_exactly(cfg):
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    _, dec = _decode_keep(cfg, w, z, cfg.frames)
    ora = oracle.OracleDecoder(cfg, w)
    for t in range(cfg.frames):
        ora.decode_frame(z[t])
    try:
        for l in range(cfg.n_blocks):
            assert ora.window_frames(l) == list(range(cfg.frames - cfg.window - 1, cfg.frames))
            _check_ring(cfg, lambda s, kv: dec.read_ring(l, 0, s, kv),
                        _backbone_candidates(cfg, ora, l), cfg.window + 1)
    finally:
        dec.close()


def test_every_stream_of_a_batch_has_its_own_exact_ring():
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    cfg = small_bf16(batch=3, window=2, frames=5)
    w = fd_synth.make_weights(cfg)
    videos = [fd_synth.make_latents(cfg, seed=1 + b) for b in range(cfg.batch)]
    # stream 2 is restarted after 2 frames: its ring then holds frames 0..2 of
    # its new video while the others hold frames 2..4
    dec = FlashDecoder(cfg, w)
    try:
        dec.reset()
        td = torch_dtype(cfg.dtype)
        z = torch.from_numpy(np.stack(videos, axis=1)).to(td).cuda()
        out = torch.empty((cfg.batch,) + tuple(cfg.out_shape), dtype=td, device="cuda")
        new2 = fd_synth.make_latents(cfg, seed=99)
        zz = z.clone()
        zz[2:, 2] = torch.from_numpy(new2[:cfg.frames - 2]).to(td).cuda()
        for t in range(cfg.frames):
            if t == 2:
                dec.reset_stream(2)
            dec.decode_frame(zz[t].contiguous(), out)
        torch.cuda.synchronize()
        assert dec.status() == 0
        for b, video, T in ((0, videos[0], cfg.frames), (1, videos[1], cfg.frames),
                            (2, new2, cfg.frames - 2)):
            ora = oracle.OracleDecoder(cfg.replace(batch=1), w)
            for t in range(T):
                ora.decode_frame(video[t])
            assert dec.frame_index(b) == T
            for l in range(cfg.n_blocks):
                _check_ring(cfg, lambda s, kv: dec.read_ring(l, b, s, kv),
                            _backbone_candidates(cfg, ora, l), cfg.window + 1)
    finally:
        dec.close()


@pytest.mark.parametrize("cfg", [
    small_bf16(head="paper", n_refine=2, window=1, frames=3),    # 12 sub-frames, 8 slots
    # 168 tokens: all 4 sub-frames per launch, mirrored ring of 11 slots x 2
    small_bf16(head="paper", n_refine=2, window=1, frames=4, grid_h=12, grid_w=14),
    small_bf16(head="paper", n_refine=1, window=2, r_t=2, frames=5, grid_h=12, grid_w=14),
    TINY.replace(head="paper", n_refine=1, window=1, r_t=2, frames=5),   # fp32 path
])
def test_refinement_ring_slots_hold_their_sub_frames_exactly(cfg):
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    _, dec = _decode_keep(cfg, w, z, cfg.frames)
    ora = oracle.OracleDecoder(cfg, w)
    for t in range(cfg.frames):
        ora.decode_frame(z[t])
    window = cfg.r_t * (cfg.window + 1)
    try:
        for l in range(cfg.n_refine):
            cap, copies = dec.ring_layout(cfg.n_blocks + l)
            assert (cap, copies) in ((window, 1), (cfg.r_t * (cfg.window + 2) - 1, 2))
            subs = ora.refine_window(l)
            assert subs == list(range(cfg.frames * cfg.r_t - window, cfg.frames * cfg.r_t))
            cand = {}
            for s in subs:
                k, v = ora.refine_cached_kv(l, s)
                cand[s] = (_rotated(cfg, k, s), np.stack([v[:, g] for g in range(cfg.n_kv_heads)]))
            _check_ring(cfg, lambda s, kv: dec.read_ring(cfg.n_blocks + l, 0, s, kv), cand, cap,
                        copies)
        # and the backbone ring of the same handle
        for l in range(cfg.n_blocks):
            _check_ring(cfg, lambda s, kv: dec.read_ring(l, 0, s, kv),
                        _backbone_candidates(cfg, ora, l), cfg.window + 1)
    finally:
        dec.close()


# ---------------------------------------------------------------- NaN ring
def _decode(cfg, w, videos, poison=False, dec=None):
    """[B][T][...] through one handle; poison fills the ring with NaN after
    the reset."""
    import torch
    from streaming_transformer_video_b200 import FlashDecoder, flashdec as fdb
    own = dec is None
    if own:
        dec = FlashDecoder(cfg, w)
    dec.reset()
    if poison:
        dec.debug_poison(fdb.FD_POISON_RING)
    td = torch_dtype(cfg.dtype)
    B = len(videos)
    z = torch.from_numpy(np.stack(videos, axis=1)).to(td).cuda()
    outs = []
    for t in range(z.shape[0]):
        out = torch.empty((B,) + tuple(cfg.out_shape), dtype=td, device="cuda")
        dec.decode_frame(z[t].contiguous(), out)
        outs.append(out)
    torch.cuda.synchronize()
    assert dec.status() == 0
    res = np.stack([o.float().cpu().numpy() for o in outs], axis=1)
    if own:
        dec.close()
    return res


@pytest.mark.parametrize("cfg", [
    TINY.replace(frames=5),
    TINY.replace(grid_h=5, grid_w=7, frames=5),                      # 35 tokens
    small_bf16(frames=5),                                            # 130 tokens: partial key tile
    small_bf16(window=3, grid_h=17, grid_w=23, frames=6, attn_splits=3),
    small_bf16(batch=2, frames=4),
    small_bf16(head="paper", n_refine=2, window=1, frames=3),        # refinement ring too
    # mirrored refinement ring (sub-frames batched), two streams
    small_bf16(head="paper", n_refine=2, window=1, frames=4, grid_h=12, grid_w=14, batch=2),
    TINY.replace(head="paper", n_refine=1, window=1, r_t=2, frames=4),
])
def test_nan_poisoned_ring_never_reaches_outputs(cfg):
    w = fd_synth.make_weights(cfg)
    videos = [fd_synth.make_latents(cfg, seed=1 + b) for b in range(cfg.batch)]
    clean = _decode(cfg, w, videos)
    poisoned = _decode(cfg, w, videos, poison=True)
    assert np.isfinite(poisoned).all()
    np.testing.assert_array_equal(poisoned, clean)
    ref = oracle.decode_video(cfg.replace(batch=1), w, videos[0])
    assert_close(cfg, poisoned[0].astype(np.float64), ref)


@pytest.mark.parametrize("cfg", [
    small_bf16(batch=2, frames=4),
    small_bf16(batch=2, frames=4, head="paper", n_refine=1, window=1, grid_h=12, grid_w=14),
])
def test_restart_after_a_nan_video_decodes_like_a_fresh_handle(cfg):
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    w = fd_synth.make_weights(cfg)
    v0 = fd_synth.make_latents(cfg, frames=7, seed=1)
    bad = np.full((3,) + v0.shape[1:], np.nan, dtype=np.float32)
    new = fd_synth.make_latents(cfg, seed=5)
    td = torch_dtype(cfg.dtype)
    dec = FlashDecoder(cfg, w)
    try:
        dec.reset()
        out = torch.empty((2,) + tuple(cfg.out_shape), dtype=td, device="cuda")
        got = []
        for t in range(7):
            z1 = bad[t] if t < 3 else new[t - 3]
            if t == 3:
                dec.reset_stream(1)              # stream 1's ring is full of NaN here
            lat = torch.from_numpy(np.stack([v0[t], z1])).to(td).cuda()
            dec.decode_frame(lat, out)
            if t >= 3:
                got.append(out[1].float().cpu().numpy())
        torch.cuda.synchronize()
        assert dec.status() == 0
    finally:
        dec.close()
    got = np.stack(got)
    assert np.isfinite(got).all()
    fresh = _decode(cfg.replace(batch=1), w, [new])[0]
    np.testing.assert_array_equal(got, fresh)


# ---------------------------------------------------------------- long videos
@pytest.mark.parametrize("cfg", [TINY, small_bf16()])
def test_frames_318_and_319_of_a_320_frame_video_match_the_oracle(cfg):
    T = 320
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=T)
    got = gpu_decode(cfg, w, z, frames=T)
    # frame t depends on frames t - n_blocks W .. t only (stacked windows):
    # the oracle, started n_blocks W + 1 frames before frame 318, gives
    # frames 318 and 319 exactly as a 320-frame run would
    s0 = T - 2 - cfg.n_blocks * cfg.window
    ref = oracle.decode_video(cfg, w, z[s0:])[-2:]
    assert_close(cfg, got[-2:], ref)


@pytest.mark.parametrize("t0", [10 ** 9 + 3, 2 ** 40 + 1])
@pytest.mark.parametrize("cfg", [TINY, small_bf16()])
def test_frames_at_a_very_large_index_match_the_oracle(cfg, t0):
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    K = cfg.n_blocks * cfg.window + 3
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=K)
    td = torch_dtype(cfg.dtype)
    dec = FlashDecoder(cfg, w)
    try:
        dec.reset()
        dec.debug_set_frame_index(t0)
        outs = []
        for t in range(K):
            out = torch.empty(cfg.out_shape, dtype=td, device="cuda")
            dec.decode_frame(torch.from_numpy(z[t]).to(td).cuda(), out)
            outs.append(out)
        torch.cuda.synchronize()
        assert dec.status() == 0
        assert dec.frame_index() == t0 + K
        got = np.stack([o.float().cpu().numpy().astype(np.float64) for o in outs])
    finally:
        dec.close()
    ref = oracle.decode_video(cfg, w, z)
    # the first n_blocks W frames after the jump still read slots left by the
    # reset; from then on the window is the video's own
    n = cfg.n_blocks * cfg.window
    assert_close(cfg, got[n:], ref[n:])
