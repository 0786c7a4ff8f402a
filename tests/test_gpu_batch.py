"""Multi-stream batching: B independent videos decoded by one handle, one
latent frame of each per call ([FD] Eq. 1 carries a batch dimension B; the
streaming step of Sec. 3.3 is independent per video).

Each output row of every kernel depends only on its own stream's inputs and
is computed with the same instruction sequence whatever the batch size, so
stream b of a batched decode must equal the unbatched decode of video b
bit-exactly; that, plus one direct oracle comparison, is what is tested.
Streams keep their own frame counters (fd_reset_stream restarts one).
"""
import numpy as np
import pytest

import fd_synth

from gpu_util import assert_close, gpu_decode, oracle_decode, small_bf16, torch_dtype

pytestmark = pytest.mark.gpu

TINY = fd_synth.CONFIGS["tiny_fp32"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from streaming_transformer_video_b200 import lib
    lib()


def batched_decode(cfg, weights, videos, dec=None, reset=True):
    """videos: list of B latent videos [T][C'][H'][W']; returns [B][T][...]
    float64 through one handle with cfg.batch = B."""
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    B, T = len(videos), videos[0].shape[0]
    assert cfg.batch == B
    own = dec is None
    if own:
        dec = FlashDecoder(cfg, weights)
    if reset:
        dec.reset()
    td = torch_dtype(cfg.dtype)
    z = torch.from_numpy(np.stack(videos, axis=1)).to(td).cuda()       # [T][B][...]
    outs = []
    for t in range(T):
        out = torch.empty((B,) + tuple(cfg.out_shape), dtype=td, device="cuda")
        dec.decode_frame(z[t].contiguous(), out)
        outs.append(out)
    torch.cuda.synchronize()
    assert dec.status() == 0
    res = np.stack([o.float().cpu().numpy().astype(np.float64) for o in outs], axis=1)
    if own:
        dec.close()
    return res


def _videos(cfg, B, frames=None):
    return [fd_synth.make_latents(cfg, frames=frames, seed=1 + b) for b in range(B)]


@pytest.mark.parametrize("cfg", [
    TINY.replace(batch=3, frames=5),                                    # CUDA-core path
    small_bf16(batch=3, frames=4),
    small_bf16(batch=2, grid_h=17, grid_w=23, frames=3),                 # 391 tokens per stream
    small_bf16(batch=2, n_heads=8, n_kv_heads=1, d_model=512, frames=3),  # GQA
    small_bf16(batch=2, head="paper", n_refine=2, window=1, frames=3),   # paper head
    # paper head, 168 tokens: all sub-frames of both streams in one launch per kernel
    small_bf16(batch=2, head="paper", n_refine=2, window=1, frames=3, grid_h=12, grid_w=14),
])
def test_batched_streams_equal_unbatched_decodes_bit_exact(cfg):
    w = fd_synth.make_weights(cfg)
    videos = _videos(cfg, cfg.batch)
    got = batched_decode(cfg, w, videos)
    for b, z in enumerate(videos):
        np.testing.assert_array_equal(got[b], gpu_decode(cfg.replace(batch=1), w, z))


def test_batched_fp8_streams_equal_unbatched_bit_exact():
    import oracle
    cfg = small_bf16(batch=2, frames=3)
    w = fd_synth.make_weights(cfg)
    videos = _videos(cfg, 2)
    w8 = {**w, **oracle.calibrate_fp8(cfg.replace(batch=1), w, videos[0])}
    c8 = cfg.replace(mlp_fp8=1)
    got = batched_decode(c8, w8, videos)
    for b, z in enumerate(videos):
        np.testing.assert_array_equal(got[b], gpu_decode(c8.replace(batch=1), w8, z))


def test_batched_ragged_streams_match_oracle():
    cfg = small_bf16(batch=3, grid_h=17, grid_w=23, frames=4)
    w = fd_synth.make_weights(cfg)
    videos = _videos(cfg, 3)
    got = batched_decode(cfg, w, videos)
    for b, z in enumerate(videos):
        assert_close(cfg, got[b], oracle_decode(cfg.replace(batch=1), w, z))


def test_streams_keep_their_own_positions():
    # stream 1 restarts with a new video after 3 frames while stream 0 goes on
    from streaming_transformer_video_b200 import FlashDecoder
    cfg = small_bf16(batch=2, frames=6)
    w = fd_synth.make_weights(cfg)
    a, b0, c = (fd_synth.make_latents(cfg, seed=s) for s in (1, 2, 3))
    dec = FlashDecoder(cfg, w)
    try:
        first = batched_decode(cfg, w, [a[:3], b0[:3]], dec=dec)
        dec.reset_stream(1)
        second = batched_decode(cfg, w, [a[3:], c[:3]], dec=dec, reset=False)
        assert dec.frame_index(0) == 6 and dec.frame_index(1) == 3
    finally:
        dec.close()
    one = cfg.replace(batch=1)
    ref_a = gpu_decode(one, w, a)
    np.testing.assert_array_equal(np.concatenate([first[0], second[0]]), ref_a)
    np.testing.assert_array_equal(first[1], gpu_decode(one, w, b0[:3]))
    np.testing.assert_array_equal(second[1], gpu_decode(one, w, c[:3]))


def test_batched_memory_and_cache_scale_with_streams():
    from streaming_transformer_video_b200 import FlashDecoder
    cfg = small_bf16(frames=2)
    w = fd_synth.make_weights(cfg)
    d1 = FlashDecoder(cfg, w)
    d4 = FlashDecoder(cfg.replace(batch=4), w)
    try:
        assert d4.cache_bytes() == 4 * d1.cache_bytes()
    finally:
        d1.close()
        d4.close()
