"""Degenerate and extreme shapes of the streaming step against the oracle:
a single token per frame (every tile ragged, TMA boxes larger than the
tensor), a single head, the largest window the tests afford, the maximum
number of streams, and a single-token paper head.
"""
import numpy as np
import pytest

import fd_synth

from gpu_util import assert_close, gpu_decode, oracle_decode, small_bf16

pytestmark = pytest.mark.gpu

TINY = fd_synth.CONFIGS["tiny_fp32"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from streaming_transformer_video_b200 import lib
    lib()


@pytest.mark.parametrize("cfg", [
    TINY.replace(grid_h=1, grid_w=1, frames=5),                         # L = 1, fp32
    TINY.replace(grid_h=2, grid_w=2, patch=2, frames=4),                # L = 1 after unshuffle
    small_bf16(grid_h=1, grid_w=1, frames=5),                           # L = 1, tcgen05 path
    small_bf16(grid_h=1, grid_w=3, frames=4),                           # 3 tokens
    small_bf16(n_heads=1, n_kv_heads=1, d_model=128, frames=4),          # one head
    small_bf16(grid_h=4, grid_w=4, window=15, frames=18),               # 16-slot ring, wraps
    small_bf16(grid_h=1, grid_w=1, head="paper", n_refine=1, window=1, frames=4),
])
def test_degenerate_shapes_match_oracle(cfg):
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    assert_close(cfg, gpu_decode(cfg, w, z), oracle_decode(cfg, w, z))


def test_maximum_stream_count():
    # 64 streams, each its own video; every stream equals its unbatched decode
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    # both sides with the same key splitting (the automatic choice depends on
    # the number of streams, and splitting changes the summation order)
    cfg = small_bf16(grid_h=2, grid_w=3, frames=3, batch=64, attn_splits=2)
    w = fd_synth.make_weights(cfg)
    videos = [fd_synth.make_latents(cfg, seed=100 + b) for b in range(64)]
    dec = FlashDecoder(cfg, w)
    dec.reset()
    z = torch.from_numpy(np.stack(videos, axis=1)).to(torch.bfloat16).cuda()
    outs = []
    for t in range(cfg.frames):
        out = torch.empty((64,) + tuple(cfg.out_shape), dtype=torch.bfloat16, device="cuda")
        dec.decode_frame(z[t].contiguous(), out)
        outs.append(out)
    torch.cuda.synchronize()
    assert dec.status() == 0
    got = np.stack([o.float().cpu().numpy() for o in outs], axis=1).astype(np.float64)
    dec.close()
    one = cfg.replace(batch=1)
    for b in (0, 17, 63):
        np.testing.assert_array_equal(got[b], gpu_decode(one, w, videos[b]))
