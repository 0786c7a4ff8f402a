"""fd_decode_frame_static_scratch: the frame step with the attention's
key-splitting scratch in the library's fixed device array instead of memory
allocated by fd_create, for callers that cannot allocate device memory while
they decode (a pre-planned memory pool, or a latency budget that a cudaMalloc
between frames would break). It must give exactly what fd_decode_frame gives,
on consecutive calls and when handles of different sizes take turns on the
array, really use the array rather than the handle's own scratch, leave the
handle's own graph as it was, and refuse handles whose scratch does not fit or
that belong to another device.
"""
import numpy as np
import pytest

import fd_synth

from gpu_util import small_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from streaming_transformer_video_b200 import lib
    lib()


def _frames(cfg, z):
    import torch
    lat = torch.from_numpy(z).to(torch.bfloat16).cuda()
    outs = [torch.empty(cfg.out_shape, dtype=torch.bfloat16, device="cuda") for _ in range(z.shape[0])]
    return lat, outs


def test_static_scratch_equals_decode_frame_on_two_calls_in_a_row():
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    cfg = small_bf16(attn_splits=3, frames=3)          # attention splits: scratch in use
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    lat, out_a = _frames(cfg, z)
    _, out_b = _frames(cfg, z)
    a, b = FlashDecoder(cfg, w), FlashDecoder(cfg, w)
    try:
        a.reset()
        b.reset()
        for t in range(2):                             # two calls in a row
            a.decode_frame(lat[t], out_a[t])
            b.decode_frame_static_scratch(lat[t], out_b[t])
        # the handle's graph is back on its own scratch afterwards
        a.decode_frame(lat[2], out_a[2])
        b.decode_frame(lat[2], out_b[2])
        torch.cuda.synchronize()
        assert a.status() == 0 and b.status() == 0
        for t in range(3):
            np.testing.assert_array_equal(out_b[t].float().cpu().numpy(),
                                          out_a[t].float().cpu().numpy())
    finally:
        a.close()
        b.close()


def test_two_handles_of_different_sizes_take_turns_on_the_array():
    # different split counts and grids put each handle's partials over the
    # other's: every call must still equal that handle's own fd_decode_frame
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    cfgs = [small_bf16(attn_splits=2, frames=4),
            small_bf16(attn_splits=3, grid_h=17, grid_w=23, frames=4),
            # two attention launch shapes in one handle: a frame, and all
            # refinement sub-frames at once (more units on the array)
            small_bf16(attn_splits=2, head="paper", n_refine=1, window=1, grid_h=12, grid_w=14,
                       frames=4)]
    ref, fixed, lats, decs = [], [], [], []
    try:
        for cfg in cfgs:
            w = fd_synth.make_weights(cfg)
            lat, outs = _frames(cfg, fd_synth.make_latents(cfg))
            _, outs_fixed = _frames(cfg, fd_synth.make_latents(cfg))
            a, b = FlashDecoder(cfg, w), FlashDecoder(cfg, w)
            a.reset()
            b.reset()
            for t in range(cfg.frames):
                a.decode_frame(lat[t], outs[t])
            ref.append(outs)
            fixed.append(outs_fixed)
            lats.append(lat)
            decs += [a, b]
        for t in range(4):                             # alternate on one stream
            for i in range(len(cfgs)):
                decs[2 * i + 1].decode_frame_static_scratch(lats[i][t], fixed[i][t])
        torch.cuda.synchronize()
        for i in range(len(cfgs)):
            assert decs[2 * i + 1].status() == 0
            for t in range(4):
                np.testing.assert_array_equal(fixed[i][t].float().cpu().numpy(),
                                              ref[i][t].float().cpu().numpy())
    finally:
        for d in decs:
            d.close()


def test_the_fixed_array_is_used_and_the_handle_scratch_left_alone():
    # garbage in the handle's own split counters breaks its own combine (the
    # positive control), but not the fixed-array call, which clears its own
    import torch
    from streaming_transformer_video_b200 import FlashDecoder, flashdec as fdb
    cfg = small_bf16(attn_splits=3, frames=3)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    lat, out_a = _frames(cfg, z)
    _, out_b = _frames(cfg, z)
    _, out_c = _frames(cfg, z)
    a, b, c = FlashDecoder(cfg, w), FlashDecoder(cfg, w), FlashDecoder(cfg, w)
    try:
        for d in (a, b, c):
            d.reset()
        b.debug_poison(fdb.FD_POISON_SPLIT_COUNTERS)
        c.debug_poison(fdb.FD_POISON_SPLIT_COUNTERS)
        for t in range(cfg.frames):
            a.decode_frame(lat[t], out_a[t])
            b.decode_frame_static_scratch(lat[t], out_b[t])
            c.decode_frame(lat[t], out_c[t])
        torch.cuda.synchronize()
        assert a.status() == 0 and b.status() == 0 and c.status() == 0
        for t in range(cfg.frames):
            np.testing.assert_array_equal(out_b[t].float().cpu().numpy(),
                                          out_a[t].float().cpu().numpy())
        assert not np.array_equal(out_c[0].float().cpu().numpy(), out_a[0].float().cpu().numpy())
    finally:
        a.close()
        b.close()
        c.close()


def test_another_device_is_refused():
    import torch
    from streaming_transformer_video_b200 import FlashDecoder, flashdec as fdb
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two CUDA devices")
    cfg = small_bf16(attn_splits=2, frames=1)
    w = fd_synth.make_weights(cfg)
    lat, outs = _frames(cfg, fd_synth.make_latents(cfg))
    dec = FlashDecoder(cfg, w)
    try:
        dec.reset()
        torch.cuda.synchronize()
        with torch.cuda.device(1):
            with pytest.raises(fdb.FDError) as e:
                dec.decode_frame_static_scratch(lat[0], outs[0])
        assert e.value.code == fdb.FD_ERR_INVALID_ARG
        assert dec.frame_index() == 0
    finally:
        dec.close()


def test_handle_without_splitting_runs_the_plain_step():
    import torch
    from streaming_transformer_video_b200 import FlashDecoder
    cfg = small_bf16(attn_splits=1, frames=2)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    lat, out_a = _frames(cfg, z)
    _, out_b = _frames(cfg, z)
    a, b = FlashDecoder(cfg, w), FlashDecoder(cfg, w)
    try:
        a.reset()
        b.reset()
        for t in range(2):
            a.decode_frame(lat[t], out_a[t])
            b.decode_frame_static_scratch(lat[t], out_b[t])
        torch.cuda.synchronize()
        for t in range(2):
            np.testing.assert_array_equal(out_b[t].float().cpu().numpy(),
                                          out_a[t].float().cpu().numpy())
    finally:
        a.close()
        b.close()


def test_oversize_scratch_is_refused():
    import torch
    from streaming_transformer_video_b200 import FlashDecoder, flashdec as fdb
    # 13 query tiles x 16 heads x 4 splits x 33 KB = 27 MB > the fixed 8 MiB
    cfg = fd_synth.CONFIGS["480p_wan21"].replace(attn_splits=4)
    w = fd_synth.make_weights(cfg)
    dec = FlashDecoder(cfg, w)
    try:
        dec.reset()
        lat = torch.zeros((cfg.latent_ch, cfg.grid_h, cfg.grid_w), dtype=torch.bfloat16, device="cuda")
        out = torch.empty(cfg.out_shape, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(fdb.FDError) as e:
            dec.decode_frame_static_scratch(lat, out)
        assert e.value.code == fdb.FD_ERR_UNSUPPORTED
        assert dec.frame_index() == 0                  # nothing was enqueued
    finally:
        dec.close()
