"""Host-side arithmetic of the benchmark, pinned to independent figures.

- FLOPs per 1080p latent frame: 16.43 TFLOP in the workload's scope table
  (24 N D^2 per block for QKV, O-projection and MLP, 4 N (W+1)N D for
  attention, plus the embedding and the final projection).
- The number of kernels per frame: counted by hand from the per-frame
  sequence (the GPU test of the timing mode checks the same list on the
  device).
- Throughput of N replicas x B streams: pixel frames over the slowest rank.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import fd_synth  # noqa: E402

C = fd_synth.CONFIGS


def test_flops_per_1080p_frame_match_the_scope_table():
    total, attn = bench.flops_per_frame(C["1080p_wan22"])
    assert total / 1e12 == pytest.approx(16.43, abs=0.005)
    assert attn / 1e12 == pytest.approx(13.09, abs=0.005)
    # and each part from its closed form
    L, D, nb = 8160, 1024, 16
    assert attn == nb * 4 * L * (3 * L) * D
    gemm = nb * 24 * L * D * D + 2 * L * 48 * D + 2 * L * D * 3072
    assert total == gemm + attn


def test_flops_of_the_480p_and_720p_frames_match_the_scope_table():
    for name, tf in [("480p_wan21", 0.840), ("720p_wan21", 3.021), ("long720p_wan22", 4.021)]:
        assert bench.flops_per_frame(C[name])[0] / 1e12 == pytest.approx(tf, abs=0.0015), name


def test_paper_head_flops_count_refinement_windows_and_sub_frames():
    cfg = C["xl_480p_wan22_paper"]
    L, D, H, G, Dh = cfg.L_frm, 1536, 24, 3, 64
    attn = bench.attn_flops_per_launch(cfg)
    # bf16, L = 1560 = 8 x 195: all r_t sub-frames of a refinement block in one launch
    assert bench.refine_batched(cfg)
    assert len(attn) == 20 + 2                                   # backbone, then n_refine
    assert attn[0] == 4 * L * (2 * L) * H * Dh                     # W = 1: two frames
    assert attn[-1] == 4 * (4 * L * (4 * 2 * L) * H * Dh)          # r_t x (r_t (W+1) = 8 sub-frames)
    # sub-frame by sub-frame (L not a multiple of 8): r_t x n_refine launches, same total
    odd = cfg.replace(grid_h=29)
    assert not bench.refine_batched(odd) and odd.L_frm % 8 != 0
    attn_odd = bench.attn_flops_per_launch(odd)
    assert len(attn_odd) == 20 + 4 * 2
    assert sum(attn_odd[20:]) == 4 * attn_odd[-1] * 2
    assert not bench.refine_batched(C["tiny_fp32"].replace(head="paper"))   # fp32 path
    k = bench.kind_flops(cfg)
    assert k["qkv"] == 2 * L * D * (H + 2 * G) * Dh
    assert k["upsample"] == 2 * L * D * 4 * D
    assert k["final"] == 2 * L * D * 3 * 16 * 16


def test_kernels_per_frame_counts_the_graph():
    # step_begin, embed, 5 per block, final
    assert bench.kernels_per_frame(C["1080p_wan22"]) == 2 + 5 * 16 + 1 == 83
    # paper head: upsample, then 5 per refinement block + 2 spatial, once for all
    # sub-frames (bf16, L % 8 == 0) or per sub-frame
    assert bench.kernels_per_frame(C["xl_480p_wan22_paper"]) == 2 + 5 * 20 + 1 + (5 * 2 + 2)
    assert bench.kernels_per_frame(C["xl_480p_wan22_paper"].replace(grid_h=29)) == \
        2 + 5 * 20 + 1 + 4 * (5 * 2 + 2)
    assert bench.kernels_per_frame(C["xl_480p_wan22_paper"].replace(mlp_fp8=1)) == \
        2 + 6 * 20 + 1 + (6 * 2 + 2)


def test_frame_kind_flops_add_up_to_the_frame():
    for name in ("1080p_wan22", "xl_480p_wan22_paper"):
        cfg = C[name]
        total, attn = bench.flops_per_frame(cfg)
        assert sum(bench.frame_kind_flops(cfg).values()) == total - attn, name


def test_batch_scales_work_and_throughput():
    one = C["480p_wan21"]
    four = one.replace(batch=4)
    assert bench.flops_per_frame(four)[0] == 4 * bench.flops_per_frame(one)[0]
    assert bench.attn_flops_per_launch(four)[0] == 4 * bench.attn_flops_per_launch(one)[0]
    # 2 replicas x 4 streams x 10 latent frames x 4 pixel frames in 50 ms (slowest rank)
    assert bench.replica_throughput(4, 20, 50.0, batch=4) == pytest.approx(4 * 4 * 20 / 0.05)
