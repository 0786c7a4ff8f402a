"""The refinement ring's two-copy layout, checked by brute force on the CPU.

FlashDecoder paper, Sec. 3.4 Step 2: sub-frame s of the paper head attends to
sub-frames max(0, s - r_t (W+1) + 1) .. s and to nothing older. When all r_t
sub-frames of a latent frame go through a refinement block in one launch,
their keys and values are all written before any of them attends. The
library then keeps R = r_t (W+2) - 1 sub-frame slots (sub-frame s in slot
s mod R), each stored twice (rows s and s + R, in units of one sub-frame), and
sub-frame s reads the contiguous run [win, win + n_valid) with
n_valid = min(s, r_t (W+1) - 1) + 1 and win = (slot - n_valid + 1) mod R
(the frame state that step_begin writes; include/flashdec.h,
fd_debug_ring_layout).

This simulates that rule slot by slot, independent of the CUDA code, and
checks that every run holds exactly the sub-frames the paper names, that the
run stays inside the doubled ring, and that R is the smallest ring for which
writing a latent frame's sub-frames first never evicts one an earlier
sub-frame of the same frame still needs.
"""
import pytest


def _simulate(r_t, W, R, frames):
    """Returns (ok, detail): decode `frames` latent frames, writing all r_t
    sub-frames of a frame into the doubled ring before any of them reads its
    run, and compare every run with the paper's window."""
    wnd = r_t * (W + 1)
    ring = [None] * (2 * R)                     # sub-frame held by each row
    for t in range(frames):
        subs = [t * r_t + tau for tau in range(r_t)]
        for s in subs:                          # the QKV launch: both copies
            ring[s % R] = s
            ring[s % R + R] = s
        for s in subs:                          # the attention launch
            slot = s % R
            nv = min(s, wnd - 1) + 1
            win = (slot - nv + 1) % R
            if win + nv > 2 * R:
                return False, f"run of sub-frame {s} leaves the ring"
            got = sorted(ring[win:win + nv])
            want = list(range(max(0, s - wnd + 1), s + 1))
            if got != want:
                return False, f"sub-frame {s}: run holds {got}, window is {want}"
    return True, ""


@pytest.mark.parametrize("r_t", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("W", [0, 1, 2, 3])
def test_two_copy_ring_runs_hold_exactly_each_window(r_t, W):
    R = r_t * (W + 2) - 1
    ok, detail = _simulate(r_t, W, R, frames=3 * (W + 2) + 2)   # several wraps
    assert ok, detail


@pytest.mark.parametrize("r_t", [2, 3, 4, 8])
@pytest.mark.parametrize("W", [0, 1, 2])
def test_one_slot_fewer_evicts_a_needed_sub_frame(r_t, W):
    # with R - 1 slots the last sub-frame of a latent frame overwrites the
    # oldest sub-frame that its first sub-frame still attends to
    R = r_t * (W + 2) - 1
    ok, _ = _simulate(r_t, W, R - 1, frames=3 * (W + 2) + 2)
    assert not ok


def test_single_sub_frame_needs_no_extra_slot():
    # r_t = 1: R = W + 1 slots, the backbone's ring size
    for W in range(4):
        assert 1 * (W + 2) - 1 == W + 1
        assert _simulate(1, W, W + 1, frames=10)[0]
