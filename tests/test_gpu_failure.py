"""Device-side failure detection, exercised without faulting the GPU.

Every wait in the decoder's kernels is bounded; on expiry the kernel records
FD_ERR_TIMEOUT and returns. Here a wait on a barrier that nothing completes is
made to run out (50 ms) and the status is read back; the context must remain
usable, so a full decode afterwards still matches the oracle.
"""
import time

import pytest

import fd_synth
from gpu_util import assert_close, gpu_decode, oracle_decode
from streaming_transformer_video_b200 import flashdec as fdb

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_bounded_wait_reports_timeout_and_context_survives():
    t0 = time.time()
    assert fdb.selftest_wait_timeout(50_000) == fdb.FD_ERR_TIMEOUT
    assert time.time() - t0 < 30
    assert "gave up" in fdb.lib().fd_last_error().decode()
    # the context still decodes correctly
    cfg = fd_synth.CONFIGS["tiny_fp32"]
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg)
    assert_close(cfg, gpu_decode(cfg, w, z), oracle_decode(cfg, w, z))


def test_selftest_rejects_bad_limits():
    assert fdb.selftest_wait_timeout(0) == fdb.FD_ERR_INVALID_ARG
    assert fdb.selftest_wait_timeout(10**8) == fdb.FD_ERR_INVALID_ARG
