"""The C-ABI library loads, exports every declared entry point, and its host
logic (argument and configuration validation) works without a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

import fd_synth
from streaming_transformer_video_b200 import flashdec as fdb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flashdec.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"FD_API\s+[\w\s\*]+?\b(fd_\w+)\s*\(", src)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = fdb.lib()
    names = _declared()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(fdb.EXPORTS) == names
    out = subprocess.run(["nm", "-D", "--defined-only", fdb.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r" T (fd_\w+)", out))
    assert exported == set(names)


def test_ctypes_structs_match_the_c_header(tmp_path):
    # compile a probe against the header and compare sizes and offsets
    probe = tmp_path / "probe.c"
    fields = [f[0] for f in fdb.FDConfigC._fields_]
    wfields = [f[0] for f in fdb.FDWeightsC._fields_]
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "flashdec.h"',
             'int main(void){', 'printf("%zu %zu\\n", sizeof(fd_config), sizeof(fd_weights));']
    lines += [f'printf("%zu\\n", offsetof(fd_config, {f}));' for f in fields]
    lines += [f'printf("%zu\\n", offsetof(fd_weights, {f}));' for f in wfields]
    lines += ['return 0;}']
    probe.write_text("\n".join(lines))
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(probe), "-o", str(exe)],
                   check=True)
    vals = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                           check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(fdb.FDConfigC)
    assert vals[1] == ctypes.sizeof(fdb.FDWeightsC)
    got = vals[2:]
    want = [getattr(fdb.FDConfigC, f).offset for f in fields] + \
           [getattr(fdb.FDWeightsC, f).offset for f in wfields]
    assert got == want


def test_error_strings():
    lib = fdb.lib()
    for code in range(0, -8, -1):
        s = lib.fd_error_string(code).decode()
        assert s and s != "unknown status"
    assert lib.fd_error_string(-99).decode() == "unknown status"


def _create(cfg_c):
    lib = fdb.lib()
    w = fdb.FDWeightsC()
    h = ctypes.c_void_p()
    return lib.fd_create(ctypes.byref(cfg_c), ctypes.byref(w), ctypes.byref(h)), h


def test_create_rejects_bad_configs_before_touching_the_device():
    base = fd_synth.CONFIGS["tiny_fp32"]
    lib = fdb.lib()
    h = ctypes.c_void_p(1234)
    assert lib.fd_create(None, None, ctypes.byref(h)) == fdb.FD_ERR_INVALID_ARG
    assert h.value is None
    cases = [
        (dict(patch=3), fdb.FD_ERR_UNSUPPORTED),
        (dict(grid_h=7, patch=2), fdb.FD_ERR_INVALID_ARG),
        (dict(n_heads=3, n_kv_heads=2), fdb.FD_ERR_INVALID_ARG),
        (dict(d_model=0), fdb.FD_ERR_INVALID_ARG),
        (dict(window=-1), fdb.FD_ERR_INVALID_ARG),
        (dict(px_per_token=4), fdb.FD_ERR_UNSUPPORTED),
        (dict(d_model=96), fdb.FD_ERR_UNSUPPORTED),
        (dict(head_dim=48), fdb.FD_ERR_UNSUPPORTED),
        (dict(dtype="bf16", head_dim=32), fdb.FD_ERR_UNSUPPORTED),
    ]
    for kw, code in cases:
        c = fdb.make_config(base.replace(**kw))
        s, _ = _create(c)
        assert s == code, (kw, s, lib.fd_last_error())
        assert lib.fd_last_error().decode()
    # output head fields (set on the C struct directly)
    paper = base.replace(head="paper")
    for field, value, code in [("head_mode", 2, fdb.FD_ERR_INVALID_ARG),
                               ("n_refine", 0, fdb.FD_ERR_UNSUPPORTED),
                               ("n_refine", 9, fdb.FD_ERR_UNSUPPORTED),
                               ("r_t", 17, fdb.FD_ERR_UNSUPPORTED)]:
        c = fdb.make_config(paper)
        setattr(c, field, value)
        s, _ = _create(c)
        assert s == code, (field, value, s, lib.fd_last_error())
    # FP8 MLP fields
    bf = base.replace(dtype="bf16", head_dim=64, n_heads=2, n_kv_heads=2, d_model=128)
    for cfg, field, value, code in [
            (bf, "mlp_fp8", 2, fdb.FD_ERR_INVALID_ARG),
            (bf, "record_mlp_amax", 2, fdb.FD_ERR_INVALID_ARG),
            (base, "mlp_fp8", 1, fdb.FD_ERR_UNSUPPORTED),                  # fp32 config
            (bf.replace(d_model=192, n_heads=3, n_kv_heads=3), "mlp_fp8", 1,
             fdb.FD_ERR_UNSUPPORTED)]:                                      # D % 128
        c = fdb.make_config(cfg)
        setattr(c, field, value)
        s, _ = _create(c)
        assert s == code, (field, value, s, lib.fd_last_error())
    for value in (0, 65):
        c = fdb.make_config(base)
        c.batch = value
        assert _create(c)[0] == fdb.FD_ERR_INVALID_ARG
    for value in (-1, 5):
        c = fdb.make_config(base)
        c.attn_splits = value
        assert _create(c)[0] == fdb.FD_ERR_INVALID_ARG
    for value in (-1, 3):
        c = fdb.make_config(base)
        c.attn_issuer = value
        assert _create(c)[0] == fdb.FD_ERR_INVALID_ARG
    c = fdb.make_config(bf.replace(mlp_fp8=1), record_mlp_amax=True)
    assert _create(c)[0] == fdb.FD_ERR_INVALID_ARG
    # FP8 without scale pointers: rejected before any device work
    c = fdb.make_config(bf.replace(mlp_fp8=1))
    assert _create(c)[0] == fdb.FD_ERR_INVALID_ARG
    # valid shape but null weights
    s, _ = _create(fdb.make_config(base))
    assert s == fdb.FD_ERR_INVALID_ARG


def test_bad_handle_calls():
    lib = fdb.lib()
    t = ctypes.c_int64()
    b = ctypes.c_size_t()
    assert lib.fd_reset(None, None) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_decode_frame(None, None, None, None) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_decode_frame_host(None, None, None, None) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_status(None) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_frame_index(None, ctypes.byref(t)) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_device_bytes(None, ctypes.byref(b)) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_cache_bytes(None, ctypes.byref(b)) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_debug_read_slot(None, 0, 0, 0, None) == fdb.FD_ERR_BAD_HANDLE
    n = ctypes.c_int32()
    assert lib.fd_mlp_fp8_scales(None, None, 0, ctypes.byref(n)) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_debug_block_mlp(None, 0, None, None) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_reset_stream(None, 0, None) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_stream_frame_index(None, 0, ctypes.byref(t)) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_decode_frame_static_scratch(None, None, None, None) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_debug_read_ring(None, 0, 0, 0, 0, None) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_debug_poison(None, fdb.FD_POISON_RING, None) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_debug_set_frame_index(None, 0, 5, None) == fdb.FD_ERR_BAD_HANDLE
    assert lib.fd_debug_ring_layout(None, 0, ctypes.byref(n), ctypes.byref(n)) == fdb.FD_ERR_BAD_HANDLE
    # a pointer to memory that is not a handle (magic check)
    junk = (ctypes.c_uint32 * 64)()
    assert lib.fd_reset(ctypes.cast(junk, ctypes.c_void_p), None) == fdb.FD_ERR_BAD_HANDLE
    lib.fd_destroy(None)
    lib.fd_destroy(ctypes.cast(junk, ctypes.c_void_p))


def test_make_config_marshals_every_field():
    cfg = fd_synth.CONFIGS["xl_720p_wan22_paper"].replace(mlp_fp8=1, batch=3, attn_splits=2,
                                                          attn_issuer=2)
    c = fdb.make_config(cfg, io_dtype="f32", kernel_timing=2)
    for n in ("latent_ch", "grid_h", "grid_w", "patch", "d_model", "n_heads", "n_kv_heads",
              "head_dim", "n_blocks", "mlp_ratio", "window", "out_ch", "r_t", "px_per_token",
              "kv_norm", "n_refine", "mlp_fp8", "batch", "attn_splits", "attn_issuer"):
        assert getattr(c, n) == getattr(cfg, n), n
    assert (c.dtype, c.io_dtype, c.head_mode, c.kernel_timing) == (fdb.FD_BF16, fdb.FD_F32, 1, 2)
    assert c.norm_eps == pytest.approx(cfg.norm_eps) and c.rope_theta == cfg.rope_theta
    assert c.record_mlp_amax == 0
    lin = fdb.make_config(fd_synth.CONFIGS["1080p_wan22"], record_mlp_amax=True)
    assert (lin.head_mode, lin.n_refine, lin.record_mlp_amax, lin.batch, lin.attn_splits,
            lin.attn_issuer) == (0, 0, 1, 1, 0, 0)
