"""ctypes binding of libflashdec.so (include/flashdec.h).

Argument marshalling only: every step of the decoder runs in the library's
CUDA kernels. PyTorch is used by callers for device memory and streams; this
module takes raw pointers (tensor.data_ptr()) and CUDA stream handles.
If the shared library is missing the import fails loudly: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# FLASHDEC_LIB=debug selects the bounds-checked build (libflashdec_debug.so,
# same ABI; out-of-range device accesses are skipped and reported as
# FD_ERR_BOUNDS by fd_status)
LIB_PATH = os.path.join(_HERE, "libflashdec_debug.so" if os.environ.get("FLASHDEC_LIB") == "debug"
                        else "libflashdec.so")

FD_OK, FD_ERR_INVALID_ARG, FD_ERR_UNSUPPORTED, FD_ERR_OOM = 0, -1, -2, -3
FD_ERR_CUDA, FD_ERR_TIMEOUT, FD_ERR_BAD_HANDLE, FD_ERR_BOUNDS = -4, -5, -6, -7
FD_POISON_RING, FD_POISON_SPLIT_COUNTERS = 1, 2
FD_F32, FD_BF16 = 0, 1
KERNEL_KINDS = ["step_begin", "embed", "qkv", "attn", "oproj", "mlp_up", "mlp_down", "final",
                "upsample", "spatial", "mlp_norm"]
HEAD_MODES = {"linear": 0, "paper": 1}

EXPORTS = ["fd_create", "fd_reset", "fd_decode_frame", "fd_decode_frame_host", "fd_destroy",
           "fd_status", "fd_error_string", "fd_last_error", "fd_frame_index", "fd_device_bytes",
           "fd_cache_bytes", "fd_debug_read_slot", "fd_last_step_kernel_ms",
           "fd_selftest_wait_timeout", "fd_mlp_fp8_scales", "fd_debug_block_mlp",
           "fd_reset_stream", "fd_stream_frame_index", "fd_decode_frame_static_scratch",
           "fd_debug_read_ring", "fd_debug_poison", "fd_debug_set_frame_index",
           "fd_debug_ring_layout"]


class FDConfigC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "latent_ch", "grid_h", "grid_w", "patch", "d_model", "n_heads", "n_kv_heads",
        "head_dim", "n_blocks", "mlp_ratio", "window", "out_ch", "r_t", "px_per_token",
        "kv_norm", "dtype", "io_dtype")] + [
        ("norm_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
        ("kernel_timing", ctypes.c_int32), ("head_mode", ctypes.c_int32),
        ("n_refine", ctypes.c_int32), ("mlp_fp8", ctypes.c_int32),
        ("record_mlp_amax", ctypes.c_int32), ("batch", ctypes.c_int32),
        ("attn_splits", ctypes.c_int32), ("attn_issuer", ctypes.c_int32)]


_PF = ctypes.POINTER(ctypes.c_float)
_PPF = ctypes.POINTER(_PF)


class FDWeightsC(ctypes.Structure):
    _fields_ = [("embed_w", _PF), ("embed_b", _PF),
                ("norm1_g", _PPF), ("wqkv", _PPF), ("bqkv", _PPF),
                ("knorm_g", _PPF), ("vnorm_g", _PPF),
                ("wo", _PPF), ("bo", _PPF), ("norm2_g", _PPF),
                ("w1", _PPF), ("b1", _PPF), ("w2", _PPF), ("b2", _PPF),
                ("final_g", _PF), ("out_w", _PF), ("out_b", _PF),
                ("up_w", _PF), ("up_b", _PF), ("sp1_w", _PF), ("sp1_b", _PF),
                ("mlp_scales", _PPF)]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} not found at {path}; build it with "
                          "`python -m streaming_transformer_video_b200.csrc.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.fd_create.argtypes = [ctypes.POINTER(FDConfigC), ctypes.POINTER(FDWeightsC),
                              ctypes.POINTER(vp)]
    lib.fd_reset.argtypes = [vp, vp]
    lib.fd_decode_frame.argtypes = [vp, vp, vp, vp]
    lib.fd_decode_frame_host.argtypes = [vp, vp, vp, vp]
    lib.fd_destroy.argtypes = [vp]
    lib.fd_destroy.restype = None
    lib.fd_status.argtypes = [vp]
    lib.fd_error_string.argtypes = [i32]
    lib.fd_error_string.restype = ctypes.c_char_p
    lib.fd_last_error.argtypes = []
    lib.fd_last_error.restype = ctypes.c_char_p
    lib.fd_frame_index.argtypes = [vp, ctypes.POINTER(i64)]
    lib.fd_device_bytes.argtypes = [vp, ctypes.POINTER(sz)]
    lib.fd_cache_bytes.argtypes = [vp, ctypes.POINTER(sz)]
    lib.fd_debug_read_slot.argtypes = [vp, i32, i32, i32, _PF]
    lib.fd_last_step_kernel_ms.argtypes = [vp, _PF, ctypes.POINTER(i32), i32,
                                           ctypes.POINTER(i32)]
    lib.fd_selftest_wait_timeout.argtypes = [i32]
    lib.fd_mlp_fp8_scales.argtypes = [vp, _PF, i32, ctypes.POINTER(i32)]
    lib.fd_debug_block_mlp.argtypes = [vp, i32, _PF, _PF]
    lib.fd_reset_stream.argtypes = [vp, i32, vp]
    lib.fd_decode_frame_static_scratch.argtypes = [vp, vp, vp, vp]
    lib.fd_stream_frame_index.argtypes = [vp, i32, ctypes.POINTER(i64)]
    lib.fd_debug_read_ring.argtypes = [vp, i32, i32, i32, i32, _PF]
    lib.fd_debug_poison.argtypes = [vp, i32, vp]
    lib.fd_debug_set_frame_index.argtypes = [vp, i32, i64, vp]
    lib.fd_debug_ring_layout.argtypes = [vp, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
    for name in EXPORTS:
        if name not in ("fd_destroy", "fd_error_string", "fd_last_error"):
            getattr(lib, name).restype = i32
    return lib


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


class FDError(RuntimeError):
    def __init__(self, code: int, where: str):
        L = lib()
        msg = L.fd_last_error().decode() or L.fd_error_string(code).decode()
        super().__init__(f"{where}: {L.fd_error_string(code).decode()} ({code}): {msg}")
        self.code = code


def _check(code: int, where: str):
    if code != FD_OK:
        raise FDError(code, where)


def _dtype_code(s) -> int:
    if s in ("bf16", FD_BF16):
        return FD_BF16
    if s in ("f32", "fp32", FD_F32):
        return FD_F32
    raise ValueError(f"unknown dtype {s!r}")


def selftest_wait_timeout(timeout_us: int) -> int:
    """Run the device-side bounded-wait self-test; returns the fd status code
    (FD_ERR_TIMEOUT when the wait gave up as designed)."""
    return int(lib().fd_selftest_wait_timeout(int(timeout_us)))


def make_config(cfg, io_dtype=None, kernel_timing: bool = False,
                record_mlp_amax: bool = False) -> FDConfigC:
    """fd_config from any object with the decoder's shape attributes."""
    c = FDConfigC()
    for n in ("latent_ch", "grid_h", "grid_w", "patch", "d_model", "n_heads", "n_kv_heads",
              "head_dim", "n_blocks", "mlp_ratio", "window", "out_ch", "r_t", "px_per_token",
              "kv_norm"):
        setattr(c, n, int(getattr(cfg, n)))
    c.dtype = _dtype_code(cfg.dtype)
    c.io_dtype = _dtype_code(io_dtype if io_dtype is not None else cfg.dtype)
    c.norm_eps = float(getattr(cfg, "norm_eps", 1e-6))
    c.rope_theta = float(getattr(cfg, "rope_theta", 1e4))
    # False/0: off; True/1: every kernel; 2: attention launches only
    c.kernel_timing = int(kernel_timing)
    c.head_mode = HEAD_MODES[getattr(cfg, "head", "linear")]
    c.n_refine = int(getattr(cfg, "n_refine", 0)) if c.head_mode else 0
    c.mlp_fp8 = int(getattr(cfg, "mlp_fp8", 0))
    c.record_mlp_amax = int(record_mlp_amax)
    c.batch = int(getattr(cfg, "batch", 1))
    c.attn_splits = int(getattr(cfg, "attn_splits", 0))
    c.attn_issuer = int(getattr(cfg, "attn_issuer", 0))
    return c


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if hasattr(stream, "cuda_stream"):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


class FlashDecoder:
    """One streaming decoder (one video at a time) on the current CUDA device.

    weights: dict name -> float32 array in PyTorch Linear layout, names
    "embed_w", "embed_b", "b{l}.norm1_g", "b{l}.wqkv", "b{l}.bqkv",
    "b{l}.knorm_g", "b{l}.vnorm_g", "b{l}.wo", "b{l}.bo", "b{l}.norm2_g",
    "b{l}.w1", "b{l}.b1", "b{l}.w2", "b{l}.b2", "final_g", "out_w", "out_b".
    With cfg.head == "paper" also "up_w", "up_b", "sp1_w", "sp1_b" and the
    refinement blocks "r{l}.*" (same keys as "b{l}.*"), l < cfg.n_refine.
    With cfg.mlp_fp8 also the static FP8 scales "b{l}.fp8_sa", "b{l}.fp8_sh"
    (and "r{l}.*") of every block, e.g. from mlp_fp8_scales() of a handle
    created with record_mlp_amax=True.
    """

    def __init__(self, cfg, weights: Dict[str, np.ndarray], io_dtype=None,
                 kernel_timing: bool = False, record_mlp_amax: bool = False):
        self._lib = lib()
        self.cfg = cfg
        self.c = make_config(cfg, io_dtype, kernel_timing, record_mlp_amax)
        self._prefixes = [f"b{l}." for l in range(cfg.n_blocks)]
        if self.c.head_mode:
            self._prefixes += [f"r{l}." for l in range(cfg.n_refine)]
        keep: List[np.ndarray] = []

        def fp(name):
            a = np.ascontiguousarray(np.asarray(weights[name], dtype=np.float32))
            keep.append(a)
            return a.ctypes.data_as(_PF)

        prefixes = self._prefixes

        def per_block(key):
            arr = (_PF * len(prefixes))(*[fp(p + key) for p in prefixes])
            keep.append(arr)
            return ctypes.cast(arr, _PPF)

        w = FDWeightsC()
        w.embed_w, w.embed_b = fp("embed_w"), fp("embed_b")
        for key in ("norm1_g", "wqkv", "bqkv", "knorm_g", "vnorm_g", "wo", "bo", "norm2_g",
                    "w1", "b1", "w2", "b2"):
            setattr(w, key, per_block(key))
        w.final_g, w.out_w, w.out_b = fp("final_g"), fp("out_w"), fp("out_b")
        if self.c.head_mode:
            w.up_w, w.up_b, w.sp1_w, w.sp1_b = (fp("up_w"), fp("up_b"), fp("sp1_w"),
                                                fp("sp1_b"))
        if self.c.mlp_fp8:
            pairs = []
            for p in prefixes:
                a = np.array([weights[p + "fp8_sa"], weights[p + "fp8_sh"]], dtype=np.float32)
                keep.append(a)
                pairs.append(a.ctypes.data_as(_PF))
            arr = (_PF * len(pairs))(*pairs)
            keep.append(arr)
            w.mlp_scales = ctypes.cast(arr, _PPF)
        h = ctypes.c_void_p()
        _check(self._lib.fd_create(ctypes.byref(self.c), ctypes.byref(w), ctypes.byref(h)),
               "fd_create")
        self.h = h
        del keep

    # ------------------------------------------------------------------
    def close(self):
        if getattr(self, "h", None):
            self._lib.fd_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # ------------------------------------------------------------------
    def reset(self, stream=None):
        _check(self._lib.fd_reset(self.h, _stream_handle(stream)), "fd_reset")

    def reset_stream(self, b: int, stream=None):
        """Start a new video in stream b only."""
        _check(self._lib.fd_reset_stream(self.h, int(b), _stream_handle(stream)),
               "fd_reset_stream")

    def decode_frame(self, latent, out, stream=None):
        """latent [B][C'][H'][W'], out [B][C][r_t][H][W] (B = cfg.batch; the
        leading axis may be omitted for B = 1): CUDA tensors or raw device
        pointers as int."""
        lp = latent.data_ptr() if hasattr(latent, "data_ptr") else int(latent)
        op = out.data_ptr() if hasattr(out, "data_ptr") else int(out)
        _check(self._lib.fd_decode_frame(self.h, ctypes.c_void_p(lp), ctypes.c_void_p(op),
                                         _stream_handle(stream)), "fd_decode_frame")

    def decode_frame_static_scratch(self, latent, out, stream=None):
        """decode_frame whose attention scratch is the library's fixed device
        array (no allocation; calls must not overlap in time)."""
        lp = latent.data_ptr() if hasattr(latent, "data_ptr") else int(latent)
        op = out.data_ptr() if hasattr(out, "data_ptr") else int(out)
        _check(self._lib.fd_decode_frame_static_scratch(self.h, ctypes.c_void_p(lp),
                                                        ctypes.c_void_p(op),
                                                        _stream_handle(stream)),
               "fd_decode_frame_static_scratch")

    def decode_frame_host(self, latent, out, stream=None):
        """latent, out: host buffers (pinned tensors or numpy arrays)."""
        lp = latent.data_ptr() if hasattr(latent, "data_ptr") else latent.ctypes.data
        op = out.data_ptr() if hasattr(out, "data_ptr") else out.ctypes.data
        _check(self._lib.fd_decode_frame_host(self.h, ctypes.c_void_p(lp), ctypes.c_void_p(op),
                                              _stream_handle(stream)), "fd_decode_frame_host")

    def status(self) -> int:
        return int(self._lib.fd_status(self.h))

    def frame_index(self, b: int = 0) -> int:
        t = ctypes.c_int64()
        _check(self._lib.fd_stream_frame_index(self.h, int(b), ctypes.byref(t)),
               "fd_stream_frame_index")
        return t.value

    def device_bytes(self) -> int:
        b = ctypes.c_size_t()
        _check(self._lib.fd_device_bytes(self.h, ctypes.byref(b)), "fd_device_bytes")
        return b.value

    def cache_bytes(self) -> int:
        b = ctypes.c_size_t()
        _check(self._lib.fd_cache_bytes(self.h, ctypes.byref(b)), "fd_cache_bytes")
        return b.value

    def read_slot(self, block: int, slot: int, kv: int) -> np.ndarray:
        """Ring slot contents as float32 [G][L_frm][D_h] (kv 0 = keys, 1 = values)."""
        cfg = self.cfg
        L = (cfg.grid_h // cfg.patch) * (cfg.grid_w // cfg.patch)
        out = np.empty((cfg.n_kv_heads, L, cfg.head_dim), dtype=np.float32)
        _check(self._lib.fd_debug_read_slot(self.h, block, slot, kv, out.ctypes.data_as(_PF)),
               "fd_debug_read_slot")
        return out

    def read_ring(self, block: int, b: int, slot: int, kv: int) -> np.ndarray:
        """Ring slot of any block (refinement blocks follow the backbone's) and
        stream b, as float32 [G][L_frm][D_h] (kv 0 = keys, 1 = values)."""
        cfg = self.cfg
        L = (cfg.grid_h // cfg.patch) * (cfg.grid_w // cfg.patch)
        out = np.empty((cfg.n_kv_heads, L, cfg.head_dim), dtype=np.float32)
        _check(self._lib.fd_debug_read_ring(self.h, block, b, slot, kv, out.ctypes.data_as(_PF)),
               "fd_debug_read_ring")
        return out

    def ring_layout(self, block: int):
        """(slots, copies) of a block's ring: frame f in slot f mod slots, and
        with copies == 2 also in slot f mod slots + slots."""
        n, c = ctypes.c_int32(0), ctypes.c_int32(0)
        _check(self._lib.fd_debug_ring_layout(self.h, block, ctypes.byref(n), ctypes.byref(c)),
               "fd_debug_ring_layout")
        return n.value, c.value

    def debug_poison(self, what: int, stream=None):
        """Fill the ring caches with NaN (FD_POISON_RING) and/or the split
        counters with garbage (FD_POISON_SPLIT_COUNTERS)."""
        _check(self._lib.fd_debug_poison(self.h, int(what), _stream_handle(stream)),
               "fd_debug_poison")

    def debug_set_frame_index(self, t: int, b: int = 0, stream=None):
        """Treat the next frame of stream b as frame t (tests of long videos)."""
        _check(self._lib.fd_debug_set_frame_index(self.h, int(b), int(t), _stream_handle(stream)),
               "fd_debug_set_frame_index")

    def debug_block_mlp(self, block: int, x: np.ndarray) -> np.ndarray:
        """x + b_o + MLP(x + b_o) of block `block` for a residual stream x
        [L_frm][D] (float32), through the block's own kernels."""
        x = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty_like(x)
        _check(self._lib.fd_debug_block_mlp(self.h, block, x.ctypes.data_as(_PF),
                                            out.ctypes.data_as(_PF)), "fd_debug_block_mlp")
        return out

    def mlp_fp8_scales(self) -> Dict[str, float]:
        """Static FP8 scales {"b{l}.fp8_sa": .., "b{l}.fp8_sh": .., ...} from
        the MLP ranges recorded since the last reset (record_mlp_amax=True)."""
        n = ctypes.c_int32()
        _check(self._lib.fd_mlp_fp8_scales(self.h, None, 0, ctypes.byref(n)), "fd_mlp_fp8_scales")
        out = (ctypes.c_float * n.value)()
        _check(self._lib.fd_mlp_fp8_scales(self.h, out, n.value, ctypes.byref(n)),
               "fd_mlp_fp8_scales")
        res = {}
        for i, p in enumerate(self._prefixes):
            res[p + "fp8_sa"], res[p + "fp8_sh"] = float(out[2 * i]), float(out[2 * i + 1])
        return res

    def kernel_ms(self) -> List[Tuple[str, float]]:
        """(kind, ms) of every timed kernel of the last frame (kernel_timing 1 or 2)."""
        n = ctypes.c_int32()
        _check(self._lib.fd_last_step_kernel_ms(self.h, None, None, 0, ctypes.byref(n)),
               "fd_last_step_kernel_ms")
        ms = (ctypes.c_float * n.value)()
        kinds = (ctypes.c_int32 * n.value)()
        _check(self._lib.fd_last_step_kernel_ms(self.h, ms, kinds, n.value, ctypes.byref(n)),
               "fd_last_step_kernel_ms")
        return [(KERNEL_KINDS[kinds[i]], float(ms[i])) for i in range(n.value)]
