"""CPU oracle for the FlashDecoder per-latent-frame streaming step.

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, obviously
correct statement of what the decoder step computes. Only the tests, the
smoke check and the benchmark's CPU-baseline leg may import it; the
product path (the CUDA library and its Python binding) never does.

Source: "FlashDecoder: Real-Time Latent-to-Pixel Streaming Decoder with
Transformers" (academ.us/article/2607.14898), cited below as [FD] with its
section and equation numbers.

Arithmetic: float64 numpy throughout. Library primitives used as steps:
numpy matmul, numpy exp, scipy.special.erf.

Readings taken where the paper is silent (each also listed in the design
notes of the repository):
  * W counts PAST frames; the cache keeps W+1 frames (current included).
  * Warm-up (t < W): attend only to the t+1 frames that exist, no padding.
  * 3D-RoPE: D_h split [D_h/4 | 3D_h/8 | 3D_h/8] for (time, row, column);
    frequencies theta^(-2m/d_part); rotation of interleaved pairs
    (2m, 2m+1); applied to queries and keys, never to values.
  * RoPE positions are relative to the current window ([FD] Sec. 4.3,
    "Long Video Decoding"): the oldest cached frame is at temporal
    position 0 and the current frame at min(t, W).
  * KV-norm: per-head RMSNorm over D_h with one learned gain vector for
    keys and one for values per block, applied before RoPE.
  * MLP: Linear D->ratio*D, exact (erf) GELU, Linear back; all Linear
    layers carry biases.
  * Output head: RMSNorm, one Linear D -> C*r_t*P^2 with channel order
    (c, tau, dy, dx), then unpatchify to [C][r_t][H_tok*P][W_tok*P].
  * FP8 MLP ([FD] Sec. 4.6, "static-calibrated FP8 quantization of all MLP
    layers"): the MLP sublayer of every Transformer block (backbone and
    refinement; not the pixel head's spatial MLP) multiplies E4M3 operands.
    Each of its two Linear layers quantizes exactly what it multiplies: its
    input activation and its weight matrix. The first Linear's input is the
    RMSNorm output a = x / rms(x) * g (gain included); the second's is the
    GELU output h. Per-tensor static scales: each weight matrix s_w =
    max|W| / 448; each activation a scale fixed by calibration (max |a| and
    max |h| over calibration frames through the unquantized decoder, / 448).
    Rounding: nearest, ties to even, saturating at +-448.

Parity pins: every function here is pinned by tests/test_oracle_pins.py
(library routines, closed forms, invariants of the method). No function
is "parity unpinned".
"""
from __future__ import annotations

import collections
from typing import Dict, List, Optional

import numpy as np
from scipy.special import erf


# --------------------------------------------------------------------------
# Elementary steps
# --------------------------------------------------------------------------

def patchify(z_t: np.ndarray, p: int) -> np.ndarray:
    """Latent frame [C'][H'][W'] -> tokens [L_frm][C' p^2].

    [FD] Sec. 3.2 "Latent Projection" (Eq. 1): a frame is flattened into
    L_frm spatial tokens in raster order. For the Wan2.1 latent space the
    frame is first PixelUnshuffled by p=2 ([FD] Sec. 4.3, "Generalization
    Across Latent Spaces"), folding each p x p block into channels in the
    order (c, dy, dx). Token n = i * (W'/p) + j.
    """
    C, Hh, Ww = z_t.shape
    Ht, Wt = Hh // p, Ww // p
    # z[c][i*p+dy][j*p+dx] -> u[i][j][c][dy][dx]
    u = z_t.reshape(C, Ht, p, Wt, p).transpose(1, 3, 0, 2, 4)
    return u.reshape(Ht * Wt, C * p * p)


def unpatchify(y: np.ndarray, out_ch: int, r_t: int, P: int, tok_h: int,
               tok_w: int) -> np.ndarray:
    """Tokens [L_frm][C r_t P^2] -> pixels [C][r_t][tok_h P][tok_w P].

    Output head of the decoder ([FD] Sec. 3.4, Step 3, depth-to-space by
    PixelShuffle): token (i, j), column ((c*r_t + tau)*P + dy)*P + dx goes to
    pixel [c][tau][i*P + dy][j*P + dx].
    """
    v = y.reshape(tok_h, tok_w, out_ch, r_t, P, P)      # [i][j][c][tau][dy][dx]
    v = v.transpose(2, 3, 0, 4, 1, 5)                    # [c][tau][i][dy][j][dx]
    return v.reshape(out_ch, r_t, tok_h * P, tok_w * P)


def linear(x: np.ndarray, w: np.ndarray, b: np.ndarray) -> np.ndarray:
    """y = x W^T + b with W in [out][in] layout."""
    return x @ w.T + b


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis with learned gain g ([FD] Sec. 3.2,
    "Base Architecture": applied before each sublayer; also the KV-norm)."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU: x * Phi(x) = x/2 (1 + erf(x/sqrt 2))."""
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


# --------------------------------------------------------------------------
# FP8 E4M3 quantization of the MLP layers ([FD] Sec. 4.6, optimization (4))
# --------------------------------------------------------------------------

E4M3_MAX = 448.0          # largest finite E4M3 value: 1.75 * 2^8


def e4m3_round(v) -> np.ndarray:
    """Nearest value of the FP8 E4M3 format: 1 sign bit, 4 exponent bits
    with bias 7, 3 fraction bits, no infinities (normal numbers
    (1 + f/8) 2^(e-7), e = 1..15, except e = 15, f = 7, which encodes NaN;
    subnormals (f/8) 2^-6). Ties go to the even neighbour; finite values and
    infinities beyond +-448 saturate to +-448; NaN stays NaN. Returns the
    rounded values as float64."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)                     # a = m 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -6)              # binade 2^e; below 2^-6 the subnormal spacing
    step = np.ldexp(1.0, e - 3)             # 3 fraction bits
    with np.errstate(invalid="ignore"):
        q = np.minimum(np.round(a / step) * step, E4M3_MAX)   # np.round: ties to even
    return np.where(np.isnan(v), np.nan, np.copysign(q, v))


def weight_scale(w: np.ndarray) -> float:
    """Static per-tensor scale of a weight matrix: fp32(max|w| / 448), or 1
    for an all-zero matrix."""
    amax = float(np.max(np.abs(w)))
    return float(np.float32(amax / E4M3_MAX)) if amax > 0 else 1.0


def quantize_weight(w: np.ndarray, s: float) -> np.ndarray:
    """Dequantized FP8 weight e4m3(w / s) s (division in float64)."""
    return e4m3_round(np.asarray(w, dtype=np.float64) / np.float64(s)) * np.float64(s)


def quantize_act(x: np.ndarray, s: float) -> np.ndarray:
    """Dequantized FP8 activation with static scale s: e4m3(x * (1/s)) s,
    where x, 1/s and their product are float32 (the precision in which the
    device takes the same rounding decision)."""
    inv = np.float32(1.0 / np.float64(s))
    v = np.asarray(x, dtype=np.float64).astype(np.float32) * inv
    return e4m3_round(v.astype(np.float64)) * np.float64(s)


def mlp(cfg, w: Dict[str, np.ndarray], p: str, x: np.ndarray,
        amax: Optional[Dict[str, float]] = None) -> np.ndarray:
    """Pre-norm MLP sublayer of block p (without the residual add):
    GELU(RMSNorm(x) W_1^T + b_1) W_2^T + b_2 ([FD] Sec. 3.2).

    With cfg.mlp_fp8 each Linear multiplies the FP8 images of its own input
    and weight ([FD] Sec. 4.6), with static per-tensor scales
    w[p + "fp8_sa"] (the normalised input a) and w[p + "fp8_sh"] (hidden h):
      a  = RMSNorm(x) (gain g included)
      h  = GELU(Q(a) Q(W_1)^T + b_1)
      y  = Q(h) Q(W_2)^T + b_2
    amax (calibration, unquantized MLP only): records the largest |a| and
    |h| of the block under keys p + "a" and p + "h"."""
    a = rms_norm(x, w[p + "norm2_g"], cfg.norm_eps)
    if not getattr(cfg, "mlp_fp8", 0):
        h = gelu(linear(a, w[p + "w1"], w[p + "b1"]))
        if amax is not None:
            amax[p + "a"] = max(amax.get(p + "a", 0.0), float(np.max(np.abs(a))))
            amax[p + "h"] = max(amax.get(p + "h", 0.0), float(np.max(np.abs(h))))
        return linear(h, w[p + "w2"], w[p + "b2"])
    w1q = quantize_weight(w[p + "w1"], weight_scale(w[p + "w1"]))
    w2q = quantize_weight(w[p + "w2"], weight_scale(w[p + "w2"]))
    h = gelu(quantize_act(a, float(w[p + "fp8_sa"])) @ w1q.T + w[p + "b1"])
    return quantize_act(h, float(w[p + "fp8_sh"])) @ w2q.T + w[p + "b2"]


def rope_split(head_dim: int):
    """Sizes of the (time, row, column) parts of one head vector."""
    d_t = head_dim // 4
    d_s = (head_dim - d_t) // 2
    return d_t, d_s, head_dim - d_t - d_s


def rope_rotate(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate interleaved pairs of x[..., d] by angle pos * theta^(-2m/d).

    x: [L][d] (d even), pos: [L]. Pair m = (x[2m], x[2m+1]) is rotated by
    angle a = pos * theta^(-2m/d):  (x0 cos a - x1 sin a, x0 sin a + x1 cos a).
    """
    d = x.shape[-1]
    m = np.arange(d // 2, dtype=np.float64)
    freq = theta ** (-2.0 * m / d)
    ang = pos.astype(np.float64)[:, None] * freq[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def rope_3d(x: np.ndarray, tau: np.ndarray, row: np.ndarray, col: np.ndarray,
            theta: float) -> np.ndarray:
    """3D-RoPE of one head's vectors x [L][D_h] ([FD] Sec. 3.2: applied
    separately to the temporal (T') and spatial (H' x W') dimensions)."""
    d_t, d_h, d_w = rope_split(x.shape[-1])
    out = np.empty_like(x)
    out[:, :d_t] = rope_rotate(x[:, :d_t], tau, theta)
    out[:, d_t:d_t + d_h] = rope_rotate(x[:, d_t:d_t + d_h], row, theta)
    out[:, d_t + d_h:] = rope_rotate(x[:, d_t + d_h:], col, theta)
    return out


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Unmasked softmax attention of one head: softmax(q k^T / sqrt(D_h)) v.

    [FD] Sec. 3.3: the current queries attend to the full cache, with no
    attention mask. q [Lq][D_h], k and v [Lk][D_h].
    """
    s = (q @ k.T) / np.sqrt(q.shape[-1])
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=-1, keepdims=True)
    return p @ v


# --------------------------------------------------------------------------
# The streaming decoder
# --------------------------------------------------------------------------

class OracleDecoder:
    """Frame-by-frame FlashDecoder forward with a rolling KV cache.

    [FD] Sec. 3.3 "Frame-by-Frame Processing": at step t the frame is
    projected (Eq. 1); new keys and values are computed, appended to the
    cache and the oldest frame evicted once the cache exceeds its capacity
    (Eq. 2); the current queries attend to the whole cache.

    The cache keeps UN-rotated keys; every step re-applies RoPE with
    window-relative temporal positions ([FD] Sec. 4.3, "Long Video
    Decoding").

    With cfg.head == "paper" the output head follows [FD] Sec. 3.4: the
    backbone output is expanded by a Linear D -> r_t D (Eq. 3) into r_t
    sub-frames; these are streamed one after another, by the same mechanism,
    through cfg.n_refine refinement blocks whose cache holds r_t (W+1)
    sub-frames; each refined sub-frame goes through RMSNorm, a 2-layer MLP
    D -> D -> C P^2 (exact GELU) and PixelShuffle by P.
    """

    def __init__(self, cfg, weights: Dict[str, np.ndarray]):
        self.cfg = cfg
        self.w = {k: np.asarray(v, dtype=np.float64) for k, v in weights.items()}
        H, G = cfg.n_heads, cfg.n_kv_heads
        assert H % G == 0
        n = np.arange(cfg.L_frm)
        self.row = (n // cfg.tok_w).astype(np.float64)   # token grid row i
        self.col = (n % cfg.tok_w).astype(np.float64)    # token grid column j
        self.amax: Optional[Dict[str, float]] = None      # set by calibrate_fp8
        self.reset()

    # -- state -------------------------------------------------------------
    def reset(self):
        """Start a new video: empty caches, frame counter 0."""
        self.t = 0
        self.cache: List[collections.deque] = [
            collections.deque() for _ in range(self.cfg.n_blocks)]
        self.rcache: List[collections.deque] = [
            collections.deque() for _ in range(self.cfg.n_refine if self.paper else 0)]

    @property
    def paper(self) -> bool:
        return getattr(self.cfg, "head", "linear") == "paper"

    def cache_bytes(self) -> int:
        """Bytes held by the rolling caches (bounded by construction)."""
        return sum(k.nbytes + v.nbytes for dq in self.cache + self.rcache for (k, v) in dq)

    # -- one block ---------------------------------------------------------
    def _block(self, p: str, dq: collections.deque, capacity: int,
               x: np.ndarray) -> np.ndarray:
        """One Transformer block (weights prefix p) for the current frame's
        tokens x; dq is the block's cache, holding at most `capacity` frames."""
        cfg, w = self.cfg, self.w
        H, G, Dh, L = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.L_frm
        # pre-attention RMSNorm and QKV projection
        a = rms_norm(x, w[p + "norm1_g"], cfg.norm_eps)
        qkv = linear(a, w[p + "wqkv"], w[p + "bqkv"])
        q = qkv[:, :H * Dh].reshape(L, H, Dh)
        k = qkv[:, H * Dh:(H + G) * Dh].reshape(L, G, Dh)
        v = qkv[:, (H + G) * Dh:].reshape(L, G, Dh)
        if cfg.kv_norm:
            k = rms_norm(k, w[p + "knorm_g"], cfg.norm_eps)
            v = rms_norm(v, w[p + "vnorm_g"], cfg.norm_eps)
        # append to the cache, evict the oldest beyond its capacity
        dq.append((k, v))
        if len(dq) > capacity:
            dq.popleft()
        n_win = len(dq)
        # window-relative temporal positions: oldest frame 0, current n_win-1
        o = np.empty((L, H, Dh))
        for h in range(H):
            g = h // (H // G)
            tau_q = np.full(L, n_win - 1, dtype=np.float64)
            qh = rope_3d(q[:, h], tau_q, self.row, self.col, cfg.rope_theta)
            ks, vs = [], []
            for f, (kf, vf) in enumerate(dq):
                tau_k = np.full(L, f, dtype=np.float64)
                ks.append(rope_3d(kf[:, g], tau_k, self.row, self.col,
                                  cfg.rope_theta))
                vs.append(vf[:, g])
            o[:, h] = attention(qh, np.concatenate(ks), np.concatenate(vs))
        x = x + linear(o.reshape(L, H * Dh), w[p + "wo"], w[p + "bo"])
        # pre-MLP RMSNorm, MLP with GELU, residual
        return x + mlp(cfg, w, p, x, self.amax)

    # -- one latent frame ----------------------------------------------------
    def embed(self, z_t: np.ndarray) -> np.ndarray:
        """Patchify + latent projection ([FD] Eq. 1)."""
        u = patchify(np.asarray(z_t, dtype=np.float64), self.cfg.patch)
        return linear(u, self.w["embed_w"], self.w["embed_b"])

    def head(self, x: np.ndarray) -> np.ndarray:
        """Linear head: final RMSNorm, Linear D -> C r_t P^2, unpatchify."""
        cfg = self.cfg
        y = linear(rms_norm(x, self.w["final_g"], cfg.norm_eps),
                   self.w["out_w"], self.w["out_b"])
        return unpatchify(y, cfg.out_ch, cfg.r_t, cfg.px_per_token,
                          cfg.tok_h, cfg.tok_w)

    def spatial(self, xs: np.ndarray) -> np.ndarray:
        """Paper head, Step 3 ([FD] Sec. 3.4): RMSNorm, MLP D -> D -> C P^2,
        PixelShuffle by P -> one pixel frame [C][tok_h P][tok_w P]."""
        cfg, w = self.cfg, self.w
        h = gelu(linear(rms_norm(xs, w["final_g"], cfg.norm_eps), w["sp1_w"], w["sp1_b"]))
        y = linear(h, w["out_w"], w["out_b"])
        return unpatchify(y, cfg.out_ch, 1, cfg.px_per_token, cfg.tok_h,
                          cfg.tok_w)[:, 0]

    def decode_frame(self, z_t: np.ndarray) -> np.ndarray:
        """One streaming step: latent frame t -> r_t pixel frames."""
        cfg = self.cfg
        x = self.embed(z_t)
        for l in range(cfg.n_blocks):
            x = self._block(f"b{l}.", self.cache[l], cfg.window + 1, x)
        self.t += 1
        if not self.paper:
            return self.head(x)
        # temporal upsampling (Eq. 3): channels [tau D, (tau+1) D) -> sub-frame tau
        up = linear(x, self.w["up_w"], self.w["up_b"])
        D = cfg.d_model
        frames = []
        for tau in range(cfg.r_t):
            xs = up[:, tau * D:(tau + 1) * D]
            for l in range(cfg.n_refine):
                xs = self._block(f"r{l}.", self.rcache[l], cfg.r_t * (cfg.window + 1), xs)
            frames.append(self.spatial(xs))
        return np.stack(frames, axis=1)                  # [C][r_t][H][W]

    def window_frames(self, l: int):
        """Frame indices currently held by block l's cache, oldest first."""
        n = len(self.cache[l])
        return list(range(self.t - n, self.t))

    def cached_kv(self, l: int, frame: int):
        """Un-rotated (k, v) [L_frm][G][D_h] of `frame` in block l's cache."""
        frames = self.window_frames(l)
        return self.cache[l][frames.index(frame)]

    def refine_window(self, l: int):
        """Paper head: sub-frame indices t r_t + tau held by refinement block
        l's cache, oldest first."""
        n = len(self.rcache[l])
        end = self.t * self.cfg.r_t
        return list(range(end - n, end))

    def refine_cached_kv(self, l: int, sub: int):
        """Un-rotated (k, v) [L_frm][G][D_h] of sub-frame `sub` in refinement
        block l's cache."""
        return self.rcache[l][self.refine_window(l).index(sub)]


def calibrate_fp8(cfg, weights, z: np.ndarray) -> Dict[str, float]:
    """Static FP8 scales of every MLP layer ([FD] Sec. 4.6: static
    calibration): stream the calibration frames z[0..T-1] through the decoder
    with unquantized MLPs, take per block the largest |a| entering the first
    MLP Linear (the RMSNorm output) and the largest |GELU output|, and set each
    scale to fp32(amax / 448), so the calibration data never saturates.
    Returns {"b{l}.fp8_sa": s, "b{l}.fp8_sh": s, ...}, with "r{l}.*" for the
    paper head's refinement blocks."""
    dec = OracleDecoder(cfg.replace(mlp_fp8=0), weights)
    dec.amax = {}
    for t in range(z.shape[0]):
        dec.decode_frame(z[t])
    out = {}
    for key, a in dec.amax.items():
        p, kind = key[:-1], key[-1]
        out[p + "fp8_s" + kind] = float(np.float32(a / E4M3_MAX)) if a > 0 else 1.0
    return out


def decode_video(cfg, weights, z: np.ndarray,
                 frames: Optional[int] = None) -> np.ndarray:
    """Stream frames z[0..T'-1] through a fresh decoder; stack the outputs
    to [T'][C][r_t][H][W]."""
    dec = OracleDecoder(cfg, weights)
    T = z.shape[0] if frames is None else frames
    return np.stack([dec.decode_frame(z[t]) for t in range(T)])


# --------------------------------------------------------------------------
# Full-sequence forward with a brute-force block-windowed mask
# --------------------------------------------------------------------------

def _masked_block(cfg, w, p, x, tau, row, col, allowed):
    """One block over a whole token sequence with a boolean attention mask
    (allowed[a, b]: query token a may see key token b); absolute positions."""
    H, G, Dh = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    S = x.shape[0]
    a = rms_norm(x, w[p + "norm1_g"], cfg.norm_eps)
    qkv = linear(a, w[p + "wqkv"], w[p + "bqkv"])
    q = qkv[:, :H * Dh].reshape(S, H, Dh)
    k = qkv[:, H * Dh:(H + G) * Dh].reshape(S, G, Dh)
    v = qkv[:, (H + G) * Dh:].reshape(S, G, Dh)
    if cfg.kv_norm:
        k = rms_norm(k, w[p + "knorm_g"], cfg.norm_eps)
        v = rms_norm(v, w[p + "vnorm_g"], cfg.norm_eps)
    o = np.empty((S, H, Dh))
    for h in range(H):
        g = h // (H // G)
        qh = rope_3d(q[:, h], tau, row, col, cfg.rope_theta)
        kh = rope_3d(k[:, g], tau, row, col, cfg.rope_theta)
        sc = (qh @ kh.T) / np.sqrt(Dh)
        sc = np.where(allowed, sc, -np.inf)
        sc = sc - sc.max(axis=-1, keepdims=True)
        pr = np.exp(sc)
        pr = pr / pr.sum(axis=-1, keepdims=True)
        o[:, h] = pr @ v[:, g]
    x = x + linear(o.reshape(S, H * Dh), w[p + "wo"], w[p + "bo"])
    return x + mlp(cfg, w, p, x)


def _window_mask(frame_of, span):
    """allowed[a, b] = frame_of[b] in [frame_of[a] - span + 1, frame_of[a]]."""
    S = frame_of.shape[0]
    allowed = np.zeros((S, S), dtype=bool)
    for a in range(S):
        for b in range(S):
            allowed[a, b] = (frame_of[a] - span + 1 <= frame_of[b] <= frame_of[a])
    return allowed


def full_sequence(cfg, weights: Dict[str, np.ndarray],
                  z: np.ndarray) -> np.ndarray:
    """One forward over all T' L_frm tokens at once.

    This is the conventional formulation the paper contrasts with
    streaming ([FD] Sec. 3.3, "Training-Inference Consistency"): the whole
    sequence goes through one pass and a materialised mask restricts each
    query of frame t to key frames t-W .. t (the sliding-window pattern of
    [FD] Sec. 3.3, "Attention Pattern"). RoPE uses ABSOLUTE frame indices.
    With the paper head, the r_t T' sub-frames go through the refinement
    blocks the same way (sub-frame s sees sub-frames s - r_t (W+1) + 1 .. s).
    Only for tiny inputs: the masks are [T' L][T' L] and [r_t T' L]^2.
    """
    w = {k: np.asarray(v, dtype=np.float64) for k, v in weights.items()}
    T = z.shape[0]
    D, L = cfg.d_model, cfg.L_frm
    frame_of = np.repeat(np.arange(T), L)                 # frame of each token
    n = np.tile(np.arange(L), T)
    row = (n // cfg.tok_w).astype(np.float64)
    col = (n % cfg.tok_w).astype(np.float64)
    allowed = _window_mask(frame_of, cfg.window + 1)

    x = np.concatenate([linear(patchify(z[t].astype(np.float64), cfg.patch),
                               w["embed_w"], w["embed_b"]) for t in range(T)])
    for l in range(cfg.n_blocks):
        x = _masked_block(cfg, w, f"b{l}.", x, frame_of.astype(np.float64), row, col, allowed)
    if getattr(cfg, "head", "linear") != "paper":
        y = linear(rms_norm(x, w["final_g"], cfg.norm_eps), w["out_w"], w["out_b"])
        return np.stack([unpatchify(y[t * L:(t + 1) * L], cfg.out_ch, cfg.r_t,
                                    cfg.px_per_token, cfg.tok_h, cfg.tok_w)
                         for t in range(T)])
    # paper head: sub-frame s = t r_t + tau takes channels [tau D, (tau+1) D)
    up = linear(x, w["up_w"], w["up_b"]).reshape(T, L, cfg.r_t, D)
    xs = up.transpose(0, 2, 1, 3).reshape(T * cfg.r_t * L, D)
    sub_of = np.repeat(np.arange(T * cfg.r_t), L)
    n = np.tile(np.arange(L), T * cfg.r_t)
    row = (n // cfg.tok_w).astype(np.float64)
    col = (n % cfg.tok_w).astype(np.float64)
    allowed = _window_mask(sub_of, cfg.r_t * (cfg.window + 1))
    for l in range(cfg.n_refine):
        xs = _masked_block(cfg, w, f"r{l}.", xs, sub_of.astype(np.float64), row, col, allowed)
    h = gelu(linear(rms_norm(xs, w["final_g"], cfg.norm_eps), w["sp1_w"], w["sp1_b"]))
    y = linear(h, w["out_w"], w["out_b"])
    out = np.empty((T,) + tuple(cfg.out_shape))
    for s in range(T * cfg.r_t):
        t, tau = divmod(s, cfg.r_t)
        out[t, :, tau] = unpatchify(y[s * L:(s + 1) * L], cfg.out_ch, 1, cfg.px_per_token,
                                    cfg.tok_h, cfg.tok_w)[:, 0]
    return out
