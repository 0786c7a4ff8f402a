"""Pins of the CPU oracle to things other than itself.

Each test ties one oracle function to a library routine with its own
documented semantics, a closed form, or an invariant that the FlashDecoder
paper (academ.us/article/2607.14898, [FD]) states for the method. The
pages print no worked numeric example, so absolute pixel values cannot be
pinned to the paper; what is pinned is every step's definition.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import fd_synth
import oracle
from oracle import flashdec_oracle as fo

TINY = fd_synth.CONFIGS["tiny_fp32"]


def _rng(seed=0):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# Elementary steps against library routines
# --------------------------------------------------------------------------

@pytest.mark.parametrize("p", [1, 2])
def test_patchify_is_pixel_unshuffle_in_raster_order(p):
    # [FD] Eq. 1 (raster flatten) and Sec. 4.3 (PixelUnshuffle by 2).
    z = _rng(1).standard_normal((5, 6 * p, 7 * p))
    u = fo.patchify(z, p)
    ref = F.pixel_unshuffle(torch.from_numpy(z)[None], p)[0]   # [C p^2][6][7]
    ref = ref.reshape(5 * p * p, 42).T.numpy()                 # token = i*7+j
    assert u.shape == (42, 5 * p * p)
    np.testing.assert_array_equal(u, ref)
    # spot check of the raster index: token (i=2, j=3), channel (c=4,dy,dx)
    i, j, c = 2, 3, 4
    for dy in range(p):
        for dx in range(p):
            assert u[i * 7 + j, c * p * p + dy * p + dx] == z[c, i * p + dy, j * p + dx]


def test_unpatchify_is_pixel_shuffle():
    C, rt, P, th, tw = 3, 4, 4, 5, 7
    y = _rng(2).standard_normal((th * tw, C * rt * P * P))
    out = fo.unpatchify(y, C, rt, P, th, tw)
    ref = torch.from_numpy(y.T.reshape(C * rt * P * P, th, tw))
    ref = F.pixel_shuffle(ref[None], P)[0].reshape(C, rt, th * P, tw * P).numpy()
    np.testing.assert_array_equal(out, ref)
    # spot check: token (1, 2), c=2, tau=3, dy=1, dx=3
    i, j, c, tau, dy, dx = 1, 2, 2, 3, 1, 3
    col = ((c * rt + tau) * P + dy) * P + dx
    assert out[c, tau, i * P + dy, j * P + dx] == y[i * tw + j, col]


def test_linear_matches_torch():
    x = _rng(3).standard_normal((9, 6))
    w = _rng(4).standard_normal((5, 6))
    b = _rng(5).standard_normal(5)
    ref = F.linear(torch.from_numpy(x), torch.from_numpy(w), torch.from_numpy(b))
    np.testing.assert_allclose(fo.linear(x, w, b), ref.numpy(), rtol=1e-13, atol=1e-13)


def test_rms_norm_matches_torch():
    x = _rng(6).standard_normal((4, 3, 32)) * 3.0
    g = 1 + 0.1 * _rng(7).standard_normal(32)
    ref = F.rms_norm(torch.from_numpy(x), (32,), torch.from_numpy(g), eps=1e-6)
    np.testing.assert_allclose(fo.rms_norm(x, g, 1e-6), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_gelu_matches_torch_exact_gelu():
    x = np.linspace(-8, 8, 1001)
    ref = F.gelu(torch.from_numpy(x), approximate="none").numpy()
    np.testing.assert_allclose(fo.gelu(x), ref, rtol=1e-12, atol=1e-14)
    # closed-form identity of x*Phi(x): gelu(x) - gelu(-x) = x
    np.testing.assert_allclose(fo.gelu(x) - fo.gelu(-x), x, atol=1e-12)


def test_attention_matches_sdpa():
    q = _rng(8).standard_normal((13, 32))
    k = _rng(9).standard_normal((40, 32))
    v = _rng(10).standard_normal((40, 32))
    ref = F.scaled_dot_product_attention(torch.from_numpy(q)[None], torch.from_numpy(k)[None],
                                         torch.from_numpy(v)[None])[0].numpy()
    np.testing.assert_allclose(fo.attention(q, k, v), ref, rtol=1e-11, atol=1e-12)


def test_attention_closed_forms():
    k = _rng(11).standard_normal((40, 16))
    v = _rng(12).standard_normal((40, 16))
    # zero query: uniform softmax, output = mean of v
    np.testing.assert_allclose(fo.attention(np.zeros((3, 16)), k, v),
                               np.repeat(v.mean(0, keepdims=True), 3, 0), atol=1e-13)
    # single key: output = that value
    np.testing.assert_allclose(fo.attention(_rng(13).standard_normal((3, 16)), k[:1], v[:1]),
                               np.repeat(v[:1], 3, 0), atol=1e-13)


# --------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------

def test_rope_split_sizes():
    assert fo.rope_split(64) == (16, 24, 24)
    assert fo.rope_split(32) == (8, 12, 12)


def test_rope_rotate_is_complex_multiplication():
    d, theta = 24, 10000.0
    x = _rng(14).standard_normal((11, d))
    pos = _rng(15).integers(0, 200, 11).astype(np.float64)
    out = fo.rope_rotate(x, pos, theta)
    zc = x[:, 0::2] + 1j * x[:, 1::2]
    freq = np.array([theta ** (-2.0 * m / d) for m in range(d // 2)])
    ref = zc * np.exp(1j * pos[:, None] * freq[None, :])
    np.testing.assert_allclose(out[:, 0::2], ref.real, atol=1e-12)
    np.testing.assert_allclose(out[:, 1::2], ref.imag, atol=1e-12)


def test_rope_angle_readback():
    # unit vector in pair m, position 1: the rotation angle is theta^(-2m/d)
    d, theta = 16, 10000.0
    for m in range(d // 2):
        e = np.zeros((1, d))
        e[0, 2 * m] = 1.0
        r = fo.rope_rotate(e, np.array([1.0]), theta)
        ang = math.atan2(r[0, 2 * m + 1], r[0, 2 * m])
        assert abs(ang - theta ** (-2.0 * m / d)) < 1e-14
        assert np.count_nonzero(np.abs(r) > 1e-15) <= 2   # stays inside its pair


def test_rope_identity_norm_and_relativity():
    x = _rng(16).standard_normal((5, 64))
    z = np.zeros(5)
    np.testing.assert_array_equal(fo.rope_3d(x, z, z, z, 1e4), x)
    tau, row, col = (_rng(s).integers(0, 50, 5).astype(float) for s in (17, 18, 19))
    r = fo.rope_3d(x, tau, row, col, 1e4)
    np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    # scores depend only on position differences: shift every position by 7
    q, k = x[:1], _rng(20).standard_normal((1, 64))
    a = fo.rope_3d(q, tau[:1], row[:1], col[:1], 1e4) @ fo.rope_3d(k, tau[1:2], row[1:2], col[1:2], 1e4).T
    b = fo.rope_3d(q, tau[:1] + 7, row[:1] + 7, col[:1] + 7, 1e4) @ \
        fo.rope_3d(k, tau[1:2] + 7, row[1:2] + 7, col[1:2] + 7, 1e4).T
    np.testing.assert_allclose(a, b, rtol=1e-11)


def test_rope_3d_parts_follow_their_own_axis():
    # a vector living only in the temporal part ignores row/column positions,
    # one living only in the row part ignores time and column, and so on
    d_t, d_h, d_w = fo.rope_split(64)
    x = _rng(21).standard_normal((1, 64))
    for lo, hi, axis in ((0, d_t, 0), (d_t, d_t + d_h, 1), (d_t + d_h, 64, 2)):
        v = np.zeros_like(x)
        v[:, lo:hi] = x[:, lo:hi]
        pos = [np.array([3.0]), np.array([5.0]), np.array([11.0])]
        base = fo.rope_3d(v, *pos, 1e4)
        for other in range(3):
            if other == axis:
                continue
            moved = [p.copy() for p in pos]
            moved[other] += 4.0
            np.testing.assert_array_equal(fo.rope_3d(v, *moved, 1e4), base)


# --------------------------------------------------------------------------
# The whole step against a composition of torch library routines
# --------------------------------------------------------------------------

def _torch_f8(t, s):
    """Dequantized FP8 E4M3 value of t with scale s through torch's own
    float8_e4m3fn cast (its rounding is an implementation independent of the
    oracle's); the quotient is formed in float32. torch's cast turns values of
    464 and more into NaN instead of saturating, so they are first clamped to
    the largest finite value 448 (the format's saturating conversion)."""
    q = (t.float() * torch.tensor(1.0 / float(s), dtype=torch.float64).float())
    return q.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).double() * float(s)


def _torch_mlp(cfg, W, p, x, amax=None):
    """MLP sublayer from torch calls; with cfg.mlp_fp8 each Linear multiplies
    FP8 images of its own input and weight (weights: per-tensor scale
    max|w|/448 in float32; activations a = RMSNorm(x) and h: the static
    scales)."""
    a = F.rms_norm(x, (cfg.d_model,), W[p + "norm2_g"], eps=cfg.norm_eps)
    if not getattr(cfg, "mlp_fp8", 0):
        h = F.gelu(F.linear(a, W[p + "w1"], W[p + "b1"]))
        if amax is not None:
            amax[p + "a"] = max(amax.get(p + "a", 0.0), float(a.abs().max()))
            amax[p + "h"] = max(amax.get(p + "h", 0.0), float(h.abs().max()))
        return F.linear(h, W[p + "w2"], W[p + "b2"])

    def wq(w):
        s = float(torch.tensor(float(w.abs().max()) / 448.0).float())
        return (w / s).to(torch.float8_e4m3fn).double() * s

    h = F.gelu(F.linear(_torch_f8(a, W[p + "fp8_sa"]), wq(W[p + "w1"]), W[p + "b1"]))
    return F.linear(_torch_f8(h, W[p + "fp8_sh"]), wq(W[p + "w2"]), W[p + "b2"])


def _torch_library_decoder(cfg, weights, z, amax=None):
    """Full-sequence forward built from torch library calls (F.linear,
    F.rms_norm, F.scaled_dot_product_attention with a boolean mask, F.gelu,
    F.pixel_unshuffle / F.pixel_shuffle) and RoPE as complex multiplication
    at absolute frame positions. Shares no code with the oracle."""
    W = {k: torch.from_numpy(np.asarray(v, np.float64)) for k, v in weights.items()}
    T = z.shape[0]
    H, G, Dh, L = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.L_frm
    zt = torch.from_numpy(np.asarray(z, np.float64))
    toks = F.pixel_unshuffle(zt, cfg.patch)                      # [T][C'p^2][th][tw]
    toks = toks.flatten(2).transpose(1, 2).reshape(T * L, cfg.c_in)
    x = F.linear(toks, W["embed_w"], W["embed_b"])
    fr = torch.arange(T).repeat_interleave(L)
    n = torch.arange(L).repeat(T)
    pos_axes = [fr.double(), (n // cfg.tok_w).double(), (n % cfg.tok_w).double()]
    parts = [Dh // 4, 3 * Dh // 8, Dh - Dh // 4 - 3 * Dh // 8]

    def rope(t):                                                 # t [S][heads][Dh]
        chunks, lo = [], 0
        for d, pos in zip(parts, pos_axes):
            c = torch.view_as_complex(t[..., lo:lo + d].reshape(*t.shape[:2], d // 2, 2).contiguous())
            freq = cfg.rope_theta ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)
            c = c * torch.polar(torch.ones(()).double(), pos[:, None, None] * freq)
            chunks.append(torch.view_as_real(c).reshape(*t.shape[:2], d))
            lo += d
        return torch.cat(chunks, -1)

    mask = (fr[None, :] <= fr[:, None]) & (fr[None, :] >= fr[:, None] - cfg.window)
    for l in range(cfg.n_blocks):
        p = f"b{l}."
        a = F.rms_norm(x, (cfg.d_model,), W[p + "norm1_g"], eps=cfg.norm_eps)
        qkv = F.linear(a, W[p + "wqkv"], W[p + "bqkv"])
        q, k, v = qkv.split([H * Dh, G * Dh, G * Dh], -1)
        q, k, v = q.view(-1, H, Dh), k.view(-1, G, Dh), v.view(-1, G, Dh)
        if cfg.kv_norm:
            k = F.rms_norm(k, (Dh,), W[p + "knorm_g"], eps=cfg.norm_eps)
            v = F.rms_norm(v, (Dh,), W[p + "vnorm_g"], eps=cfg.norm_eps)
        q, k = rope(q), rope(k)
        k = k.repeat_interleave(H // G, dim=1)
        v = v.repeat_interleave(H // G, dim=1)
        o = F.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1),
                                           v.transpose(0, 1), attn_mask=mask)
        x = x + F.linear(o.transpose(0, 1).reshape(-1, H * Dh), W[p + "wo"], W[p + "bo"])
        x = x + _torch_mlp(cfg, W, p, x, amax)
    y = F.linear(F.rms_norm(x, (cfg.d_model,), W["final_g"], eps=cfg.norm_eps),
                 W["out_w"], W["out_b"])
    y = y.view(T, cfg.tok_h, cfg.tok_w, cfg.c_out).permute(0, 3, 1, 2)
    out = F.pixel_shuffle(y, cfg.px_per_token)
    return out.reshape(T, *cfg.out_shape).numpy()


def _small(**kw):
    base = dict(grid_h=4, grid_w=6, latent_ch=4, patch=1, d_model=32, n_heads=2,
                n_kv_heads=2, head_dim=16, n_blocks=2, window=2, px_per_token=2)
    base.update(kw)
    return TINY.replace(name="small", **base)


@pytest.mark.parametrize("kw", [
    dict(),
    dict(kv_norm=0),
    dict(n_heads=4, n_kv_heads=2),
    dict(patch=2, grid_h=8, grid_w=6, window=1),
    dict(window=0, n_blocks=1),
])
def test_streaming_oracle_matches_torch_library_composition(kw):
    cfg = _small(**kw)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=6)
    got = oracle.decode_video(cfg, w, z)
    ref = _torch_library_decoder(cfg, w, z)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)


# --------------------------------------------------------------------------
# The method's invariants
# --------------------------------------------------------------------------

def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("kw", [dict(), dict(n_heads=4, n_kv_heads=2), dict(kv_norm=0, window=1)])
def test_invariant1_streaming_equals_masked_full_sequence(kw):
    # [FD] Sec. 3.3: streaming with a rolling cache computes the same result
    # as one pass with a sliding-window mask. T'=7 > W+1: wrap-around covered.
    cfg = TINY.replace(**kw)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=7)
    s = oracle.decode_video(cfg, w, z)
    f = oracle.full_sequence(cfg, w, z)
    assert _rel(s, f) <= 1e-12


def test_invariant2_causality():
    # [FD] Sec. 3.3: future frames have not been fed, so they cannot matter.
    cfg = TINY
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=6)
    base = oracle.decode_video(cfg, w, z)
    for s in (3, 5):
        pert = oracle.decode_video(cfg, w, fd_synth.perturb_frame(z, s))
        np.testing.assert_array_equal(pert[:s], base[:s])
        assert not np.array_equal(pert[s], base[s])


def test_invariant3a_one_block_window_bound():
    # a 1-block model: frame t depends on frames t-W .. t only
    cfg = TINY.replace(n_blocks=1)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=7)
    base = oracle.decode_video(cfg, w, z)
    t = 6
    for s in range(0, t - cfg.window):
        pert = oracle.decode_video(cfg, w, fd_synth.perturb_frame(z, s))
        np.testing.assert_array_equal(pert[t], base[t])
    pert = oracle.decode_video(cfg, w, fd_synth.perturb_frame(z, t - cfg.window))
    assert not np.array_equal(pert[t], base[t])


def test_invariant3b_receptive_field_of_the_full_model():
    # n_blocks stacked windows: frame t depends on frames >= t - n_blocks*W.
    # Positive control: a frame older than W (but inside n_blocks*W) matters.
    cfg = TINY.replace(window=1)            # n_blocks*W = 2
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=7)
    base = oracle.decode_video(cfg, w, z)
    t, reach = 6, cfg.n_blocks * cfg.window
    for s in range(0, t - reach):
        pert = oracle.decode_video(cfg, w, fd_synth.perturb_frame(z, s))
        np.testing.assert_array_equal(pert[t], base[t])
    pert = oracle.decode_video(cfg, w, fd_synth.perturb_frame(z, t - cfg.window - 1))
    assert not np.array_equal(pert[t], base[t])


def test_invariant4_cache_memory_constant():
    # [FD] Sec. 3.3 "Complexity Analysis": the cache holds at most W+1 frames.
    cfg = _small(grid_h=2, grid_w=2)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=200)
    dec = oracle.OracleDecoder(cfg, w)
    sizes = []
    for t in range(200):
        dec.decode_frame(z[t])
        sizes.append(dec.cache_bytes())
        assert all(len(dq) == min(t + 1, cfg.window + 1) for dq in dec.cache)
    assert len(set(sizes[cfg.window:])) == 1
    assert sizes[0] * (cfg.window + 1) == sizes[-1]


def test_zero_query_weights_give_window_mean_of_values():
    # closed form: W_q = 0, b_q = 0 -> uniform attention over the window
    cfg = _small(n_blocks=1)
    w = fd_synth.make_weights(cfg)
    H, Dh = cfg.n_heads, cfg.head_dim
    w["b0.wqkv"][:H * Dh] = 0
    w["b0.bqkv"][:H * Dh] = 0
    z = fd_synth.make_latents(cfg, frames=5)
    dec = oracle.OracleDecoder(cfg, w)
    for t in range(5):
        x0 = dec.embed(z[t])
        dec.decode_frame(z[t])
        # expected attention output from the cached values, by hand
        vs = np.stack([kv[1] for kv in dec.cache[0]])            # [frames][L][G][Dh]
        mean_v = vs.mean(axis=(0, 1))                             # [G][Dh]
        o = np.broadcast_to(mean_v.reshape(1, -1), (cfg.L_frm, H * Dh))
        x1 = x0 + fo.linear(o, dec.w["b0.wo"], dec.w["b0.bo"])
        a = fo.rms_norm(x1, dec.w["b0.norm2_g"], cfg.norm_eps)
        x2 = x1 + fo.linear(fo.gelu(fo.linear(a, dec.w["b0.w1"], dec.w["b0.b1"])),
                            dec.w["b0.w2"], dec.w["b0.b2"])
        # the decoder's own output for frame t equals the head of x2
        ref = dec.head(x2)
        dec2 = oracle.OracleDecoder(cfg, w)
        for s in range(t + 1):
            out = dec2.decode_frame(z[s])
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# The paper's output head ([FD] Sec. 3.4)
# --------------------------------------------------------------------------

def _paper(**kw):
    base = dict(head="paper", n_refine=2, window=1, n_blocks=1)
    base.update(kw)
    return _small(**base)


def _torch_library_paper_decoder(cfg, weights, z):
    """Paper head on top of the torch-library backbone: F.linear for the
    temporal upsampling, the same masked library block for the refinement
    blocks over all r_t T' sub-frames (absolute sub-frame positions),
    F.rms_norm + F.linear + F.gelu + F.linear, F.pixel_shuffle."""
    W = {k: torch.from_numpy(np.asarray(v, np.float64)) for k, v in weights.items()}
    T, L, D, rt = z.shape[0], cfg.L_frm, cfg.d_model, cfg.r_t
    H, G, Dh = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    parts = [Dh // 4, 3 * Dh // 8, Dh - Dh // 4 - 3 * Dh // 8]

    def rope(t, pos_axes):
        chunks, lo = [], 0
        for d, pos in zip(parts, pos_axes):
            c = torch.view_as_complex(t[..., lo:lo + d].reshape(*t.shape[:2], d // 2, 2).contiguous())
            freq = cfg.rope_theta ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)
            c = c * torch.polar(torch.ones(()).double(), pos[:, None, None] * freq)
            chunks.append(torch.view_as_real(c).reshape(*t.shape[:2], d))
            lo += d
        return torch.cat(chunks, -1)

    def block(x, p, fr, span):
        n = torch.arange(x.shape[0]) % L
        pos_axes = [fr.double(), (n // cfg.tok_w).double(), (n % cfg.tok_w).double()]
        mask = (fr[None, :] <= fr[:, None]) & (fr[None, :] > fr[:, None] - span)
        a = F.rms_norm(x, (D,), W[p + "norm1_g"], eps=cfg.norm_eps)
        q, k, v = F.linear(a, W[p + "wqkv"], W[p + "bqkv"]).split([H * Dh, G * Dh, G * Dh], -1)
        q, k, v = q.view(-1, H, Dh), k.view(-1, G, Dh), v.view(-1, G, Dh)
        if cfg.kv_norm:
            k = F.rms_norm(k, (Dh,), W[p + "knorm_g"], eps=cfg.norm_eps)
            v = F.rms_norm(v, (Dh,), W[p + "vnorm_g"], eps=cfg.norm_eps)
        q, k = rope(q, pos_axes), rope(k, pos_axes)
        k, v = k.repeat_interleave(H // G, 1), v.repeat_interleave(H // G, 1)
        o = F.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1),
                                           v.transpose(0, 1), attn_mask=mask)
        x = x + F.linear(o.transpose(0, 1).reshape(-1, H * Dh), W[p + "wo"], W[p + "bo"])
        return x + _torch_mlp(cfg, W, p, x)

    zt = torch.from_numpy(np.asarray(z, np.float64))
    toks = F.pixel_unshuffle(zt, cfg.patch).flatten(2).transpose(1, 2).reshape(T * L, cfg.c_in)
    x = F.linear(toks, W["embed_w"], W["embed_b"])
    fr = torch.arange(T).repeat_interleave(L)
    for l in range(cfg.n_blocks):
        x = block(x, f"b{l}.", fr, cfg.window + 1)
    up = F.linear(x, W["up_w"], W["up_b"]).view(T, L, rt, D).permute(0, 2, 1, 3).reshape(-1, D)
    sub = torch.arange(T * rt).repeat_interleave(L)
    for l in range(cfg.n_refine):
        up = block(up, f"r{l}.", sub, rt * (cfg.window + 1))
    h = F.gelu(F.linear(F.rms_norm(up, (D,), W["final_g"], eps=cfg.norm_eps), W["sp1_w"], W["sp1_b"]))
    y = F.linear(h, W["out_w"], W["out_b"]).view(T * rt, cfg.tok_h, cfg.tok_w, cfg.c_px)
    px = F.pixel_shuffle(y.permute(0, 3, 1, 2), cfg.px_per_token)      # [T rt][C][H][W]
    return px.view(T, rt, *px.shape[1:]).permute(0, 2, 1, 3, 4).numpy()


@pytest.mark.parametrize("kw", [dict(), dict(n_heads=4, n_kv_heads=2), dict(window=0, n_refine=1)])
def test_paper_head_streaming_matches_torch_library_composition(kw):
    cfg = _paper(**kw)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=4)
    got = oracle.decode_video(cfg, w, z)
    ref = _torch_library_paper_decoder(cfg, w, z)
    assert got.shape == ref.shape == (4,) + tuple(cfg.out_shape)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)


def test_paper_head_streaming_equals_masked_full_sequence():
    # 4 latent frames -> 16 sub-frames through a refinement window of
    # r_t (W+1) = 8 sub-frames: eviction in the refinement cache is covered
    cfg = _paper(grid_h=2, grid_w=4)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=4)
    s = oracle.decode_video(cfg, w, z)
    f = oracle.full_sequence(cfg, w, z)
    assert _rel(s, f) <= 1e-12


def test_paper_head_causality_and_cache_bound():
    cfg = _paper()
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=5)
    base = oracle.decode_video(cfg, w, z)
    pert = oracle.decode_video(cfg, w, fd_synth.perturb_frame(z, 3))
    np.testing.assert_array_equal(pert[:3], base[:3])
    assert not np.array_equal(pert[3], base[3])
    dec = oracle.OracleDecoder(cfg, w)
    for t in range(5):
        dec.decode_frame(z[t])
        assert all(len(dq) == min(cfg.r_t * (t + 1), cfg.r_t * (cfg.window + 1)) for dq in dec.rcache)
