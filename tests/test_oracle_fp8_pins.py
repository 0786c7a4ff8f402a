"""Pins of the oracle's FP8 MLP ([FD] Sec. 4.6, optimization (4): static-
calibrated FP8 quantization of all MLP layers) to things other than itself:
torch's float8_e4m3fn cast (an independent rounding implementation), the
E4M3 value set enumerated by torch from all 256 bit patterns, a full decoder
composed of torch calls, and the method's invariants with FP8 on.
"""
import numpy as np
import pytest
import torch

import fd_synth
import oracle
from oracle import flashdec_oracle as fo

from test_oracle_pins import _paper, _rel, _small, _torch_library_decoder, \
    _torch_library_paper_decoder


def _e4m3_values():
    v = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    return v[~np.isnan(v)]


def test_e4m3_round_equals_torch_cast_on_every_bf16_value_in_range():
    # all 65536 bf16 bit patterns: every binade, the subnormal range, exact ties
    v = torch.arange(-32768, 32768, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
    v = v[torch.isfinite(v) & (v.abs() < 464)]
    got = fo.e4m3_round(v.double().numpy())
    ref = v.to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))          # -0 stays -0


def test_e4m3_round_equals_torch_cast_on_random_float32():
    g = np.random.default_rng(3)
    mag = np.exp2(g.uniform(-14, np.log2(463), 200000))
    v = (mag * g.choice([-1.0, 1.0], mag.size)).astype(np.float32)
    got = fo.e4m3_round(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(got, ref)


def test_e4m3_value_set_saturation_and_idempotence():
    vals = _e4m3_values()
    assert vals.size == 254 and len(set(vals.tolist())) == 253     # +0 and -0
    assert vals.max() == fo.E4M3_MAX == 448.0
    g = np.random.default_rng(4)
    v = g.standard_normal(50000) * np.exp2(g.uniform(-12, 12, 50000))
    q = fo.e4m3_round(v)
    assert set(np.unique(q)).issubset(set(vals.tolist()))
    np.testing.assert_array_equal(fo.e4m3_round(q), q)
    assert np.all(np.diff(fo.e4m3_round(np.sort(v))) >= 0)           # monotonic
    # satfinite: beyond the largest finite value, including infinities
    big = np.array([464.0, 479.9, 480.0, 1e6, np.inf, -500.0, -np.inf])
    np.testing.assert_array_equal(fo.e4m3_round(big), [448, 448, 448, 448, 448, -448, -448])
    assert np.isnan(fo.e4m3_round(np.array([np.nan]))[0])
    # smallest subnormal 2^-9; half of it is a tie and goes to the even 0
    np.testing.assert_array_equal(fo.e4m3_round(np.array([2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10])),
                                  [2.0 ** -9, 0.0, 2.0 ** -8])


def test_activation_rounding_is_decided_in_float32():
    # 1.0625 is the tie between 1.0 and 1.125; in float64 the value just above
    # it would round up, but its float32 image is the tie itself -> even 1.0
    x = np.array([1.0625 + 2.0 ** -40])
    assert fo.e4m3_round(x)[0] == 1.125
    assert fo.quantize_act(x, 1.0)[0] == 1.0
    # the scale divides: x = 3 s is exactly representable
    assert fo.quantize_act(np.array([0.75]), 0.25)[0] == 0.75


def test_weight_quantization_uses_a_float32_per_tensor_scale():
    w = np.random.default_rng(5).standard_normal((8, 16))
    s = fo.weight_scale(w)
    assert s == float(np.float32(np.abs(w).max() / 448.0))
    q = fo.quantize_weight(w, s)
    assert np.abs(q).max() == pytest.approx(448.0 * s, rel=1e-6)
    codes = q / s
    assert set(np.unique(codes)).issubset(set(_e4m3_values().tolist()))
    assert fo.weight_scale(np.zeros((3, 3))) == 1.0


def _fp8(cfg_kw, frames=5):
    cfg = _small(**cfg_kw)
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=frames)
    scales = oracle.calibrate_fp8(cfg, w, z)
    return cfg.replace(mlp_fp8=1), {**w, **scales}, z, scales


@pytest.mark.parametrize("kw", [dict(), dict(n_heads=4, n_kv_heads=2), dict(window=0, n_blocks=1)])
def test_fp8_streaming_decoder_matches_torch_library_composition(kw):
    cfg, w, z, _ = _fp8(kw)
    got = oracle.decode_video(cfg, w, z)
    ref = _torch_library_decoder(cfg, w, z)
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-9)


def test_fp8_paper_head_matches_torch_library_composition():
    cfg = _paper()
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=4)
    scales = oracle.calibrate_fp8(cfg, w, z)
    assert set(scales) == {f"{p}fp8_s{k}" for p in ("b0.", "r0.", "r1.") for k in "ah"}
    cfg8, w8 = cfg.replace(mlp_fp8=1), {**w, **scales}
    got = oracle.decode_video(cfg8, w8, z)
    np.testing.assert_allclose(got, _torch_library_paper_decoder(cfg8, w8, z), rtol=1e-9, atol=1e-9)


def test_calibration_is_the_amax_of_the_unquantized_mlp_activations():
    cfg = _small()
    w = fd_synth.make_weights(cfg)
    z = fd_synth.make_latents(cfg, frames=5)
    scales = oracle.calibrate_fp8(cfg, w, z)
    amax = {}
    _torch_library_decoder(cfg, w, z, amax)               # one pass over all frames
    assert set(scales) == {f"b{l}.fp8_s{k}" for l in range(cfg.n_blocks) for k in "ah"}
    for key, a in amax.items():
        p, kind = key[:-1], key[-1]
        assert scales[p + "fp8_s" + kind] == float(np.float32(a / 448.0))


def test_fp8_invariants():
    cfg, w, z, _ = _fp8(dict(), frames=7)
    s = oracle.decode_video(cfg, w, z)
    # streaming == masked full sequence (static scales: position independent)
    assert _rel(s, oracle.full_sequence(cfg, w, z)) <= 1e-12
    # causality with FP8 on
    pert = oracle.decode_video(cfg, w, fd_synth.perturb_frame(z, 5))
    np.testing.assert_array_equal(pert[:5], s[:5])
    # FP8 changes the result, but only by the format's relative precision
    ref = oracle.decode_video(cfg.replace(mlp_fp8=0), w, z)
    assert 1e-4 < _rel(s, ref) < 5e-2
