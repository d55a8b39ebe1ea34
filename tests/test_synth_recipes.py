"""The seeded input recipes (the synthetic workloads stand in for the pages' audio):
each clip and weight tensor is what the recipe states, checked against its own definition
written out here."""
import numpy as np

import oracle as O
from speech_audio_encoder_b200 import synth


def test_tones_clip_is_two_tones_plus_small_noise():
    x = synth.tones_clip(16000, 0).astype(np.float64)
    t = np.arange(16000) / 16000.0
    noise = x - (0.5 * np.sin(2 * np.pi * 440 * t) + 0.2 * np.sin(2 * np.pi * 1000 * t))
    assert abs(noise.std() - 0.01) < 0.0005 and abs(noise.mean()) < 0.001


def test_bursts_clip_noise_is_a_one_pole_lowpass_of_white_noise():
    n = 4000
    x = synth.bursts_clip(n, seed=3, n_bursts=0).astype(np.float64)
    w = np.random.default_rng(3).normal(0.0, 0.1, n)
    y = np.empty(n)
    acc = 0.0
    for i in range(n):  # y[n] = 0.95 y[n-1] + 0.05 w[n]
        acc = 0.95 * acc + 0.05 * w[i]
        y[i] = acc
    assert np.allclose(x, y.astype(np.float32), atol=1e-6)


def test_envelope_recipe_multiplies_by_the_4hz_syllable_rate():
    n = 8000
    plain = synth.bursts_clip(n, seed=5).astype(np.float64)
    env = synth.bursts_clip(n, seed=5, envelope=True).astype(np.float64)
    t = np.arange(n) / 16000.0
    assert np.allclose(env, (plain * (0.55 + 0.45 * np.sin(2 * np.pi * 4 * t))).astype(np.float32), atol=1e-6)


def test_workloads_match_their_stated_lengths():
    for name, (B, secs) in {"tones_1s": (1, 1), "clip_30s": (1, 30), "batch16_60s": (16, 60),
                            "rec_10min": (1, 600), "rec_1h": (1, 3600)}.items():
        wl = synth.WORKLOADS[name]
        assert wl.batch == B and wl.n_samples == secs * 16000
        assert O.position_count(wl.n_samples) == ((secs * 16000 - 400) // 160 + 1) // 8


def test_speaker_activity_recipe():
    P = synth.speaker_activity(2000, seed=4)
    assert P.shape == (2000, 8) and P.dtype == np.float32
    assert P.min() >= 0.0 and P.max() <= 1.0
    assert (P == 0.5).sum() >= 1                       # threshold entries are present
    active = P > 0.5
    assert active[:, :3].mean() > 0.2                  # three speakers take turns
    assert active[:, 3:].mean() < 0.02                 # unused slots stay near 0 (noise only)


def test_weight_recipes_and_bf16_rounding():
    w = synth.make_weights(1, seed=11)
    bits, vals = w["layers"][0]["w_qkv"]
    assert bits.shape == (3840, 1280) and vals.dtype == np.float32
    raw = np.random.default_rng(11 + 4 + 2).standard_normal((3840, 1280)) * 0.02  # 4 globals, then ln1_g, ln1_b
    assert np.allclose(vals, raw, rtol=2 ** -8, atol=0)
    assert np.array_equal(synth.bf16_to_f32(synth.bf16_bits(vals)), vals)  # already representable
    g = w["layers"][0]["ln1_g"][1]
    assert abs(g.mean() - 1.0) < 0.01 and 0.01 < g.std() < 0.03
    fz = synth.make_fusion_weights()
    assert fz["w_conn"][0].shape == (2688, 1280) and fz["spk_g"][0].shape == (8,)
    cw = synth.make_ctc_weights(n_layers=1, classes=100, in_width=64, width=32, ffn=128, head_dim=8)
    assert cw["w_up"][0].shape == (2, 32, 64) and cw["w_out"][0].shape == (100, 32)
    assert cw["layers"][0]["w1"][0].shape == (128, 32)
