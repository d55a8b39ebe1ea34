"""The C++ oracle (oracle/sal_oracle.cpp) against a second formulation of every step in
numpy (tests/numpy_oracle.py), on seeded random inputs and on the synthetic audio.

The two share no code: the C++ side is textbook loops in double precision, the numpy side
one library primitive per step. Agreement to ~1e-12 means a mistake would have had to be
made twice, in two languages and two styles. The properties each function must have are
pinned separately (tests/test_oracle_*.py); this file only ties the two formulations.
"""
import numpy as np
import pytest

import numpy_oracle as N
import oracle as O
from speech_audio_encoder_b200 import synth

RTOL = 1e-12


def _close(a, b, tol=RTOL):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert a.shape == b.shape
    scale = max(np.abs(b).max(), 1e-300)
    assert np.abs(a - b).max() <= tol * scale, np.abs(a - b).max() / scale


def test_front_end_tables():
    _close(O.hann_window(), N.hann_window(), 1e-15)
    _close(O.mel_filterbank(), N.mel_filterbank(), 1e-13)
    f = np.array([0.0, 300.0, 999.0, 1000.0, 2500.0, 8000.0])
    _close(O.hz_to_mel(f), N.hz_to_mel(f), 1e-14)
    _close(O.mel_to_hz(O.hz_to_mel(f)), f, 1e-13)


@pytest.mark.parametrize("name", ["tones_1s", "clip_30s"])
def test_log_mel_and_stacking(name):
    wave = synth.WORKLOADS[name].audio()[0]
    a, b = O.log_mel(wave), N.log_mel(wave)
    assert np.abs(a - b).max() < 1e-9  # log of sums: absolute, as the GPU bar is
    _close(O.stack_frames(a), N.stack_frames(a), 0.0)
    y = N.frame_signal(wave, 5, 7)
    _close(O.frame_signal(wave, 5, 7), y, 1e-15)
    _close(O.power_spectrum(y), N.power_spectrum(y), 1e-11)


def test_encoder_pieces():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((37, 96))
    w, b = rng.standard_normal((50, 96)), rng.standard_normal(50)
    _close(O.linear(x, w, b), N.linear(x, w, b))
    g, bb = rng.standard_normal(96), rng.standard_normal(96)
    _close(O.layer_norm(x, g, bb), N.layer_norm(x, g, bb))
    _close(O.rms_norm(x, g), N.rms_norm(x, g))
    q = rng.standard_normal((3, 37, 16))
    pos = np.arange(37) * 97.0
    _close(O.rope(q, pos), N.rope(q, pos))
    k, v = rng.standard_normal((3, 41, 16)), rng.standard_normal((3, 41, 16))
    _close(O.attention(q, k, v), N.attention(q, k, v))
    _close(O.attention_probs(q[0], k[0]), N.attention_probs(q[0], k[0]))
    _close(O.gelu(x), N.gelu(x))
    z = rng.standard_normal((4, 1000)) * 5
    _close(O.log_softmax(z), N.log_softmax(z))
    _close(O.speaker_kernel(), N.speaker_kernel(), 1e-14)


def test_full_width_layer_and_rows():
    w = synth.weights_f32(synth.make_weights(1))
    lw = w["layers"][0]
    x = np.random.default_rng(1).standard_normal((300, 1280))
    _close(O.encoder_layer(x, lw), N.encoder_layer(x, lw))
    rows = np.array([299, 0, 150])
    _close(O.encoder_layer_rows(x, lw, rows), N.encoder_layer_rows(x, lw, rows))
    _close(O.encoder_layer_chunked(x, lw, 128), N.encoder_layer_chunked(x, lw, 128))


def test_windows_fusion_connector_ctc():
    dims = O.EncoderDims(width=16, heads=2, head_dim=8, ffn=64, stack_in=32)
    w = synth.weights_f32(synth.make_weights(2, seed=5, width=16, ffn=64, head_dim=8, stack_in=32,
                                             std=0.3, gain_std=0.3))
    x = np.random.default_rng(2).standard_normal((23, 16))
    _close(O.encoder_forward_windowed(x, w, 2, 6, 2, dims), N.encoder_forward_windowed(x, w, 2, 6, 2, dims))
    assert O.window_bounds(1234) == N.window_bounds(1234)
    rng = np.random.default_rng(3)
    H, P = rng.standard_normal((40, 1280)), rng.random((40, 8))
    g, b = 1 + 0.1 * rng.standard_normal(8), 0.1 * rng.standard_normal(8)
    _close(O.speaker_fuse(H, P, g, b), N.speaker_fuse(H, P, g, b))
    W, bias = rng.standard_normal((2688, 1280)) * 0.02, rng.standard_normal(2688)
    _close(O.connector(H, W, bias), N.connector(H, W, bias))
    cd = O.CtcDims(in_width=16, width=16, heads=2, head_dim=8, ffn=64, layers=2, classes=50)
    cw = synth.weights_f32(synth.make_ctc_weights(seed=9, in_width=16, width=16, head_dim=8, ffn=64,
                                                  classes=50))
    h = rng.standard_normal((9, 16))
    _close(O.ctc_adapter(h, cw, cd), N.ctc_adapter(h, cw, N.CtcDims(in_width=16, width=16, heads=2,
                                                                    head_dim=8, ffn=64, layers=2,
                                                                    classes=50)))
