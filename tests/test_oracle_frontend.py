"""Pins for the oracle's front end: counts, window, DFT power, mel filters, log, stacking.

Each test checks the oracle against something other than itself: numbers the pages
print (tests/golden/page_facts.json), closed forms, identities (Parseval, scaling),
library routines for special cases (numpy's FFT), or brute force on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


# ---------------------------------------------------------------- counts

def test_window_and_hop_from_page_facts():
    fe = GOLDEN["front_end"]
    assert O.WIN == fe["sample_rate_hz"] * fe["window_ms"] // 1000
    assert O.HOP == fe["sample_rate_hz"] * fe["hop_ms"] // 1000
    assert O.NFFT == fe["fft_points"] and O.NMEL == fe["n_mels"] and O.STACK == fe["stacked_frames"]
    # 100 frames/s and 12.5 embeddings/s, 80 ms per position
    assert fe["sample_rate_hz"] / O.HOP == fe["frames_per_second_approx"]
    assert fe["frames_per_second_approx"] / O.STACK == fe["embeddings_per_second"]
    assert 1000 * O.STACK * O.HOP / fe["sample_rate_hz"] == fe["ms_per_position"]


def _frames_brute(n):
    # enumerate every start s = 160 f whose 400-sample window fits in n samples
    return sum(1 for s in range(0, n + 1, O.HOP) if s + O.WIN <= n)


@pytest.mark.parametrize("n", list(range(0, 1200)) + [400 + 160 * k + d for k in (5, 97, 1000) for d in (-1, 0, 1)])
def test_frame_count_brute_force(n):
    assert O.frame_count(n) == _frames_brute(n)
    assert O.position_count(n) == _frames_brute(n) // 8


def test_position_counts_against_page_nominals():
    pos = GOLDEN["positions"]
    t30 = O.position_count(30 * 16000)
    t1h = O.position_count(3600 * 16000)
    assert (t30, t1h) == (374, 44999)
    # the pages quote 12.5 D "ignoring padding/rounding at the ends"
    assert abs(t30 - pos["per_30s_nominal"]) <= 1
    assert abs(t1h - pos["per_hour_nominal"]) <= 1
    assert t1h <= O.MAX_POSITIONS


def test_hour_waveform_size():
    wb = GOLDEN["waveform_bytes"]
    n = 3600 * 16000
    assert n * 4 == pytest.approx(wb["hour_fp32_mb"] * 1e6)
    assert n * 2 == pytest.approx(wb["hour_pcm16_mb"] * 1e6)


# ---------------------------------------------------------------- window and DFT

def test_hann_periodic_closed_form():
    w = O.hann_window()
    assert w.shape == (400,)
    assert w[0] == 0.0 and w[200] == pytest.approx(1.0, abs=1e-15)
    assert np.allclose(w[1:], w[1:][::-1], atol=1e-15)  # periodic: w[n] = w[400 - n]
    assert w.sum() == pytest.approx(200.0, abs=1e-9)      # sum of a periodic Hann = N / 2
    assert (w * w).sum() == pytest.approx(150.0, abs=1e-9)  # 3N/8


def test_power_matches_numpy_fft():
    rng = np.random.default_rng(5)
    y = rng.standard_normal((7, 400))
    ref = np.abs(np.fft.rfft(y, n=512, axis=-1)) ** 2
    got = O.power_spectrum(y)
    assert got.shape == (7, 257)
    assert np.allclose(got, ref, rtol=1e-10, atol=1e-9)


def test_parseval():
    rng = np.random.default_rng(6)
    y = rng.standard_normal((5, 400))
    P = O.power_spectrum(y)
    # Hermitian extension: bins 1..255 appear twice in the full 512-point spectrum
    full = P[:, 0] + P[:, 256] + 2.0 * P[:, 1:256].sum(axis=1)
    assert np.allclose(full, 512.0 * (y * y).sum(axis=1), rtol=1e-11)


@pytest.mark.parametrize("freq,bin_", [(1000.0, 32), (440.0, 14), (4000.0, 128), (250.0, 8)])
def test_tone_peak_bin(freq, bin_):
    t = np.arange(400) / 16000.0
    y = np.sin(2 * np.pi * freq * t) * O.hann_window()
    P = O.power_spectrum(y[None])[0]
    assert int(np.argmax(P)) == bin_
    assert freq * 512 / 16000 == pytest.approx(bin_, abs=0.5)


def test_circular_shift_invariance():
    # |X_k|^2 does not depend on where the 400 samples sit in the 512 buffer
    rng = np.random.default_rng(7)
    y = rng.standard_normal(400)
    buf = np.zeros(512)
    buf[:400] = y
    P0 = O.power_spectrum(buf[None])[0]
    P1 = O.power_spectrum(np.roll(buf, 77)[None])[0]
    assert np.allclose(P0, P1, rtol=1e-10, atol=1e-9)
    assert np.allclose(P0, O.power_spectrum(y[None])[0], rtol=1e-12, atol=1e-10)


# ---------------------------------------------------------------- mel filters

def test_slaney_mel_scale_closed_forms():
    assert O.hz_to_mel(0.0) == 0.0
    assert O.hz_to_mel(1000.0) == pytest.approx(15.0, abs=1e-12)
    assert O.hz_to_mel(500.0) == pytest.approx(7.5, abs=1e-12)
    assert O.hz_to_mel(6400.0) == pytest.approx(15.0 + 27.0, abs=1e-12)  # ln(6.4)/27 per mel
    assert O.hz_to_mel(8000.0) == pytest.approx(15.0 + 27.0 * math.log(8.0) / math.log(6.4))
    f = np.array([0.0, 10.0, 999.0, 1000.0, 1234.5, 7999.0])
    assert np.allclose(O.mel_to_hz(O.hz_to_mel(f)), f, rtol=1e-12, atol=1e-9)


def test_mel_filterbank_structure():
    W = O.mel_filterbank()
    assert W.shape == (128, 257)
    nz = W > 0
    assert nz.sum() == 504
    assert nz.sum(axis=1).min() >= 1          # no empty filter
    assert nz.sum(axis=0).max() <= 2          # each bin in at most two filters
    pts = O.mel_to_hz(np.linspace(0.0, O.hz_to_mel(8000.0), 130))
    fk = np.arange(257) * 31.25
    for m in range(128):
        idx = np.nonzero(nz[m])[0]
        assert np.all(np.diff(idx) == 1)      # contiguous support
        assert fk[idx[0]] > pts[m] and fk[idx[-1]] < pts[m + 2]
        # rising below the apex f_{m+1}, falling above
        row = W[m, idx]
        apex = int(np.argmax(row))
        assert np.all(np.diff(row[:apex + 1]) >= 0) and np.all(np.diff(row[apex:]) <= 0)
        assert abs(fk[idx[apex]] - pts[m + 1]) <= 31.25
        # apex height is the Slaney area normalisation 2 / (f_{m+2} - f_m) times <= 1
        assert row.max() <= 2.0 / (pts[m + 2] - pts[m]) + 1e-15


def test_mel_unnormalised_partition_of_unity():
    W = O.mel_filterbank()
    pts = O.mel_to_hz(np.linspace(0.0, O.hz_to_mel(8000.0), 130))
    un = W / (2.0 / (pts[2:] - pts[:-2]))[:, None]
    fk = np.arange(257) * 31.25
    inside = (fk >= pts[1]) & (fk <= pts[128])
    assert np.allclose(un[:, inside].sum(axis=0), 1.0, atol=1e-12)


def test_mel_area_normalisation():
    # each triangle has unit area in Hz; the 31.25 Hz sampling of wide ones is close to it
    W = O.mel_filterbank()
    pts = O.mel_to_hz(np.linspace(0.0, O.hz_to_mel(8000.0), 130))
    width = pts[2:] - pts[:-2]
    wide = width > 6 * 31.25
    area = W.sum(axis=1) * 31.25
    assert wide.sum() >= 29
    assert np.allclose(area[wide], 1.0, atol=0.02)
    # every filter's area is within the sampling error of a triangle a few bins wide
    assert np.all(np.abs(area - 1.0) < 0.5)


# ---------------------------------------------------------------- log and stacking

def test_log_floor_on_silence():
    M = O.log_mel(np.zeros(16000, np.float32))
    assert M.shape == (98, 128)
    assert np.all(M == math.log(1e-10))


def test_log_mel_scaling_identity():
    # power is quadratic and the log is natural: log_mel(a x) = log_mel(x) + 2 ln a
    rng = np.random.default_rng(8)
    x = rng.standard_normal(4000).astype(np.float32)
    M1 = O.log_mel(x)
    M2 = O.log_mel((4.0 * x).astype(np.float32))
    assert np.allclose(M2 - M1, 2.0 * math.log(4.0), atol=1e-9)


def test_log_mel_brute_force_small():
    rng = np.random.default_rng(9)
    x = rng.standard_normal(400 + 160 * 3).astype(np.float32)
    M = O.log_mel(x)
    W = O.mel_filterbank()
    for f in range(4):
        y = [float(x[160 * f + n]) * (0.5 - 0.5 * math.cos(2 * math.pi * n / 400)) for n in range(400)]
        for m in (0, 5, 64, 127):
            e = 0.0
            for k in range(257):
                if W[m, k] == 0.0:
                    continue
                re = sum(y[n] * math.cos(2 * math.pi * k * n / 512) for n in range(400))
                im = sum(y[n] * math.sin(2 * math.pi * k * n / 512) for n in range(400))
                e += W[m, k] * (re * re + im * im)
            assert M[f, m] == pytest.approx(math.log(max(e, 1e-10)), abs=1e-9)


def test_stack_layout_brute_force():
    rng = np.random.default_rng(10)
    M = rng.standard_normal((8 * 5 + 3, 128))
    S = O.stack_frames(M)
    assert S.shape == (5, 1024)
    for t in range(5):
        for j in range(8):
            for m in (0, 77, 127):
                assert S[t, 128 * j + m] == M[8 * t + j, m]


def test_identity_projection_returns_first_frame():
    rng = np.random.default_rng(11)
    M = rng.standard_normal((24, 128))
    P = np.zeros((1280, 1024))
    P[:128, :128] = np.eye(128)
    x = O.stack_project(O.stack_frames(M), {"w_proj": P, "b_proj": np.zeros(1280)})
    assert np.array_equal(x[:, :128], M[0::8])
    assert np.all(x[:, 128:] == 0)
