"""GPU parity of the front-end kernel (sal_frontend) against the fp64 oracle.

Tolerances: log-mel within 1e-4 absolute of the fp64 oracle (fp32 FFT and filters);
frame and position counts bit-exact; the bf16 stacked copy equals the round-to-nearest-
even bf16 of the kernel's own fp32 log-mel, bit for bit, and is laid out frame-major.
"""
import numpy as np
import pytest
import torch

import oracle as O
from speech_audio_encoder_b200 import synth

pytestmark = pytest.mark.gpu

LOGMEL_TOL = 1e-4


def _api():
    from speech_audio_encoder_b200 import api
    return api


def _check_clip(wave_np, logmel_gpu, stacked_gpu, frames=None):
    F = O.frame_count(wave_np.shape[-1])
    T = O.position_count(wave_np.shape[-1])
    assert logmel_gpu.shape[-2] == F
    if frames is None:
        ref = O.log_mel(wave_np)
        got = logmel_gpu.double().cpu().numpy()
    else:
        first, count = frames
        ref = O.log_mel(wave_np, first=first, count=count)
        got = logmel_gpu[first:first + count].double().cpu().numpy()
    err = np.abs(got - ref).max() if ref.size else 0.0
    assert err <= LOGMEL_TOL, f"log-mel max abs error {err}"
    if stacked_gpu is not None:
        assert stacked_gpu.shape == (T, 1024)
        want = logmel_gpu[:8 * T].to(torch.bfloat16).reshape(T, 1024)
        assert torch.equal(stacked_gpu.view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("name", ["tones_1s", "clip_30s"])
def test_frontend_workloads(name):
    api = _api()
    wave = synth.WORKLOADS[name].audio()
    lm, st = api.sal_frontend(torch.from_numpy(wave).cuda())
    torch.cuda.synchronize()
    _check_clip(wave[0], lm[0], st[0])


def test_frontend_batch16_60s_sampled():
    api = _api()
    wl = synth.WORKLOADS["batch16_60s"]
    wave = wl.audio()
    lm, st = api.sal_frontend(torch.from_numpy(wave).cuda())
    torch.cuda.synchronize()
    for b in (0, 7, 15):
        _check_clip(wave[b], lm[b], st[b], frames=(b * 300, 700))


def test_frontend_one_hour_sampled():
    """Full 57.6 M-sample clip on the GPU; oracle on frames spread over the hour."""
    api = _api()
    wave = synth.WORKLOADS["rec_1h"].audio()
    lm, st = api.sal_frontend(torch.from_numpy(wave).cuda())
    torch.cuda.synchronize()
    F = O.frame_count(wave.shape[1])
    assert F == 359998 and st.shape == (1, 44999, 1024)
    for first in (0, 123457, F - 2048):
        _check_clip(wave[0], lm[0], None, frames=(first, 2048))
    # the stacked copy, frame-major, over the whole hour
    want = lm[0, :8 * 44999].to(torch.bfloat16).reshape(44999, 1024)
    assert torch.equal(st[0].view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("n", [0, 399, 400, 401, 559, 560, 561, 1679, 1680, 16000 + 3])
def test_frontend_edge_lengths(n):
    api = _api()
    rng = np.random.default_rng(n)
    wave = rng.standard_normal((3, n)).astype(np.float32) * 0.3
    assert api.frame_count(n) == O.frame_count(n)
    assert api.position_count(n) == O.position_count(n)
    lm, st = api.sal_frontend(torch.from_numpy(wave).cuda())
    torch.cuda.synchronize()
    for b in range(3):  # odd n: clips 1 and 2 start off a 16-byte boundary
        _check_clip(wave[b], lm[b], st[b])


def test_frontend_silence_and_scaling():
    api = _api()
    z = torch.zeros((1, 4000), device="cuda")
    lm, _ = api.sal_frontend(z)
    assert (lm.double() - np.log(1e-10)).abs().max().item() < 1e-5
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 8000)).astype(np.float32)
    a, _ = api.sal_frontend(torch.from_numpy(x).cuda())
    b, _ = api.sal_frontend(torch.from_numpy(4 * x).cuda())
    assert (b - a - 2 * np.log(4.0)).abs().max().item() < 1e-4


def test_frontend_rejects_bad_arguments():
    api = _api()
    lib = api.lib()
    buf = torch.empty(1024, device="cuda")
    assert lib.sal_frontend(buf.data_ptr(), 1000, -1, buf.data_ptr(), 0, 0) == 1  # EINVAL
    assert lib.sal_frontend(0, 1000, 1, buf.data_ptr(), 0, 0) == 1
    assert lib.sal_frontend(buf.data_ptr() + 4, 1000, 1, buf.data_ptr(), 0, 0) == 1  # misaligned
    assert lib.sal_frontend(buf.data_ptr(), 3600 * 16000 + 16000, 1, buf.data_ptr(), 0, 0) == 2  # > 1 h
