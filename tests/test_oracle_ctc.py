"""Pins of the oracle's CTC timestamp adapter (page "Nemotron 3.5 Transcribe: From Recorded
Speech to Dataset Audits", section "Use alignment and audio questions as supporting
evidence"): the parameter count the page gives, the transposed convolution against
torch's own, log-softmax against scipy, and the whole adapter at a tiny width against a
per-element composition of independently written pieces."""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O
from speech_audio_encoder_b200 import synth
from test_oracle_encoder import _naive_layer


def test_param_count_is_about_50m_only_at_width_1024():
    # the page: "approximately 50M-parameter CTC adapter"
    assert 45e6 <= O.ctc_param_count() <= 55e6
    for w in (768, 1280):  # the neighbouring widths with 16 heads land far from 50M
        n = O.ctc_param_count(O.CtcDims(width=w, head_dim=w // 16, ffn=4 * w))
        assert not 45e6 <= n <= 55e6


def test_upsample_is_a_stride_two_transposed_convolution():
    rng = np.random.default_rng(0)
    T, cin, cout = 7, 12, 10
    h = rng.standard_normal((T, cin))
    w = rng.standard_normal((2, cout, cin))
    b = rng.standard_normal(cout)
    got = O.ctc_upsample(h, w, b)
    # torch: input [N, C_in, L], weight [C_in, C_out, kernel], output length (L - 1) * 2 + 2
    ref = torch.nn.functional.conv_transpose1d(
        torch.from_numpy(h.T[None]), torch.from_numpy(np.transpose(w, (2, 1, 0))), torch.from_numpy(b), stride=2)
    assert ref.shape == (1, cout, 2 * T)
    assert np.allclose(got, ref[0].numpy().T, rtol=1e-12, atol=1e-12)
    # element by element
    for t in range(T):
        for j in range(2):
            for c in (0, cout - 1):
                assert got[2 * t + j, c] == pytest.approx(sum(h[t, i] * w[j, c, i] for i in range(cin)) + b[c],
                                                          abs=1e-12)


def test_log_softmax_matches_scipy_and_normalises():
    rng = np.random.default_rng(1)
    z = rng.standard_normal((4, 23863)) * 3
    got = O.log_softmax(z)
    assert np.allclose(got, scipy.special.log_softmax(z, axis=-1), rtol=1e-13, atol=1e-12)
    assert np.allclose(np.exp(got).sum(axis=-1), 1.0, atol=1e-12)
    assert np.allclose(O.log_softmax(z + 123.0), got, atol=1e-10)  # shift invariance
    assert np.all(got <= 0)


def _tiny():
    dims = O.CtcDims(in_width=8, width=16, heads=2, head_dim=8, ffn=64, layers=2, classes=5)
    w = synth.make_ctc_weights(seed=31, in_width=8, width=16, ffn=64, head_dim=8, n_layers=2, classes=5,
                               std=0.3, gain_std=0.3)
    cw = {k: np.asarray(v[1], np.float64) for k, v in w.items() if k != "layers"}
    cw["layers"] = [{k: np.asarray(v[1], np.float64) for k, v in lw.items()} for lw in w["layers"]]
    return dims, cw


@pytest.mark.parametrize("T", [1, 3])
def test_tiny_adapter_brute_force(T):
    dims, cw = _tiny()
    rng = np.random.default_rng(T)
    h = rng.standard_normal((T, 8))
    got = O.ctc_adapter(h, cw, dims)
    assert got.shape == (2 * T, 5)
    # second formulation: loops for the upsampling, the per-element layer, LN, projection,
    # log-softmax
    W = 16
    x = [[sum(h[t, i] * cw["w_up"][j, c, i] for i in range(8)) + cw["b_up"][c] for c in range(W)]
         for t in range(T) for j in range(2)]
    for lw in cw["layers"]:
        x = _naive_layer(x, {k: v.tolist() for k, v in lw.items()}, 2, 8)
    ref = []
    for row in x:
        mu = sum(row) / W
        var = sum((r - mu) ** 2 for r in row) / W
        n = [(row[i] - mu) / math.sqrt(var + 1e-5) * cw["lnf_g"][i] + cw["lnf_b"][i] for i in range(W)]
        z = [sum(n[i] * cw["w_out"][o, i] for i in range(W)) + cw["b_out"][o] for o in range(5)]
        lse = math.log(sum(math.exp(a) for a in z))
        ref.append([a - lse for a in z])
    assert np.allclose(got, np.array(ref), rtol=1e-11, atol=1e-11)


def test_adapter_rows_of_a_clip_depend_on_the_whole_clip_only_through_attention():
    # the up-sampled position 2t + j sees input t only before the first attention: with
    # the attention output projection zeroed, the adapter is per input position
    dims, cw = _tiny()
    for lw in cw["layers"]:
        lw["w_o"] = np.zeros_like(lw["w_o"])
    rng = np.random.default_rng(9)
    h = rng.standard_normal((4, 8))
    full = O.ctc_adapter(h, cw, dims)
    for t in range(4):
        assert np.allclose(O.ctc_adapter(h[t:t + 1], cw, dims), full[2 * t:2 * t + 2], atol=1e-12)
