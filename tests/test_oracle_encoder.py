"""Pins for the oracle's encoder pieces and for a whole layer at width 16.

The whole-layer test compares the oracle against a second, deliberately naive
formulation written here with per-element loops (explicit sums, explicit exponentials,
complex-number RoPE), so a transposed operand, a wrong pairing or a dropped term in
either one shows up as a mismatch.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from speech_audio_encoder_b200 import synth

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


# ---------------------------------------------------------------- norms

def test_layer_norm_moments_and_constant_row():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((6, 1280)) * 3 + 2
    y = O.layer_norm(x, np.ones(1280), np.zeros(1280))
    assert np.allclose(y.mean(axis=1), 0, atol=1e-12)
    assert np.allclose(y.var(axis=1), 1 / (1 + 1e-5 / x.var(axis=1)), rtol=1e-12)
    beta = rng.standard_normal(1280)
    c = O.layer_norm(np.full((1, 1280), 7.0), rng.standard_normal(1280), beta)
    assert np.allclose(c[0], beta, atol=1e-12)


def test_layer_norm_matches_torch():
    rng = np.random.default_rng(2)
    x, g, b = rng.standard_normal((5, 64)), rng.standard_normal(64), rng.standard_normal(64)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (64,), torch.from_numpy(g),
                                         torch.from_numpy(b), eps=1e-5).numpy()
    assert np.allclose(O.layer_norm(x, g, b), ref, rtol=1e-12, atol=1e-12)


def test_rms_norm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 10, 128)) * 5
    y = O.rms_norm(x, np.ones(128))
    assert np.allclose(np.sqrt((y * y).mean(axis=-1)), 1.0, atol=1e-6)
    assert np.allclose(O.rms_norm(3.0 * x, np.ones(128)), y, atol=1e-6)
    g = rng.standard_normal(128)
    assert np.allclose(O.rms_norm(x, g), y * g, rtol=1e-12)


# ---------------------------------------------------------------- RoPE

def test_rope_identity_at_position_zero_and_norm():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 5, 128))
    r = O.rope(x, np.arange(5))
    assert np.array_equal(r[:, 0], x[:, 0])
    assert np.allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)


def test_rope_relative_position():
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal(128), rng.standard_normal(128)

    def dot(m, n):
        return float(O.rope(q[None], np.array([m]))[0] @ O.rope(k[None], np.array([n]))[0])

    for m, n, s in [(3, 10, 7), (0, 44998, 123), (1000, 20, 5000)]:
        assert dot(m, n) == pytest.approx(dot(m + s, n + s), rel=1e-9, abs=1e-9)


def test_rope_complex_formulation():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((7, 128))
    pos = np.array([0, 1, 2, 100, 7499, 30000, 44998])
    r = O.rope(x, pos)
    for t in range(7):
        for i in (0, 1, 31, 63):
            theta = 10000.0 ** (-2.0 * i / 128)
            z = complex(x[t, i], x[t, i + 64]) * complex(math.cos(pos[t] * theta), math.sin(pos[t] * theta))
            assert r[t, i] == pytest.approx(z.real, abs=1e-9)
            assert r[t, i + 64] == pytest.approx(z.imag, abs=1e-9)


# ---------------------------------------------------------------- attention and GELU

def test_attention_rows_sum_to_one_and_special_cases():
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((2, 9, 16)) for _ in range(3))
    P = O.attention_probs(q[0], k[0])
    assert np.allclose(P.sum(axis=1), 1.0, atol=1e-14)
    # one position: output is that value row
    assert np.allclose(O.attention(q[:, :1], k[:, :1], v[:, :1]), v[:, :1], atol=1e-15)
    # identical keys: uniform weights, output is the mean value row
    kk = np.repeat(k[:, :1], 9, axis=1)
    assert np.allclose(O.attention(q, kk, v), np.repeat(v.mean(axis=1, keepdims=True), 9, axis=1), atol=1e-12)
    # one dominant logit selects its value row
    kd = k.copy()
    kd[:, 4] = 1e3 * q[:, 0]
    out = O.attention(q[:, :1], kd, v)
    assert np.allclose(out[:, 0], v[:, 4], atol=1e-9)


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((3, 17, 128)) for _ in range(3))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0].numpy()
    assert np.allclose(O.attention(q, k, v, chunk=5), ref, rtol=1e-10, atol=1e-12)


def test_gelu_identities_and_torch():
    x = np.linspace(-8, 8, 101)
    g = O.gelu(x)
    assert O.gelu(np.array([0.0]))[0] == 0.0
    assert np.allclose(g - O.gelu(-x), x, atol=1e-14)
    assert O.gelu(np.array([40.0]))[0] == pytest.approx(40.0, abs=1e-12)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="none").numpy()
    assert np.allclose(g, ref, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- parameter count

def test_param_count_two_matrix_ffn():
    n = O.param_count(32)
    target = GOLDEN["asr_params_approx"]["value"]
    assert n == 631_000_832
    assert abs(n - target) / target < 0.06
    # a gated (three-matrix) FFN would be far from "roughly 600M"
    gated = n + 32 * 1280 * 5120
    assert abs(gated - target) / target > 0.3


def test_chunk_pair_ratio():
    c = GOLDEN["chunk_attention"]
    T, w = c["T"], c["w"]
    assert (T * T) / ((T // w) * w * w) == pytest.approx(c["ratio"])


# ---------------------------------------------------------------- whole layer, width 16

def _naive_layer(x, lw, H, hd):
    """Second formulation: per-element loops, explicit exp sums, complex RoPE."""
    T, W = len(x), len(x[0])
    Fd = len(lw["w1"])

    def ln(row, g, b):
        mu = sum(row) / W
        var = sum((r - mu) ** 2 for r in row) / W
        return [(row[i] - mu) / math.sqrt(var + 1e-5) * g[i] + b[i] for i in range(W)]

    def lin(row, w, b):
        return [sum(row[i] * w[o][i] for i in range(len(row))) + b[o] for o in range(len(w))]

    h = [ln(x[t], lw["ln1_g"], lw["ln1_b"]) for t in range(T)]
    qkv = [lin(h[t], lw["w_qkv"], lw["b_qkv"]) for t in range(T)]
    half = hd // 2

    def head_vec(t, part, hh):
        base = part * W + hh * hd
        return qkv[t][base:base + hd]

    def norm_rope(vec, g, t):
        rms = math.sqrt(sum(a * a for a in vec) / hd + 1e-6)
        n = [vec[i] / rms * g[i] for i in range(hd)]
        out = [0.0] * hd
        for i in range(half):
            th = t * 10000.0 ** (-2.0 * i / hd)
            z = complex(n[i], n[i + half]) * complex(math.cos(th), math.sin(th))
            out[i], out[i + half] = z.real, z.imag
        return out

    o = [[0.0] * W for _ in range(T)]
    for hh in range(H):
        Q = [norm_rope(head_vec(t, 0, hh), lw["qn_g"], t) for t in range(T)]
        K = [norm_rope(head_vec(t, 1, hh), lw["kn_g"], t) for t in range(T)]
        V = [head_vec(t, 2, hh) for t in range(T)]
        for t in range(T):
            logits = [sum(Q[t][d] * K[s][d] for d in range(hd)) / math.sqrt(hd) for s in range(T)]
            mx = max(logits)
            e = [math.exp(a - mx) for a in logits]
            z = sum(e)
            for d in range(hd):
                o[t][hh * hd + d] = sum(e[s] * V[s][d] for s in range(T)) / z
    x1 = [[x[t][i] + v for i, v in enumerate(lin(o[t], lw["w_o"], lw["b_o"]))] for t in range(T)]
    out = []
    for t in range(T):
        h2 = ln(x1[t], lw["ln2_g"], lw["ln2_b"])
        u = [0.5 * a * (1 + math.erf(a / math.sqrt(2))) for a in lin(h2, lw["w1"], lw["b1"])]
        assert len(u) == Fd
        out.append([x1[t][i] + v for i, v in enumerate(lin(u, lw["w2"], lw["b2"]))])
    return out


@pytest.mark.parametrize("T", [1, 2, 5])
def test_width16_layer_brute_force(T):
    dims = O.EncoderDims(width=16, heads=2, head_dim=8, ffn=64, stack_in=32)
    w = synth.weights_f32(synth.make_weights(1, seed=77 + T, width=16, ffn=64, head_dim=8,
                                             stack_in=32, std=0.3, gain_std=0.3))
    lw = {k: np.asarray(v, np.float64) for k, v in w["layers"][0].items()}
    rng = np.random.default_rng(T)
    x = rng.standard_normal((T, 16))
    got = O.encoder_layer(x, lw, dims)
    ref = np.array(_naive_layer(x.tolist(), {k: v.tolist() for k, v in lw.items()}, 2, 8))
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)
    rows = np.array([T - 1, 0])
    assert np.allclose(O.encoder_layer_rows(x, lw, rows, dims), got[rows], rtol=1e-12, atol=1e-12)


def test_encoder_forward_zero_layers_is_final_ln():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((3, 1280))
    w = {"lnf_g": rng.standard_normal(1280), "lnf_b": rng.standard_normal(1280), "layers": []}
    assert np.allclose(O.encoder_forward(x, w, 0), O.layer_norm(x, w["lnf_g"], w["lnf_b"]))


# ---------------------------------------------------------------- synthetic inputs

def test_bf16_rounding_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.14159, 1e-20], np.float64)
    bits = synth.bf16_bits(vals)
    ref = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)


def test_workload_shapes():
    wl = synth.WORKLOADS
    assert O.position_count(wl["tones_1s"].n_samples) == 12
    assert O.position_count(wl["clip_30s"].n_samples) == 374
    assert O.position_count(wl["batch16_60s"].n_samples) == 749
    assert O.position_count(wl["rec_10min"].n_samples) == 7499
    assert O.position_count(wl["rec_1h"].n_samples) == 44999
    a = synth.WORKLOADS["tones_1s"].audio()
    assert a.shape == (1, 16000) and a.dtype == np.float32


# ---------------------------------------------------------------- chunked encoder

def test_chunk_bounds():
    assert O.chunk_bounds(10, 4) == [(0, 4), (4, 8), (8, 10)]
    assert O.chunk_bounds(10, 0) == [(0, 10)] and O.chunk_bounds(10, 10) == [(0, 10)]
    assert O.chunk_bounds(44999, 375)[-1] == (44625, 44999) and len(O.chunk_bounds(44999, 375)) == 120


def _small_layer(seed):
    dims = O.EncoderDims(width=16, heads=2, head_dim=8, ffn=64, stack_in=32)
    w = synth.weights_f32(synth.make_weights(1, seed=seed, width=16, ffn=64, head_dim=8,
                                             stack_in=32, std=0.3, gain_std=0.3))
    return dims, {k: np.asarray(v, np.float64) for k, v in w["layers"][0].items()}


def test_chunk_equal_to_length_is_the_full_layer():
    dims, lw = _small_layer(5)
    x = np.random.default_rng(0).standard_normal((9, 16))
    full = O.encoder_layer(x, lw, dims)
    assert np.array_equal(O.encoder_layer_chunked(x, lw, 9, dims), full)
    assert np.array_equal(O.encoder_layer_chunked(x, lw, 50, dims), full)


def test_chunk_of_one_attends_to_itself():
    """With one position per chunk the softmax has one key: the attention output is v, and
    RoPE (position 0) is the identity."""
    dims, lw = _small_layer(6)
    x = np.random.default_rng(1).standard_normal((5, 16))
    got = O.encoder_layer_chunked(x, lw, 1, dims)
    h = O.layer_norm(x, lw["ln1_g"], lw["ln1_b"])
    v = O.linear(h, lw["w_qkv"], lw["b_qkv"])[:, 32:]
    x1 = x + O.linear(v, lw["w_o"], lw["b_o"])
    ref = x1 + O.linear(O.gelu(O.linear(O.layer_norm(x1, lw["ln2_g"], lw["ln2_b"]), lw["w1"], lw["b1"])),
                        lw["w2"], lw["b2"])
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_chunks_are_independent_and_shift_invariant():
    """A chunk's output depends only on its own positions (re-indexed from 0)."""
    dims, lw = _small_layer(7)
    x = np.random.default_rng(2).standard_normal((11, 16))
    got = O.encoder_layer_chunked(x, lw, 4, dims)
    assert np.allclose(got[4:8], O.encoder_layer(x[4:8], lw, dims), rtol=1e-12, atol=1e-12)
    y = x.copy()
    y[:4] += 1.0  # change the first chunk only
    assert np.array_equal(O.encoder_layer_chunked(y, lw, 4, dims)[4:], got[4:])
    rows = np.array([0, 3, 4, 10])
    assert np.allclose(O.encoder_layer_rows_chunked(x, lw, rows, 4, dims), got[rows], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- speaker fusion and connector

def test_speaker_kernel_closed_forms():
    K = O.speaker_kernel()
    assert K.shape == (8, 1280)
    assert np.array_equal(K[0, 0::2], np.zeros(640)) and np.array_equal(K[0, 1::2], np.ones(640))
    assert np.allclose(K[:, 0::2] ** 2 + K[:, 1::2] ** 2, 1.0, atol=1e-15)
    for s_ in (1, 3, 7):
        assert K[s_, 0] == pytest.approx(math.sin(s_)) and K[s_, 1] == pytest.approx(math.cos(s_))
        i = 300
        w = 10000.0 ** (-2.0 * i / 1280)
        assert K[s_, 2 * i] == pytest.approx(math.sin(s_ * w)) and K[s_, 2 * i + 1] == pytest.approx(math.cos(s_ * w))


def test_speaker_fuse_brute_force_and_special_cases():
    rng = np.random.default_rng(3)
    H = rng.standard_normal((6, 1280))
    P = rng.uniform(0, 1, (6, 8))
    P[0] = 0.5  # exactly at the threshold: inactive (strict)
    g, b = 1 + 0.1 * rng.standard_normal(8), 0.1 * rng.standard_normal(8)
    got = O.speaker_fuse(H, P, g, b)
    for t in range(6):
        a = [1.0 if P[t, s_] > 0.5 else 0.0 for s_ in range(8)]
        mu = sum(a) / 8
        var = sum((v - mu) ** 2 for v in a) / 8
        ah = [(a[s_] - mu) / math.sqrt(var + 1e-5) * g[s_] + b[s_] for s_ in range(8)]
        for c in (0, 1, 2, 639, 1278, 1279):
            i = c // 2
            w = 10000.0 ** (-2.0 * i / 1280)
            k = [math.sin(s_ * w) if c % 2 == 0 else math.cos(s_ * w) for s_ in range(8)]
            assert got[t, c] == pytest.approx(H[t, c] + sum(ah[s_] * k[s_] for s_ in range(8)), abs=1e-12)
    # no active slot (or all active): LayerNorm of a constant is beta, so H + beta K
    K = O.speaker_kernel()
    assert np.allclose(O.speaker_fuse(H, np.zeros((6, 8)), g, b), H + b @ K, atol=1e-12)
    assert np.allclose(O.speaker_fuse(H, np.ones((6, 8)), g, b), H + b @ K, atol=1e-12)


def test_connector_is_a_linear_map_to_the_language_width():
    rng = np.random.default_rng(4)
    x, W, b = rng.standard_normal((3, 1280)), rng.standard_normal((2688, 1280)), rng.standard_normal(2688)
    y = O.connector(x, W, b)
    assert y.shape == (3, O.LLM_WIDTH)
    assert np.allclose(y[1, 7], sum(x[1, i] * W[7, i] for i in range(1280)) + b[7])
