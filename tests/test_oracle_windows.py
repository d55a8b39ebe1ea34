"""Pins for the oracle's serving windows (page "Nemotron 3.5 Transcribe: From Recorded
Speech to Dataset Audits", section "Local encoder windows, recording-wide language
context", the paragraph on the serving path: context-extended windows, overlap outputs
discarded, core outputs concatenated; 500 core and 50 context positions by default).

Pinned by brute force on the window geometry, by the two limits that reduce to other
pinned functions (one window is the whole-clip encoder; no context is the chunked
encoder with chunks of the core length), by locality (an output moves only with inputs
inside its own window) and, at width 16, by a composition of the per-element layer of the
width-16 brute force.
"""
import numpy as np
import pytest

import oracle as O
from speech_audio_encoder_b200 import synth
from test_oracle_encoder import _naive_layer


def _brute_windows(T, core, ctx):
    """Window of each position by enumeration: position p is in the core of window p // core;
    window w covers every position within ctx of its core, inside [0, T)."""
    out = []
    for w in range(-(-T // core) if T > 0 else 0):
        core_pos = [p for p in range(T) if p // core == w]
        cover = [p for p in range(T) if any(abs(p - c) <= ctx for c in core_pos)
                 and min(core_pos) - ctx <= p <= max(core_pos) + ctx]
        out.append((min(cover), min(core_pos), max(core_pos) + 1, max(cover) + 1))
    return out


@pytest.mark.parametrize("T", [0, 1, 49, 50, 499, 500, 501, 549, 550, 551, 1000, 1049, 1234])
def test_window_bounds_brute_force(T):
    assert O.window_bounds(T, 500, 50) == _brute_windows(T, 500, 50)


def test_window_bounds_defaults_and_hour():
    assert (O.WINDOW_CORE, O.WINDOW_CONTEXT) == (500, 50)
    b = O.window_bounds(44999)
    assert len(b) == 90
    assert b[0] == (0, 0, 500, 550) and b[1] == (450, 500, 1000, 1050)
    assert b[-1] == (44450, 44500, 44999, 44999)
    # the cores partition the clip in order
    assert [c0 for _, c0, _, _ in b] == list(range(0, 44999, 500))
    assert all(b[i][2] == b[i + 1][1] for i in range(len(b) - 1))
    # at most 50 positions of context on each side; exactly 50 away from the clip ends
    assert all(c0 - lo <= 50 and hi - c1 <= 50 for lo, c0, c1, hi in b)
    assert all(c0 - lo == 50 for lo, c0, _, _ in b[1:]) and all(hi - c1 == 50 for _, _, c1, hi in b[:-1])


def _small(seed, n_layers=2):
    dims = O.EncoderDims(width=16, heads=2, head_dim=8, ffn=64, stack_in=32)
    w = synth.weights_f32(synth.make_weights(n_layers, seed=seed, width=16, ffn=64, head_dim=8,
                                             stack_in=32, std=0.3, gain_std=0.3))
    w = {k: (np.asarray(v, np.float64) if k != "layers" else
             [{kk: np.asarray(vv, np.float64) for kk, vv in lw.items()} for lw in v]) for k, v in w.items()}
    return dims, w


def test_one_window_is_the_whole_clip_encoder():
    dims, w = _small(31)
    x = np.random.default_rng(0).standard_normal((13, 16))
    full = O.encoder_forward(x, w, 2, dims)
    assert np.array_equal(O.encoder_forward_windowed(x, w, 2, core=13, context=5, dims=dims), full)
    assert np.array_equal(O.encoder_forward_windowed(x, w, 2, core=100, context=0, dims=dims), full)


def test_no_context_is_the_chunked_encoder():
    dims, w = _small(32)
    x = np.random.default_rng(1).standard_normal((17, 16))
    got = O.encoder_forward_windowed(x, w, 2, core=5, context=0, dims=dims)
    assert np.allclose(got, O.encoder_forward_chunked(x, w, 2, 5, dims), rtol=1e-13, atol=1e-13)


def test_outputs_depend_only_on_their_window():
    dims, w = _small(33)
    T, core, ctx = 23, 6, 2
    x = np.random.default_rng(2).standard_normal((T, 16))
    base = O.encoder_forward_windowed(x, w, 2, core, ctx, dims)
    assert base.shape == (T, 16)
    bump = np.random.default_rng(9).standard_normal(16)  # not constant: LayerNorm removes a shift
    for lo, c0, c1, hi in O.window_bounds(T, core, ctx):
        for p in range(T):
            y = x.copy()
            y[p] += 0.5 * bump
            moved = np.abs(O.encoder_forward_windowed(y, w, 2, core, ctx, dims)[c0:c1] - base[c0:c1]).max()
            if lo <= p < hi:
                assert moved > 1e-6, (p, lo, hi)
            else:
                assert moved == 0.0, (p, lo, hi)


def test_width16_windows_brute_force():
    """Windows composed by hand from the per-element layer: slice each window, run two
    naive layers and the final LayerNorm written out, keep the core rows."""
    dims, w = _small(34)
    T, core, ctx = 11, 4, 1
    x = np.random.default_rng(3).standard_normal((T, 16))
    lws = [{k: v.tolist() for k, v in lw.items()} for lw in w["layers"]]
    rows = []
    for c0 in range(0, T, core):
        c1 = min(c0 + core, T)
        lo, hi = max(0, c0 - ctx), min(T, c1 + ctx)
        y = x[lo:hi].tolist()
        for lw in lws:
            y = _naive_layer(y, lw, 2, 8)
        for r in y[c0 - lo:c1 - lo]:
            mu = sum(r) / 16
            var = sum((a - mu) ** 2 for a in r) / 16
            rows.append([(r[i] - mu) / np.sqrt(var + 1e-5) * w["lnf_g"][i] + w["lnf_b"][i] for i in range(16)])
    got = O.encoder_forward_windowed(x, w, 2, core, ctx, dims)
    assert np.allclose(got, np.array(rows), rtol=1e-12, atol=1e-12)
