"""GPU parity of the serving windows (sal_encoder_forward_ex with window_core /
window_context) against the oracle's windowed encoder.

Page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset Audits", section "Local
encoder windows, recording-wide language context", the paragraph on the serving path:
context-extended windows are encoded, the overlap outputs discarded and the core outputs
concatenated; 500 core and 50 context positions by default.

The oracle takes the GPU's own residual stream x0 (upcast), so the front end is not part
of the comparison. Bars as for the whole-clip encoder: embeddings within rel-L2 2e-2; the
residual stream's update x - x0 (core rows, from the window that owns each row) within
1e-2 after one or two layers and 2e-2 after 32. Rows at window borders (the last core row of one window and the first of the next)
are also checked on their own.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import rel_l2, to64, weights
from speech_audio_encoder_b200 import synth

pytestmark = pytest.mark.gpu

EMB_TOL = 2e-2


def _api():
    from speech_audio_encoder_b200 import api
    return api


def _oracle_windowed_stream(x0, wf, n_layers, core, ctx):
    """(emb, residual stream) of the oracle's windowed encoder: per window, the layers on its
    positions, the final LayerNorm, and the core rows of both."""
    emb, xs = [], []
    for lo, c0, c1, hi in O.window_bounds(len(x0), core, ctx):
        x = x0[lo:hi]
        for i in range(n_layers):
            x = O.encoder_layer(x, wf["layers"][i])
        xs.append(x[c0 - lo:c1 - lo])
        emb.append(O.layer_norm(x, wf["lnf_g"], wf["lnf_b"])[c0 - lo:c1 - lo])
    return np.concatenate(emb), np.concatenate(xs)


def _border_rows(T, core):
    rows = []
    for c in range(core, T, core):
        rows += [c - 1, c]
    return np.array(rows, dtype=np.int64)


def _check(batch, T, n_layers, core, ctx, x0=None, seed=0):
    api = _api()
    _, wf, dw = weights(32)
    if x0 is None:
        x0 = np.random.default_rng(seed).standard_normal((batch * T, 1280)).astype(np.float32)
    x = torch.from_numpy(np.ascontiguousarray(x0)).cuda()
    emb = api.sal_encoder_forward_ex(x, batch, T, dw, n_layers, window_core=core, window_context=ctx)
    assert api.sal_last_device_status() == 0
    got_e, got_x = to64(emb), to64(x)
    x_tol = 1e-2 if n_layers <= 2 else EMB_TOL  # the stream's update after many layers: the embedding bar
    for b in range(batch):
        xb = x0[b * T:(b + 1) * T].astype(np.float64)
        ref_e, ref_x = _oracle_windowed_stream(xb, wf, n_layers, core, ctx)
        ge, gx = got_e[b * T:(b + 1) * T], got_x[b * T:(b + 1) * T]
        assert rel_l2(ge, ref_e) < EMB_TOL
        assert rel_l2(gx - xb, ref_x - xb) < x_tol
        br = _border_rows(T, core)
        if len(br):
            assert rel_l2(ge[br], ref_e[br]) < EMB_TOL
            assert rel_l2(gx[br] - xb[br], ref_x[br] - xb[br]) < x_tol


@pytest.mark.parametrize("batch,T,core,ctx", [(1, 1234, 500, 50), (2, 300, 64, 16), (1, 200, 500, 50),
                                              (1, 1001, 500, 50), (1, 130, 40, 100)])
def test_windows_one_layer(batch, T, core, ctx):
    """Window counts 1 to 8, a last window of one core position (1,001), a context wider
    than the core (40 / 100), and a batch of two recordings."""
    _check(batch, T, 1, core, ctx, seed=T)


def test_windows_32_layers():
    _check(1, 1100, 32, 500, 50, seed=3)


def test_rec_10min_windows_two_layers():
    """The ten-minute recording (7,499 positions, 15 windows of the default geometry) from
    the GPU's own front end and projection, two layers, every row compared."""
    api = _api()
    wl = synth.WORKLOADS["rec_10min"]
    _, wf, dw = weights(32)
    wave = wl.audio()
    lm, st = api.sal_frontend(torch.from_numpy(wave).cuda())
    x0 = to64(api.sal_stack_project(st, dw)).astype(np.float32)
    _check(1, O.position_count(wl.n_samples), 2, 500, 50, x0=x0)


def test_windows_argument_checks():
    api = _api()
    import ctypes
    _, _, dw = weights(32)
    x = torch.empty((100, 1280), device="cuda")
    emb = torch.empty((100, 1280), dtype=torch.bfloat16, device="cuda")
    ws = api.encoder_workspace_ex(1, 100, window_core=50, window_context=10)
    lib = api.lib()
    rec = ctypes.byref(dw.record)
    both = api.sal_forward_options(20, None, 50, 10)   # chunks and windows together
    neg = api.sal_forward_options(0, None, 50, -1)     # negative context
    assert lib.sal_encoder_forward_ex(x.data_ptr(), 1, 100, rec, 1, emb.data_ptr(), ws.data_ptr(), ws.numel(), 0,
                                      ctypes.byref(both)) == 1
    assert lib.sal_encoder_forward_ex(x.data_ptr(), 1, 100, rec, 1, emb.data_ptr(), ws.data_ptr(), ws.numel(), 0,
                                      ctypes.byref(neg)) == 1
    ok = api.sal_forward_options(0, None, 50, 10)
    assert lib.sal_encoder_forward_ex(x.data_ptr(), 1, 100, rec, 1, emb.data_ptr(), ws.data_ptr(),
                                      ws.numel() - 256, 0, ctypes.byref(ok)) == 3
