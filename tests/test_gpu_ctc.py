"""GPU parity of the CTC timestamp adapter (page "Nemotron 3.5 Transcribe: From Recorded
Speech to Dataset Audits", section "Use alignment and audio questions as supporting
evidence") against the fp64 oracle.

Tolerances:
* attention with 16 heads of 64: rel-L2 < 1e-2 (bf16 P, as for the encoder's heads);
* log-softmax of fp32 scores: abs error < 2e-5 (fp32 sums over 23,863 terms);
* the whole adapter: rel-L2 < 2e-2 on row-centred log-probabilities (centring removes
  the log-sum-exp, so this measures the class scores; the bar of the encoder's output),
  and every row's probabilities sum to 1 within 1e-4.
Inputs: unfused states drawn N(0, 1) and rounded to bf16 (the encoder output is a
LayerNorm, of that scale), the same bits on both sides.
"""
import functools

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import rand_bf16, rel_l2, to64
from speech_audio_encoder_b200 import synth

pytestmark = pytest.mark.gpu


def _api():
    from speech_audio_encoder_b200 import api
    return api


@functools.lru_cache(maxsize=1)
def _weights():
    api = _api()
    w = synth.make_ctc_weights()
    cw = {k: v[1].astype(np.float64) for k, v in w.items() if k != "layers"}
    cw["layers"] = [{k: v[1].astype(np.float64) for k, v in lw.items()} for lw in w["layers"]]
    return cw, api.DeviceCtcWeights(w)


def _centred(a):
    return a - a.mean(axis=-1, keepdims=True)


@pytest.mark.parametrize("batch,T", [(1, 1), (1, 127), (2, 300), (1, 749), (2, 640), (1, 1100)])
def test_attention_16_heads_of_64(batch, T):
    """Query tiles go to the two-tile kernel in pairs: odd tile counts (1, 127, 300, 640,
    1,100 positions) leave the second tile of the last pair empty."""
    api = _api()
    q, q64 = rand_bf16((batch, 16, T, 64), 300 + T, 2.0)
    k, k64 = rand_bf16((batch, 16, T, 64), 310 + T, 1.0)
    v, v64 = rand_bf16((batch, 16, T, 64), 320 + T, 1.0)
    o = to64(api.sal_attention_heads(q, k, v)).reshape(batch, T, 16, 64)
    for b in range(batch):
        ref = O.attention(q64[b], k64[b], v64[b]).transpose(1, 0, 2)
        assert rel_l2(o[b], ref) < 1e-2


def test_head_width_128_matches_the_encoder_attention():
    api = _api()
    q, _ = rand_bf16((1, 10, 300, 128), 1, 1.0)
    k, _ = rand_bf16((1, 10, 300, 128), 2, 1.0)
    v, _ = rand_bf16((1, 10, 300, 128), 3, 1.0)
    assert torch.equal(api.sal_attention_heads(q, k, v).reshape(1, 300, 1280), api.sal_attention(q, k, v).reshape(1, 300, 1280))


@pytest.mark.parametrize("rows,n,ld", [(3, 23863, 23872), (5, 100, 100), (2, 1, 4)])
def test_log_softmax(rows, n, ld):
    api = _api()
    rng = np.random.default_rng(n)
    z = (rng.standard_normal((rows, ld)) * 4).astype(np.float32)
    got = api.sal_log_softmax(torch.from_numpy(z).cuda(), n).double().cpu().numpy()
    ref = O.log_softmax(z[:, :n].astype(np.float64))
    assert np.abs(got - ref).max() < 2e-5


@pytest.mark.parametrize("batch,T", [(1, 12), (1, 374), (2, 60), (1, 1500)])
def test_ctc_adapter(batch, T):
    api = _api()
    cw, dw = _weights()
    h, h64 = rand_bf16((batch * T, 1280), 400 + T, 1.0)
    logp = api.sal_ctc_adapter(h, batch, T, dw)
    got = to64(logp).reshape(batch, 2 * T, O.CTC.classes)
    assert np.isfinite(got).all()
    assert np.abs(np.exp(got).sum(axis=-1) - 1.0).max() < 1e-4
    for b in range(batch):
        ref = O.ctc_adapter(h64[b * T:(b + 1) * T], cw)
        assert rel_l2(_centred(got[b]), _centred(ref)) < 2e-2


def test_ctc_adapter_one_hour_properties():
    """The one-hour size (44,999 positions, 89,998 at 40 ms): every row is a finite,
    normalised distribution. The oracle cannot run 89,998 positions; parity is checked at
    the sizes above, with the same kernels."""
    api = _api()
    _, dw = _weights()
    T = 44999
    h, _ = rand_bf16((T, 1280), 999, 1.0)
    logp = api.sal_ctc_adapter(h, 1, T, dw)
    rows = torch.tensor([0, 1, 44998, 44999, 89996, 89997], device=logp.device)
    sel = logp[rows].double()
    assert torch.isfinite(sel).all()
    assert (sel.exp().sum(dim=-1) - 1.0).abs().max().item() < 1e-4
    assert torch.isfinite(logp).all().item()
