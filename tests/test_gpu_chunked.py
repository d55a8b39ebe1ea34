"""GPU parity of chunked attention (the training-time scheme of independent 30-second
post-feature chunks: no attention across a chunk border, RoPE positions restart in each
chunk) against the fp64 oracle, which encodes every chunk as its own sequence.

Tolerances as in the unchunked tests: attention rel-L2 < 1e-2 (bf16 P), the layer update
rel-L2 < 1e-2, sampled rows of a layer of the chunked one-hour encoder rel-L2 < 1e-2.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import rand_bf16, rel_l2, to64, weights
from speech_audio_encoder_b200 import synth

pytestmark = pytest.mark.gpu


def _api():
    from speech_audio_encoder_b200 import api
    return api


# (batch, T, chunk): chunk = 1 (a chunk per position), chunks not aligned to 128-row tiles,
# chunks aligned to tiles, the 30-second chunk of 375 positions; (8, 1000) and (1, 3000) run
# the two-tile kernel in pairs, (1, 4000) in 14 pairs and 4 split-mode tiles, (1, 749) with
# every tile in split mode (the warpgroups of a split tile take alternate key tiles of its
# chunks, with masked borders), the others the one-tile kernel.
@pytest.mark.parametrize("batch,T,chunk", [(1, 129, 1), (2, 383, 100), (1, 749, 128), (1, 749, 375),
                                           (8, 1000, 375), (1, 3000, 375), (1, 4000, 375), (1, 4000, 1000)])
def test_attention_chunked(batch, T, chunk):
    api = _api()
    q, q64 = rand_bf16((batch, 10, T, 128), 150 + T, 2.0)
    k, k64 = rand_bf16((batch, 10, T, 128), 160 + T, 1.0)
    v, v64 = rand_bf16((batch, 10, T, 128), 170 + T, 1.0)
    o = api.sal_attention_chunked(q, k, v, chunk)
    got = to64(o).reshape(batch, T, 10, 128)
    for b in range(batch):
        ref = np.concatenate([O.attention(q64[b][:, a:e], k64[b][:, a:e], v64[b][:, a:e]).transpose(1, 0, 2)
                              for a, e in O.chunk_bounds(T, chunk)])
        assert rel_l2(got[b], ref) < 1e-2


def test_chunk_of_whole_clip_is_full_attention():
    api = _api()
    q, _ = rand_bf16((1, 10, 300, 128), 1, 1.0)
    k, _ = rand_bf16((1, 10, 300, 128), 2, 1.0)
    v, _ = rand_bf16((1, 10, 300, 128), 3, 1.0)
    full = api.sal_attention(q, k, v)
    for chunk in (0, 300, 5000):
        assert torch.equal(api.sal_attention_chunked(q, k, v, chunk), full)


@pytest.mark.parametrize("batch,T,chunk", [(1, 383, 100), (2, 260, 128), (1, 300, 1)])
def test_chunked_layer(batch, T, chunk):
    api = _api()
    _, wf, dw = weights(2)
    rng = np.random.default_rng(T + chunk)
    x0 = rng.standard_normal((batch * T, 1280)).astype(np.float32)
    x = torch.from_numpy(x0).cuda()
    api.sal_encoder_forward_ex(x, batch, T, dw, 1, chunk=chunk)
    lw = {k: v.astype(np.float64) for k, v in wf["layers"][0].items()}
    for b in range(batch):
        xb = x0[b * T:(b + 1) * T].astype(np.float64)
        ref = O.encoder_layer_chunked(xb, lw, chunk)
        assert rel_l2(to64(x[b * T:(b + 1) * T]) - xb, ref - xb) < 1e-2


def test_rec_1h_chunked_teacher_forced():
    """The hour in 30-second chunks (375 positions): layer 31 at sampled rows, fed the GPU's
    own residual stream after 31 chunked layers."""
    api = _api()
    wl = synth.WORKLOADS["rec_1h"]
    _, wf, dw = weights(wl.n_layers)
    T = O.position_count(wl.n_samples)
    lm, st = api.sal_frontend(torch.from_numpy(wl.audio()).cuda())
    x = api.sal_stack_project(st, dw)
    ws = api.encoder_workspace(1, T)
    api.sal_encoder_forward_ex(x, 1, T, dw, 31, workspace=ws, chunk=375)
    x_in = to64(x)
    api.sal_encoder_forward_ex(x, 1, T, dw.sub(31, 1), 1, workspace=ws, chunk=375)
    x_out = to64(x)
    rows = np.array([0, 374, 375, 20000, 44624, 44625, 44998])  # chunk borders and the short last chunk
    lw = {k: v.astype(np.float64) for k, v in wf["layers"][31].items()}
    ref = O.encoder_layer_rows_chunked(x_in, lw, rows, 375)
    assert rel_l2(x_out[rows] - x_in[rows], ref - x_in[rows]) < 1e-2
