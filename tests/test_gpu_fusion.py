"""GPU parity of the steps after the encoder: speaker-activity fusion and the identity
connector (readings of the Dataset Audits page, its fusion equation being missing from the
text; see the oracle), against the fp64 oracle.

Tolerances: bf16 outputs within 2^-8 |ref| + 2e-3 rms(ref) (one bf16 rounding, fp32
arithmetic); the whole chain encoder -> fusion -> connector on the 1 s clip within the
2e-2 relative L2 bar of the embeddings.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import bf16_tensor, rand_bf16, rel_l2, to64, weights
from speech_audio_encoder_b200 import synth

pytestmark = pytest.mark.gpu


def _api():
    from speech_audio_encoder_b200 import api
    return api


def _close(got, ref):
    err = np.abs(got - ref)
    return bool((err <= 2.0 ** -8 * np.abs(ref) + 2e-3 * np.sqrt(np.mean(ref ** 2))).all())


@pytest.mark.parametrize("T", [1, 7, 749, 7499])
def test_speaker_fuse(T):
    api = _api()
    fw = synth.make_fusion_weights()
    H, H64 = rand_bf16((T, 1280), 200 + T, 1.0)
    P = synth.speaker_activity(T, T)
    g, b = bf16_tensor(fw["spk_g"][0]), bf16_tensor(fw["spk_b"][0])
    out = api.sal_speaker_fuse(H, torch.from_numpy(P).cuda(), g, b)
    ref = O.speaker_fuse(H64, P, fw["spk_g"][1], fw["spk_b"][1])
    assert _close(to64(out), ref)
    # in place (out aliases H)
    api.sal_speaker_fuse(H, torch.from_numpy(P).cuda(), g, b, out=H)
    assert torch.equal(H.view(torch.int16), out.view(torch.int16))


@pytest.mark.parametrize("M", [1, 374, 4100])
def test_connector(M):
    api = _api()
    fw = synth.make_fusion_weights()
    x, x64 = rand_bf16((M, 1280), 300 + M, 1.0)
    out = api.sal_connector(x, bf16_tensor(fw["w_conn"][0]), bf16_tensor(fw["b_conn"][0]))
    assert out.shape == (M, 2688)
    assert _close(to64(out), O.connector(x64, fw["w_conn"][1], fw["b_conn"][1]))


def test_encoder_fusion_connector_chain_tones_1s():
    api = _api()
    wl = synth.WORKLOADS["tones_1s"]
    _, wf, dw = weights(wl.n_layers)
    fw = synth.make_fusion_weights()
    wave = wl.audio()
    T = O.position_count(wl.n_samples)
    emb = api.sal_encode(torch.from_numpy(wave).cuda(), dw, wl.n_layers)[0]
    P = synth.speaker_activity(T, 9)
    fused = api.sal_speaker_fuse(emb, torch.from_numpy(P).cuda(), bf16_tensor(fw["spk_g"][0]),
                                 bf16_tensor(fw["spk_b"][0]))
    y = api.sal_connector(fused, bf16_tensor(fw["w_conn"][0]), bf16_tensor(fw["b_conn"][0]))
    H = O.encode(wave[0], wf, wl.n_layers)
    ref = O.connector(O.speaker_fuse(H, P, fw["spk_g"][1], fw["spk_b"][1]), fw["w_conn"][1], fw["b_conn"][1])
    assert rel_l2(to64(y), ref) < 2e-2
