"""sal_weights_file_load on the GPU: the flat weight file streamed into device memory.

- The device buffer it fills equals, byte for byte, the buffer the in-memory path builds
  from the same seeded weights (the file's data region is the device layout).
- An encoder forward with the loaded record gives the same bytes as one with the
  in-memory record. At 1,900 rows no GEMM splits K, so both runs are reproducible.
- Each pointer of the record lands at its tensor.
- A file larger than one staging buffer (two layers, ~80 MB) crosses several chunks.
- The load also runs on a non-default stream.
"""
import numpy as np
import pytest
import torch

from gpu_util import weights
from speech_audio_encoder_b200 import synth

pytestmark = pytest.mark.gpu


def _api():
    from speech_audio_encoder_b200 import api
    return api


@pytest.fixture(scope="module")
def weight_file(tmp_path_factory):
    w, _, dw = weights(2)
    path = str(tmp_path_factory.mktemp("wf") / "enc2.salw")
    data = synth.write_weight_file(w, path)
    return w, dw, path, data


def test_loaded_buffer_is_the_device_layout(weight_file):
    api = _api()
    w, dw, path, data = weight_file
    s = torch.cuda.Stream()
    loaded = api.DeviceWeights.from_file(path, stream=s)
    assert loaded.n_layers == 2 and loaded.record.n_layers == 2
    assert loaded.buffer.numel() == data
    ref = dw.buffer.view(torch.uint8)
    assert ref.numel() <= data
    assert torch.equal(loaded.buffer[:ref.numel()], ref)
    assert not bool(loaded.buffer[ref.numel():].any())  # padding after the last tensor
    # every pointer sits at the same offset as the in-memory record's
    base_l, base_r = loaded.buffer.data_ptr(), dw.buffer.data_ptr()
    for key, p in dw.ptr.items():
        assert loaded.ptr[key] - base_l == p - base_r, key


def test_record_points_at_each_tensor(weight_file):
    api = _api()
    w, _, path, _ = weight_file
    loaded = api.DeviceWeights.from_file(path)
    host = loaded.buffer.cpu().numpy()
    base = loaded.buffer.data_ptr()

    def at(ptr, n):
        off = ptr - base
        return host[off:off + 2 * n].view("<u2")

    for k in synth.WEIGHT_FILE_ORDER_GLOBAL:
        bits = w[k][0].reshape(-1)
        assert np.array_equal(at(getattr(loaded.record, k), bits.size), bits), k
    for i in range(2):
        for k, (bits, _) in w["layers"][i].items():
            assert np.array_equal(at(getattr(loaded.layer(i), k), bits.size), bits.reshape(-1)), (i, k)


def test_encoder_output_matches_in_memory_weights(weight_file):
    api = _api()
    _, dw, path, _ = weight_file
    loaded = api.DeviceWeights.from_file(path)
    batch, T = 1, 1900
    x0 = torch.randn((batch * T, 1280), device="cuda")
    outs = []
    for rec in (dw, loaded):
        x = x0.clone()
        outs.append(api.sal_encoder_forward(x, batch, T, rec, 2).clone())
        outs.append(x)
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))
    assert torch.equal(outs[1], outs[3])
