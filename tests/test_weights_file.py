"""The flat weight file (include/sal.h, "Flat weight file"), without a GPU.

The seeded generator writes the file (synth.write_weight_file); these tests check that:
- reading it back gives every tensor bit for bit;
- the header's fields are the ones the format states;
- the library's header reader (sal_weights_file_info, host only) agrees on the layer
  count and the device size;
- the reader refuses every malformed file with the documented status.
The device load itself is tested on the GPU (test_gpu_weights_file.py).
"""
import ctypes
import os

import numpy as np
import pytest

from speech_audio_encoder_b200 import synth

SAL_OK, SAL_EINVAL, SAL_ESHAPE, SAL_EWORKSPACE, SAL_EIO = 0, 1, 2, 3, 7

# elements of the tensors, in file order (the sizes the format states)
GLOBAL_ELEMS = [1280 * 1024, 1280, 1280, 1280]
LAYER_ELEMS = [1280, 1280, 3840 * 1280, 3840, 128, 128, 1280 * 1280, 1280, 1280, 1280, 5120 * 1280, 5120,
               1280 * 5120, 1280]


def _pad(n):
    return -(-2 * n // 256) * 256


def _data_bytes(n_layers):
    return sum(_pad(n) for n in GLOBAL_ELEMS) + n_layers * sum(_pad(n) for n in LAYER_ELEMS)


@pytest.fixture(scope="module")
def api():
    from speech_audio_encoder_b200 import api as a
    from speech_audio_encoder_b200 import build
    build.build(quiet=True)
    return a


@pytest.fixture(scope="module")
def one_layer(tmp_path_factory):
    w = synth.make_weights(1, seed=4321)
    path = str(tmp_path_factory.mktemp("wf") / "enc1.salw")
    data = synth.write_weight_file(w, path)
    return w, path, data


def _info(api, path):
    n, b = ctypes.c_int(-1), ctypes.c_size_t(99)
    st = api.lib().sal_weights_file_info(os.fsencode(path), ctypes.byref(n), ctypes.byref(b))
    return st, n.value, b.value


def test_round_trip_bit_for_bit(one_layer):
    w, path, _ = one_layer
    r = synth.read_weight_file(path)
    for k in synth.WEIGHT_FILE_ORDER_GLOBAL:
        assert np.array_equal(r[k][0], w[k][0]) and r[k][0].shape == w[k][0].shape
    assert len(r["layers"]) == 1
    for k, v in w["layers"][0].items():
        assert np.array_equal(r["layers"][0][k][0], v[0]), k
        assert np.array_equal(r["layers"][0][k][1], v[1]), k


def test_header_and_length(one_layer):
    _, path, data = one_layer
    raw = np.fromfile(path, dtype=np.uint8)
    assert raw[:8].tobytes() == b"SALENCW1"
    f = raw[8:48].view("<u4")
    assert list(f) == [1, 256, 1, 1280, 10, 128, 5120, 1024, 1, 256]
    assert int(raw[48:56].view("<u8")[0]) == data == _data_bytes(1)
    assert raw.size == 256 + data
    assert not raw[56:256].any()
    # w_proj starts right after the header; b_proj on the next 256-byte boundary
    assert raw[256:258].view("<u2")[0] == synth.make_weights(0, seed=4321)["w_proj"][0].reshape(-1)[0]


def test_library_reads_the_header(api, one_layer):
    _, path, data = one_layer
    assert _info(api, path) == (SAL_OK, 1, data)


def test_zero_layers(api, tmp_path):
    w = synth.make_weights(0, seed=11)
    p = str(tmp_path / "enc0.salw")
    data = synth.write_weight_file(w, p)
    assert data == _data_bytes(0)
    assert _info(api, p) == (SAL_OK, 0, data)
    assert synth.read_weight_file(p)["layers"] == []


def _corrupt(src, dst, offset, payload):
    raw = bytearray(open(src, "rb").read())
    raw[offset:offset + len(payload)] = payload
    open(dst, "wb").write(raw)


@pytest.mark.parametrize("what,offset,payload,status", [
    ("magic", 0, b"SALENCW2", SAL_EINVAL),
    ("version", 8, (2).to_bytes(4, "little"), SAL_EINVAL),
    ("header size", 12, (128).to_bytes(4, "little"), SAL_EINVAL),
    ("dtype", 16, (2).to_bytes(4, "little"), SAL_EINVAL),
    ("width", 20, (1024).to_bytes(4, "little"), SAL_ESHAPE),
    ("heads", 24, (16).to_bytes(4, "little"), SAL_ESHAPE),
    ("ffn", 32, (4096).to_bytes(4, "little"), SAL_ESHAPE),
    ("layer count", 40, (2).to_bytes(4, "little"), SAL_EINVAL),
    ("alignment", 44, (128).to_bytes(4, "little"), SAL_EINVAL),
    ("data size", 48, (12345).to_bytes(8, "little"), SAL_EINVAL),
    ("reserved byte", 200, b"\x01", SAL_EINVAL),
])
def test_malformed_headers_are_refused(api, one_layer, tmp_path, what, offset, payload, status):
    _, path, _ = one_layer
    bad = str(tmp_path / "bad.salw")
    _corrupt(path, bad, offset, payload)
    assert _info(api, bad) == (status, 0, 0), what


def test_wrong_length_and_missing_file(api, one_layer, tmp_path):
    _, path, _ = one_layer
    raw = open(path, "rb").read()
    short = str(tmp_path / "short.salw")
    open(short, "wb").write(raw[:-256])
    assert _info(api, short) == (SAL_EINVAL, 0, 0)
    long_ = str(tmp_path / "long.salw")
    open(long_, "wb").write(raw + b"\0")
    assert _info(api, long_) == (SAL_EINVAL, 0, 0)
    tiny = str(tmp_path / "tiny.salw")
    open(tiny, "wb").write(raw[:100])
    assert _info(api, tiny) == (SAL_EINVAL, 0, 0)
    assert _info(api, str(tmp_path / "absent.salw")) == (SAL_EIO, 0, 0)


def test_load_argument_checks_before_any_cuda_call(api, one_layer):
    _, path, data = one_layer
    lib = api.lib()
    layers = (api.sal_layer * 1)()
    rec = api.sal_weights()
    p = os.fsencode(path)
    assert lib.sal_weights_file_load(None, 256, data, layers, 1, ctypes.byref(rec), None) == SAL_EINVAL
    assert lib.sal_weights_file_load(p, None, data, layers, 1, ctypes.byref(rec), None) == SAL_EINVAL
    assert lib.sal_weights_file_load(p, 256 + 16, data, layers, 1, ctypes.byref(rec), None) == SAL_EINVAL
    assert lib.sal_weights_file_load(p, 256, data, layers, 1, None, None) == SAL_EINVAL
    # too small a buffer or record array: refused after the header, before any copy
    assert lib.sal_weights_file_load(p, 256, data - 1, layers, 1, ctypes.byref(rec), None) == SAL_EWORKSPACE
    assert lib.sal_weights_file_load(p, 256, data, layers, 0, ctypes.byref(rec), None) == SAL_EWORKSPACE
