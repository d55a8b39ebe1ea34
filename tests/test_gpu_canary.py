"""Guard bands around every output and workspace: each entry point writes only inside the
buffers it is given.

Each buffer the library writes is carved out of a larger device allocation with 4 KiB of
guard bytes (0xA5) before and after it; after the call and a synchronisation the guards
must be unchanged. Shapes include ragged tails (T not a multiple of the 128-row tiles,
a last serving window shorter than the others) where an out-of-range store would land
just past the end of an output.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import rand_bf16, weights
from speech_audio_encoder_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """A device buffer of `nbytes` (256-byte aligned) between two guard bands."""

    def __init__(self, nbytes: int):
        self.nbytes = nbytes
        self.raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")

    def view(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        assert n <= self.nbytes
        return self.raw[GUARD:GUARD + n].view(dtype).view(shape)

    def ptr(self) -> int:
        return self.raw.data_ptr() + GUARD

    def intact(self) -> bool:
        torch.cuda.synchronize()
        head = self.raw[:GUARD].cpu().numpy()
        tail = self.raw[GUARD + self.nbytes:].cpu().numpy()
        return bool((head == PATTERN).all() and (tail == PATTERN).all())


def _api():
    from speech_audio_encoder_b200 import api
    return api


@pytest.mark.parametrize("batch,n", [(1, 16_000), (2, 16_555)])
def test_front_end_and_projection(batch, n):
    api = _api()
    _, _, dw = weights(2)
    F, T = api.frame_count(n), api.position_count(n)
    wave = torch.randn((batch, n), device="cuda")
    lm = Guarded(batch * F * 128 * 4)
    st = Guarded(batch * T * 1024 * 2)
    x = Guarded(batch * T * 1280 * 4)
    lib = api.lib()
    assert lib.sal_frontend(wave.data_ptr(), n, batch, lm.ptr(), st.ptr(), 0) == 0
    assert lib.sal_stack_project(st.ptr(), batch, T, ctypes.byref(dw.record), x.ptr(), 0) == 0
    assert lm.intact() and st.intact() and x.intact()


@pytest.mark.parametrize("batch,T,window", [(1, 300, 0), (2, 129, 0), (1, 1130, 500)])
def test_encoder_forward(batch, T, window):
    api = _api()
    _, _, dw = weights(2)
    x0 = torch.randn((batch * T, 1280), device="cuda")
    x = Guarded(batch * T * 1280 * 4)
    x.view((batch * T, 1280), torch.float32).copy_(x0)
    emb = Guarded(batch * T * 1280 * 2)
    opts = api.sal_forward_options(0, None, window, 50 if window else 0)
    nws = api.lib().sal_encoder_workspace_bytes_ex(batch, T, ctypes.byref(opts))
    ws = Guarded((nws + 255) // 256 * 256)
    st = api.lib().sal_encoder_forward_ex(x.ptr(), batch, T, ctypes.byref(dw.record), 2, emb.ptr(), ws.ptr(), nws,
                                          0, ctypes.byref(opts))
    assert st == 0
    assert api.sal_last_device_status() == 0
    assert x.intact() and emb.intact() and ws.intact()


@pytest.mark.parametrize("batch,T", [(1, 129), (1, 5000), (3, 300)])
def test_attention_output(batch, T):
    api = _api()
    q, _ = rand_bf16((batch, 10, T, 128), 1, 1.0)
    k, _ = rand_bf16((batch, 10, T, 128), 2, 1.0)
    v, _ = rand_bf16((batch, 10, T, 128), 3, 1.0)
    o = Guarded(batch * T * 1280 * 2)
    assert api.lib().sal_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), batch, T, o.ptr(), 0) == 0
    assert o.intact()


@pytest.mark.parametrize("M,K,N,epi", [(300, 1280, 5120, 2), (4100, 1280, 1280, 3), (129, 1024, 1280, 0),
                                       (1000, 1280, 3840, 1)])
def test_linear_outputs(M, K, N, epi):
    api = _api()
    A, _ = rand_bf16((M, K), 4, 1.0)
    W, _ = rand_bf16((N, K), 5, 0.02)
    b, _ = rand_bf16((N,), 6, 0.02)
    out = Guarded(M * N * (4 if epi in (0, 3) else 2))
    if epi == 3:
        out.view((M, N), torch.float32).zero_()
    assert api.lib().sal_linear(epi, A.data_ptr(), M, K, W.data_ptr(), N, b.data_ptr(), out.ptr(), 0) == 0
    assert out.intact()


def test_qkv_heads():
    api = _api()
    _, _, dw = weights(1)
    batch, T = 2, 300
    h, _ = rand_bf16((batch * T, 1280), 7, 1.0)
    bufs = [Guarded(batch * 10 * T * 128 * 2) for _ in range(3)]
    cs = Guarded(2 * T * 64 * 4)
    st = api.lib().sal_qkv_rope(h.data_ptr(), batch, T, ctypes.byref(dw.layer(0)), bufs[0].ptr(), bufs[1].ptr(),
                                bufs[2].ptr(), cs.ptr(), 0)
    assert st == 0
    assert all(b.intact() for b in bufs) and cs.intact()


def test_fusion_connector_ctc():
    api = _api()
    rows = 301
    H, _ = rand_bf16((rows, 1280), 8, 1.0)
    P = torch.from_numpy(synth.speaker_activity(rows, 1)).cuda()
    g, _ = rand_bf16((8,), 9, 1.0)
    bb, _ = rand_bf16((8,), 10, 0.1)
    fused = Guarded(rows * 1280 * 2)
    assert api.lib().sal_speaker_fuse(H.data_ptr(), P.data_ptr(), rows, g.data_ptr(), bb.data_ptr(), fused.ptr(),
                                      0) == 0
    W, _ = rand_bf16((2688, 1280), 11, 0.02)
    cb, _ = rand_bf16((2688,), 12, 0.02)
    conn = Guarded(rows * 2688 * 2)
    assert api.lib().sal_connector(H.data_ptr(), rows, W.data_ptr(), cb.data_ptr(), conn.ptr(), 0) == 0
    dcw = api.DeviceCtcWeights(synth.make_ctc_weights())
    T = 45
    h, _ = rand_bf16((T, 1280), 13, 1.0)
    logp = Guarded(2 * T * api.CTC_CLASSES * 4)
    nws = api.lib().sal_ctc_workspace_bytes(1, T)
    ws = Guarded((nws + 255) // 256 * 256)
    assert api.lib().sal_ctc_adapter(h.data_ptr(), 1, T, ctypes.byref(dcw.record), logp.ptr(), ws.ptr(), nws,
                                     0) == 0
    assert fused.intact() and conn.intact() and logp.intact() and ws.intact()
