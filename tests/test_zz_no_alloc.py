"""sal_qkv_rope_noalloc: the QKV + QK-norm + RoPE step for callers that cannot allocate
device memory while it runs (a real-time or serving loop that must not stall or fail on
cudaMalloc, a host that forbids device allocations after start-up). Its rotation table
lives in a fixed array inside the library instead of a caller scratch buffer.

The test calls it through the C-ABI twice in a row (different inputs and lengths, so the
second call must fully replace the first call's table) and compares each result with the
scratch-buffer entry point sal_qkv_rope, within the bf16 tolerance the kernel tests use.
It lives in its own file so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import rand_bf16, to64, weights

pytestmark = pytest.mark.gpu


def _close(got, ref):
    err = np.abs(got - ref)
    tol = 2.0 ** -8 * np.abs(ref) + 2e-3 * float(np.sqrt(np.mean(ref ** 2)))
    return bool((err <= tol).all())


def test_qkv_rope_noalloc_matches_scratch_entry_point():
    from speech_audio_encoder_b200 import api
    lib = api.lib()
    _, _, dw = weights(1)
    layer = dw.layer(0)
    for call, (batch, T) in enumerate([(2, 300), (1, 4096)]):
        h, _ = rand_bf16((batch * T, 1280), 900 + call, 1.0)
        ref = api.sal_qkv_rope(h, batch, T, layer)
        out = [torch.empty((batch, 10, T, 128), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
        st = lib.sal_qkv_rope_noalloc(h.data_ptr(), batch, T, ctypes.byref(layer), out[0].data_ptr(),
                                      out[1].data_ptr(), out[2].data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0, api.status_string(st)
        torch.cuda.synchronize()
        for got, want in zip(out, ref):
            assert _close(to64(got), to64(want))


def test_qkv_rope_noalloc_rejects_long_clips():
    from speech_audio_encoder_b200 import api
    _, _, dw = weights(1)
    h = torch.empty((4097, 1280), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((1, 10, 4097, 128), dtype=torch.bfloat16, device="cuda")
    st = api.lib().sal_qkv_rope_noalloc(h.data_ptr(), 1, 4097, ctypes.byref(dw.layer(0)), q.data_ptr(),
                                        q.data_ptr(), q.data_ptr(), 0)
    assert st == 2  # SAL_ESHAPE: beyond the fixed array
