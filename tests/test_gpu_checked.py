"""The bounds-checked build (libsal_checked.so, include/sal.h "Bounds-checked build").

Every entry point runs once through libsal.so and once through libsal_checked.so on the
same inputs, with outputs and workspaces pre-filled with one byte pattern:
  * the checked build must refuse no access (every plain load and store of every kernel
    lies inside the ranges its launch declared), and
  * its outputs must equal the normal build's byte for byte (the checks change no
    arithmetic).
Shapes are ragged: T not a multiple of the 128-row tiles, a clip border inside a tile, an
odd number of query tiles (the two-tile attention kernel's split-mode CTAs), a serving
window shorter than the others. Whole encoder layers run at 1,793 rows or more (2,305 in
the CTC adapter, at width 1,024): below that the residual GEMMs split K, and the TMA
reduce-adds of the partial sums land in no fixed order, so not even two runs of the normal
build agree to the last bit.

Then the checker is shown to catch what it should: with the test hook
sal_check_shrink_writable, the declared output ranges end early, so the kernel's last
stores fall outside them. Those stores must be refused (not made: the bytes keep the
pattern), counted exactly, and reported at the lowest refused address with the file of
the kernel that made them; everything before the cut must match the normal build. No
access leaves the buffers the test allocated: a refused access goes to the library's
own sink.
"""
import ctypes

import pytest
import torch

from gpu_util import rand_bf16, weights
from speech_audio_encoder_b200 import synth

pytestmark = pytest.mark.gpu

PATTERN = 0x5A


def _api():
    from speech_audio_encoder_b200 import api
    return api


def _buf(nbytes: int) -> torch.Tensor:
    return torch.full((max(nbytes, 256),), PATTERN, dtype=torch.uint8, device="cuda")


def _both(run):
    """run(lib) -> list of uint8 device tensors. Returns (normal outputs, checked outputs,
    the checked build's report)."""
    api = _api()
    ref = [t.clone() for t in run(api.lib())]
    torch.cuda.synchronize()
    with api.checked_library() as lc:
        assert lc.sal_checked_build() == 1
        api.check_report()  # start from a clear report
        got = [t.clone() for t in run(lc)]
        rep = api.check_report()
    return ref, got, rep


def _assert_clean(ref, got, rep):
    assert rep["count"] == 0, rep
    for i, (a, b) in enumerate(zip(ref, got)):
        assert torch.equal(a, b), f"output {i} differs between the normal and the checked build"


@pytest.mark.parametrize("batch,n", [(1, 16_000), (2, 16_555)])
def test_front_end_and_projection(batch, n):
    api = _api()
    _, _, dw = weights(2)
    F, T = api.frame_count(n), api.position_count(n)
    wave = torch.randn((batch, n), device="cuda")

    def run(lib):
        lm, st, x = _buf(batch * F * 128 * 4), _buf(batch * T * 1024 * 2), _buf(batch * T * 1280 * 4)
        assert lib.sal_frontend(wave.data_ptr(), n, batch, lm.data_ptr(), st.data_ptr(), 0) == 0
        assert lib.sal_stack_project(st.data_ptr(), batch, T, ctypes.byref(dw.record), x.data_ptr(), 0) == 0
        return [lm, st, x]

    _assert_clean(*_both(run))


@pytest.mark.parametrize("batch,T,window,chunk", [(1, 1900, 0, 0), (2, 1000, 0, 0), (1, 1130, 500, 0),
                                                  (1, 1900, 0, 375)])
def test_encoder_forward(batch, T, window, chunk):
    api = _api()
    _, _, dw = weights(2)
    x0 = torch.randn((batch * T, 1280), device="cuda")

    def run(lib):
        x = _buf(batch * T * 1280 * 4)
        x[:batch * T * 1280 * 4].view(torch.float32).copy_(x0.reshape(-1))
        emb = _buf(batch * T * 1280 * 2)
        opts = api.sal_forward_options(chunk, None, window, 50 if window else 0)
        nws = lib.sal_encoder_workspace_bytes_ex(batch, T, ctypes.byref(opts))
        ws = _buf(nws)
        assert lib.sal_encoder_forward_ex(x.data_ptr(), batch, T, ctypes.byref(dw.record), 2, emb.data_ptr(),
                                          ws.data_ptr(), nws, 0, ctypes.byref(opts)) == 0
        return [x, emb]

    _assert_clean(*_both(run))


def test_encode_from_audio():
    api = _api()
    _, _, dw = weights(2)
    n = 1850 * 1280 + 555  # 1,850 positions
    wave = torch.randn((1, n), device="cuda")
    T = api.position_count(n)

    def run(lib):
        emb = _buf(T * 1280 * 2)
        nws = lib.sal_encode_workspace_bytes(1, n)
        ws = _buf(nws)
        assert lib.sal_encode(wave.data_ptr(), n, 1, ctypes.byref(dw.record), 2, emb.data_ptr(), ws.data_ptr(),
                              nws, 0) == 0
        return [emb]

    _assert_clean(*_both(run))


@pytest.mark.parametrize("batch,T,chunk", [(1, 129, 0), (1, 5000, 0), (3, 300, 0), (1, 4000, 1000)])
def test_attention(batch, T, chunk):
    q, _ = rand_bf16((batch, 10, T, 128), 1, 1.0)
    k, _ = rand_bf16((batch, 10, T, 128), 2, 1.0)
    v, _ = rand_bf16((batch, 10, T, 128), 3, 1.0)

    def run(lib):
        o = _buf(batch * T * 1280 * 2)
        if chunk:
            st = lib.sal_attention_chunked(q.data_ptr(), k.data_ptr(), v.data_ptr(), batch, T, chunk, o.data_ptr(), 0)
        else:
            st = lib.sal_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), batch, T, o.data_ptr(), 0)
        assert st == 0
        return [o]

    _assert_clean(*_both(run))


@pytest.mark.parametrize("M,K,N,epi", [(300, 1280, 5120, 2), (4100, 1280, 1280, 3), (129, 1024, 1280, 0),
                                       (1000, 1280, 3840, 1)])
def test_linear(M, K, N, epi):
    A, _ = rand_bf16((M, K), 4, 1.0)
    W, _ = rand_bf16((N, K), 5, 0.02)
    b, _ = rand_bf16((N,), 6, 0.02)

    def run(lib):
        out = _buf(M * N * (4 if epi in (0, 3) else 2))
        if epi == 3:
            out.zero_()
        assert lib.sal_linear(epi, A.data_ptr(), M, K, W.data_ptr(), N, b.data_ptr(), out.data_ptr(), 0) == 0
        return [out]

    _assert_clean(*_both(run))


def test_layernorm_and_qkv_heads():
    _, _, dw = weights(1)
    batch, T = 2, 300
    x = torch.randn((batch * T, 1280), device="cuda")
    h, _ = rand_bf16((batch * T, 1280), 7, 1.0)
    layer = dw.layer(0)

    def run(lib):
        y = _buf(batch * T * 1280 * 2)
        assert lib.sal_layernorm(x.data_ptr(), batch * T, layer.ln1_g, layer.ln1_b, y.data_ptr(), 0) == 0
        qkv = [_buf(batch * 10 * T * 128 * 2) for _ in range(3)]
        cs = _buf(2 * T * 64 * 4)
        assert lib.sal_qkv_rope(h.data_ptr(), batch, T, ctypes.byref(layer), qkv[0].data_ptr(), qkv[1].data_ptr(),
                                qkv[2].data_ptr(), cs.data_ptr(), 0) == 0
        na = [_buf(batch * 10 * T * 128 * 2) for _ in range(3)]
        assert lib.sal_qkv_rope_noalloc(h.data_ptr(), batch, T, ctypes.byref(layer), na[0].data_ptr(),
                                        na[1].data_ptr(), na[2].data_ptr(), 0) == 0
        return [y, *qkv, cs, *na]

    _assert_clean(*_both(run))


def test_fusion_connector_ctc():
    api = _api()
    rows = 301
    H, _ = rand_bf16((rows, 1280), 8, 1.0)
    P = torch.from_numpy(synth.speaker_activity(rows, 1)).cuda()
    g, _ = rand_bf16((8,), 9, 1.0)
    bb, _ = rand_bf16((8,), 10, 0.1)
    W, _ = rand_bf16((2688, 1280), 11, 0.02)
    cb, _ = rand_bf16((2688,), 12, 0.02)
    dcw = api.DeviceCtcWeights(synth.make_ctc_weights())
    T = 1200  # 2,400 rows at 40 ms
    h, _ = rand_bf16((T, 1280), 13, 1.0)

    def run(lib):
        fused, conn = _buf(rows * 1280 * 2), _buf(rows * 2688 * 2)
        assert lib.sal_speaker_fuse(H.data_ptr(), P.data_ptr(), rows, g.data_ptr(), bb.data_ptr(),
                                    fused.data_ptr(), 0) == 0
        assert lib.sal_connector(H.data_ptr(), rows, W.data_ptr(), cb.data_ptr(), conn.data_ptr(), 0) == 0
        logp = _buf(2 * T * api.CTC_CLASSES * 4)
        nws = lib.sal_ctc_workspace_bytes(1, T)
        ws = _buf(nws)
        assert lib.sal_ctc_adapter(h.data_ptr(), 1, T, ctypes.byref(dcw.record), logp.data_ptr(), ws.data_ptr(),
                                   nws, 0) == 0
        return [fused, conn, logp]

    _assert_clean(*_both(run))


# ----------------------------------------------------------------- the checker catches


def _shrunk(run, cut: int):
    """run(lib) through the checked build with every writable range `cut` bytes short;
    returns (its outputs, the report, sal_launch_count before the call)."""
    api = _api()
    with api.checked_library() as lc:
        api.check_report()
        lc.sal_check_shrink_writable(cut)
        try:
            before = lc.sal_launch_count()
            out = [t.clone() for t in run(lc)]
            rep = api.check_report()
        finally:
            lc.sal_check_shrink_writable(0)
    return out, rep, before


def test_refused_layernorm_stores():
    api = _api()
    _, _, dw = weights(1)
    rows = 37
    x = torch.randn((rows, 1280), device="cuda")
    layer = dw.layer(0)
    bufs = {}

    def run(lib):
        y = _buf(rows * 1280 * 2)
        bufs["y"] = y
        assert lib.sal_layernorm(x.data_ptr(), rows, layer.ln1_g, layer.ln1_b, y.data_ptr(), 0) == 0
        return [y]

    (ref,) = [t.clone() for t in run(api.lib())]
    row_bytes = 1280 * 2
    (got,), rep, before = _shrunk(run, row_bytes)
    # the last row's 320 stores of 8 bytes (32 lanes x 10) are refused, nothing else
    assert rep["count"] == row_bytes // 8, rep
    assert rep["file"] == "rowops.cu"
    assert rep["first_address"] == bufs["y"].data_ptr() + (rows - 1) * row_bytes
    assert rep["first_launch"] == before
    cut = (rows - 1) * row_bytes
    assert torch.equal(got[:cut], ref[:cut])
    assert bool((got[cut:] == PATTERN).all())


def test_refused_attention_stores():
    api = _api()
    batch, T = 1, 5000  # 40 query tiles: pairs and split-mode CTAs in one launch
    q, _ = rand_bf16((batch, 10, T, 128), 21, 1.0)
    k, _ = rand_bf16((batch, 10, T, 128), 22, 1.0)
    v, _ = rand_bf16((batch, 10, T, 128), 23, 1.0)
    bufs = {}

    def run(lib):
        o = _buf(batch * T * 1280 * 2)
        bufs["o"] = o
        assert lib.sal_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), batch, T, o.data_ptr(), 0) == 0
        return [o]

    (ref,) = [t.clone() for t in run(api.lib())]
    row_bytes = 1280 * 2
    (got,), rep, before = _shrunk(run, row_bytes)
    # the last position's row: ten heads x 128 bf16, stored 16 bytes at a time
    assert rep["count"] == row_bytes // 16, rep
    assert rep["file"] == "attention.cu"
    assert rep["first_address"] == bufs["o"].data_ptr() + (T - 1) * row_bytes
    assert rep["first_launch"] == before
    cut = (T - 1) * row_bytes
    assert torch.equal(got[:cut], ref[:cut])
    assert bool((got[cut:] == PATTERN).all())


def test_refused_front_end_stores():
    api = _api()
    n = 16_555  # 101 frames, 12 positions: the stacked copy holds frames 0 .. 95
    F, T = api.frame_count(n), api.position_count(n)
    wave = torch.randn((1, n), device="cuda")
    bufs = {}

    def run(lib):
        lm, st = _buf(F * 128 * 4), _buf(T * 1024 * 2)
        bufs["lm"], bufs["st"] = lm, st
        assert lib.sal_frontend(wave.data_ptr(), n, 1, lm.data_ptr(), st.data_ptr(), 0) == 0
        return [lm, st]

    ref = [t.clone() for t in run(api.lib())]
    (lm, st), rep, before = _shrunk(run, 4)
    # the last log-mel value (4 bytes) and the last two stacked bf16 values
    assert rep["count"] == 3, rep
    assert rep["file"] == "frontend.cu"
    ends = {bufs["lm"].data_ptr() + F * 128 * 4 - 4, bufs["st"].data_ptr() + T * 1024 * 2 - 4}
    assert rep["first_address"] == min(ends)
    assert rep["first_launch"] == before
    nl, ns = F * 128 * 4 - 4, T * 1024 * 2 - 4
    assert torch.equal(lm[:nl], ref[0][:nl]) and bool((lm[nl:nl + 4] == PATTERN).all())
    assert torch.equal(st[:ns], ref[1][:ns]) and bool((st[ns:ns + 4] == PATTERN).all())
