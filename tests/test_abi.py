"""The C-ABI library loads and exports every entry point include/sal.h declares.

Runs without a GPU: it only calls host-side functions (counts, workspace sizes, status
strings) and argument checks that return before any CUDA call.
"""
import ctypes
import os
import re

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "sal.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sal_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def api():
    from speech_audio_encoder_b200 import api as a
    from speech_audio_encoder_b200 import build
    build.build(quiet=True)
    return a


def test_every_declared_symbol_is_exported(api):
    names = _declared()
    assert len(names) >= 14
    lib = api.lib()
    for n in names:
        assert hasattr(lib, n), n
        assert n in api.EXPORTS, f"{n} has no binding"


def test_checked_build_exports_the_same_calls(api):
    """libsal_checked.so (the bounds-checked build) exports every declared call too, and
    each library says which build it is. Only host-side calls: no CUDA call is made."""
    import ctypes
    names = _declared()
    for n in ("sal_checked_build", "sal_check_report", "sal_check_shrink_writable"):
        assert n in names
    assert api.lib().sal_checked_build() == 0
    with api.checked_library() as lc:
        assert api.lib() is lc
        for n in names:
            assert hasattr(lc, n), n
        assert lc.sal_checked_build() == 1
        # argument checks return before any CUDA call in the checked build as well
        assert lc.sal_frontend(None, 16000, -1, None, None, None) == 1
        assert lc.sal_check_report(None, None, None, None, None) == 1
    assert api.lib().sal_checked_build() == 0
    # the normal build has no report: SAL_EINVAL, outputs zeroed
    c, a, s = ctypes.c_uint64(7), ctypes.c_uint64(7), ctypes.c_uint64(7)
    f, ln = ctypes.c_int(7), ctypes.c_int(7)
    st = api.lib().sal_check_report(ctypes.byref(c), ctypes.byref(a), ctypes.byref(f), ctypes.byref(ln),
                                    ctypes.byref(s))
    assert st == 1 and (c.value, a.value, f.value, ln.value, s.value) == (0, 0, 0, 0, 0)
    api.lib().sal_check_shrink_writable(0)  # no effect in the normal build


def test_counts_match_oracle(api):
    for n in list(range(0, 2000, 7)) + [480000, 960000, 9600000, 57600000]:
        assert api.frame_count(n) == O.frame_count(n)
        assert api.position_count(n) == O.position_count(n)


def test_status_strings(api):
    for s in range(8):
        assert api.status_string(s)
        assert "unknown" not in api.status_string(s)
    assert "unknown" in api.status_string(99)


def test_workspace_sizes(api):
    lib = api.lib()
    assert lib.sal_encoder_workspace_bytes(0, 10) == 0
    w1 = lib.sal_encoder_workspace_bytes(1, 44999)
    w2 = lib.sal_encoder_workspace_bytes(2, 44999)
    # bf16 h + max(q, k, v, o; u) + RoPE table, 256-byte aligned
    assert w1 >= 44999 * (1280 * 2 + 5120 * 2) and w2 > w1
    assert lib.sal_encode_workspace_bytes(1, 480000) > lib.sal_encoder_workspace_bytes(1, 374)


def test_windowed_workspace_sizes(api):
    """Serving windows: the windowed fp32 stream and bf16 embeddings over every window's
    slots, plus the encoder workspace of the windowed batch; no windows: the plain size."""
    lib = api.lib()
    plain = lib.sal_encoder_workspace_bytes(1, 44999)
    assert lib.sal_encoder_workspace_bytes_ex(1, 44999, None) == plain
    none = api.sal_forward_options(375, None, 0, 0)
    assert lib.sal_encoder_workspace_bytes_ex(1, 44999, ctypes.byref(none)) == plain
    o = api.sal_forward_options(0, None, 500, 50)
    rows = 90 * 600  # 90 windows, the longest 600 positions
    assert lib.sal_encoder_workspace_bytes_ex(1, 44999, ctypes.byref(o)) == (
        rows * 1280 * 6 + lib.sal_encoder_workspace_bytes(90, 600))
    assert lib.sal_encoder_workspace_bytes_ex(0, 44999, ctypes.byref(o)) == 0


def test_argument_checks_before_any_cuda_call(api):
    lib = api.lib()
    assert lib.sal_frontend(0, 1000, -1, 0, 0, 0) == 1          # negative batch
    assert lib.sal_frontend(0, 399, 1, 0, 0, 0) == 0            # no frame: nothing to do
    assert lib.sal_frontend(0, 57_616_000, 1, 0, 0, 0) == 2     # more than one hour
    assert lib.sal_linear(7, 0, 1, 64, 0, 64, 0, 0, 0) == 1     # unknown epilogue
    assert lib.sal_linear(0, 0, 0, 64, 0, 64, 0, 0, 0) == 0     # M = 0
    assert lib.sal_attention(0, 0, 0, 1, 45001, 0, 0) == 2
    assert lib.sal_attention(0, 0, 0, 1, 0, 0, 0) == 0


def test_ctc_adapter_host_checks(api):
    lib = api.lib()
    assert lib.sal_ctc_workspace_bytes(0, 10) == 0
    w1 = lib.sal_ctc_workspace_bytes(1, 374)
    # per 40 ms position at least: fp32 x, bf16 h/q/k/v/o, fp32 class scores over 23,872 columns
    assert w1 >= 748 * (1024 * 4 + 5 * 1024 * 2 + 23872 * 4)
    assert lib.sal_ctc_workspace_bytes(2, 374) > w1
    rec = api.sal_ctc_weights()
    assert lib.sal_ctc_adapter(0, -1, 10, ctypes.byref(rec), 0, 0, 0, 0) == 1      # negative batch
    assert lib.sal_ctc_adapter(0, 1, 45001, ctypes.byref(rec), 0, 0, 0, 0) == 2    # more than one hour
    assert lib.sal_ctc_adapter(0, 4096, 10, ctypes.byref(rec), 0, 0, 0, 0) == 2    # attention grid.y
    assert lib.sal_ctc_adapter(0, 0, 10, ctypes.byref(rec), 0, 0, 0, 0) == 0       # nothing to do
    assert lib.sal_ctc_adapter(0, 1, 10, ctypes.byref(rec), 0, 0, 0, 0) == 1       # null pointers
    assert lib.sal_attention_heads(0, 0, 0, 1, 10, 16, 96, 0, 0) == 2              # head width 96
    assert lib.sal_attention_heads(0, 0, 0, 1, 90001, 16, 64, 0, 0) == 2
    assert lib.sal_attention_heads(0, 0, 0, 1, 10, 16, 64, 0, 0) == 1
    assert lib.sal_log_softmax(0, 4, 10, 5, 0, 0) == 1                             # ld < n
    assert lib.sal_log_softmax(0, 0, 10, 10, 0, 0) == 0


def test_attention_plan_matches_the_stated_schedule(api):
    """The library's split of query tiles between the two attention kernels equals the
    rule its header states (list scheduling, written out in the GPU tests), over clip
    lengths and batch sizes on both sides of every threshold.

    SAL_ATTN_PP in the environment forces the split (the library reads it once per
    process), so the stated rule is only checked when it is unset."""
    if os.environ.get("SAL_ATTN_PP") or os.environ.get("SAL_ATTN_PAIRS"):
        pytest.skip("SAL_ATTN_PP / SAL_ATTN_PAIRS force the split in this process")
    from test_gpu_kernels import _pairs_for_two_tile_kernel
    cases = [(b, T) for b in (1, 2, 8, 16, 30) for T in (1, 129, 749, 1000, 2000, 2047, 2048, 3000)]
    cases += [(b, T) for b in (1, 2) for T in (5000, 7499, 12000, 20000, 44999)]
    for batch, T in cases:
        assert api.attention_plan(batch, T) == _pairs_for_two_tile_kernel(batch, T), (batch, T)
    assert api.attention_plan(1, 20000, heads=16, head_dim=64) == (78, 157)  # 64-wide heads: pairs + 1 split
    assert api.attention_plan(0, 100) == (0, 1)
    p, q = ctypes.c_int(), ctypes.c_int()
    assert api.lib().sal_attention_plan(1, 90001, 10, 128, 148, ctypes.byref(p), ctypes.byref(q)) == 2


def test_withhold_hook_argument_checks(api):
    lib = api.lib()
    assert lib.sal_attention_withhold(0, 0, 0, 1, 512, 3, 2, 0, 0) == 1    # no such kernel
    assert lib.sal_attention_withhold(0, 0, 0, 1, 512, 1, -1, 0, 0) == 1   # negative tile
    assert lib.sal_attention_withhold(0, 0, 0, 1, 45001, 1, 2, 0, 0) == 2  # more than one hour
    assert lib.sal_attention_withhold(0, 0, 0, 1, 0, 1, 2, 0, 0) == 0      # nothing to do
    assert lib.sal_attention_withhold(0, 0, 0, 1, 512, 1, 2, 0, 0) == 1    # null pointers
