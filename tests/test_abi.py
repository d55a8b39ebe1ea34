"""The C-ABI library loads and exports every entry point include/sal.h declares.

Runs without a GPU: it only calls host-side functions (counts, workspace sizes, status
strings) and argument checks that return before any CUDA call.
"""
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


def test_counts_match_oracle(api):
    for n in list(range(0, 2000, 7)) + [480000, 960000, 9600000, 57600000]:
        assert api.frame_count(n) == O.frame_count(n)
        assert api.position_count(n) == O.position_count(n)


def test_status_strings(api):
    for s in range(7):
        assert api.status_string(s)
    assert "unknown" in api.status_string(99)


def test_workspace_sizes(api):
    lib = api.lib()
    assert lib.sal_encoder_workspace_bytes(0, 10) == 0
    w1 = lib.sal_encoder_workspace_bytes(1, 44999)
    w2 = lib.sal_encoder_workspace_bytes(2, 44999)
    # bf16 h + max(q, k, v, o; u) + RoPE table, 256-byte aligned
    assert w1 >= 44999 * (1280 * 2 + 5120 * 2) and w2 > w1
    assert lib.sal_encode_workspace_bytes(1, 480000) > lib.sal_encoder_workspace_bytes(1, 374)


def test_argument_checks_before_any_cuda_call(api):
    lib = api.lib()
    assert lib.sal_frontend(0, 1000, -1, 0, 0, 0) == 1          # negative batch
    assert lib.sal_frontend(0, 399, 1, 0, 0, 0) == 0            # no frame: nothing to do
    assert lib.sal_frontend(0, 57_616_000, 1, 0, 0, 0) == 2     # more than one hour
    assert lib.sal_linear(7, 0, 1, 64, 0, 64, 0, 0, 0) == 1     # unknown epilogue
    assert lib.sal_linear(0, 0, 0, 64, 0, 64, 0, 0, 0) == 0     # M = 0
    assert lib.sal_attention(0, 0, 0, 1, 45001, 0, 0) == 2
    assert lib.sal_attention(0, 0, 0, 1, 0, 0, 0) == 0
