"""Bounded device waits: a wait that can never complete gives up, the kernel winds down
and returns, sal_last_device_status reports SAL_ETIMEOUT, and the next normal call is
correct.

The failure is made with the test hook sal_attention_withhold: every CTA's producer never
issues the loads of one key/value tile, so the consumer waits on a barrier that nothing
will complete. Nothing is in flight for that tile, so the wind-down (each CTA waits for
the loads and MMAs it did issue, then frees its tensor memory) ends at once. The wait
limit is 20 ms for the failing call and is restored afterwards.
"""
import time

import numpy as np
import pytest

import oracle as O
from gpu_util import rand_bf16, rel_l2, to64

pytestmark = pytest.mark.gpu

SAL_ETIMEOUT = 5
DEFAULT_LIMIT_NS = 4_000_000_000


@pytest.mark.parametrize("kernel", [1, 2])
def test_withheld_tile_times_out_and_the_next_call_is_correct(kernel):
    from speech_audio_encoder_b200 import api
    T = 512  # 4 key tiles per CTA; tile 2 is withheld after two have been used
    q, q64 = rand_bf16((1, 10, T, 128), 81, 1.0)
    k, k64 = rand_bf16((1, 10, T, 128), 82, 1.0)
    v, v64 = rand_bf16((1, 10, T, 128), 83, 1.0)
    assert api.sal_last_device_status() == 0
    api.sal_set_wait_limit_ns(20_000_000)
    try:
        t0 = time.perf_counter()
        api.sal_attention_withhold(q, k, v, kernel, 2)
        status = api.sal_last_device_status()
        elapsed = time.perf_counter() - t0
    finally:
        api.sal_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert status == SAL_ETIMEOUT
    # every CTA gave up at about the 20 ms limit (one wave), not at the 4 s default
    assert elapsed < 2.0, elapsed
    # reading the status cleared it
    assert api.sal_last_device_status() == 0
    # the context is usable and the same inputs give the right result
    o = api.sal_attention(q, k, v)
    assert api.sal_last_device_status() == 0
    ref = O.attention(q64[0], k64[0], v64[0]).transpose(1, 0, 2)
    assert rel_l2(to64(o).reshape(T, 10, 128), ref) < 1e-2


def test_withhold_beyond_the_last_tile_changes_nothing():
    """A withheld index past every CTA's key tiles never matches: the call completes and
    equals sal_attention bit for bit."""
    from speech_audio_encoder_b200 import api
    T = 300
    q, _ = rand_bf16((1, 10, T, 128), 84, 1.0)
    k, _ = rand_bf16((1, 10, T, 128), 85, 1.0)
    v, _ = rand_bf16((1, 10, T, 128), 86, 1.0)
    a = api.sal_attention_withhold(q, k, v, 1, 3)
    assert api.sal_last_device_status() == 0
    b = api.sal_attention(q, k, v)
    assert np.array_equal(to64(a), to64(b))


def test_one_and_two_tile_kernels_agree_bit_for_bit():
    """With no tile withheld (an index past every CTA's key tiles), the hook forces the
    one-tile kernel (1) or the two-tile kernel for every query-tile pair (2). At head dim 128
    both do the same per-row arithmetic in the same order, so their outputs are equal bit
    for bit; 1,000 positions give 8 query tiles (4 pairs) over 8 key tiles."""
    from speech_audio_encoder_b200 import api
    T = 1000
    q, _ = rand_bf16((1, 10, T, 128), 91, 1.0)
    k, _ = rand_bf16((1, 10, T, 128), 92, 1.0)
    v, _ = rand_bf16((1, 10, T, 128), 93, 1.0)
    one = to64(api.sal_attention_withhold(q, k, v, 1, 1000))
    two = to64(api.sal_attention_withhold(q, k, v, 2, 1000))
    assert api.sal_last_device_status() == 0
    assert np.array_equal(one, two)
