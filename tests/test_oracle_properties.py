"""Property-based pins of the oracle (random shapes and values drawn by hypothesis): the
invariances the definitions imply, checked where a plausible slip (a wrong axis, a missing
max subtraction, a transposed operand) would break them."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle as O

SET = settings(max_examples=40, deadline=None)
seeds = st.integers(0, 2 ** 31 - 1)


@SET
@given(seeds, st.integers(1, 6), st.integers(1, 40), st.sampled_from([2, 4, 8, 16]))
def test_attention_is_invariant_to_a_joint_permutation_of_keys_and_values(seed, H, T, hd):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((H, T, hd)) * 2 for _ in range(3))
    perm = rng.permutation(T)
    assert np.allclose(O.attention(q, k, v), O.attention(q, k[:, perm], v[:, perm]), atol=1e-12)


@SET
@given(seeds, st.integers(1, 5), st.integers(2, 64), st.floats(-50, 50), st.floats(0.01, 100))
def test_layer_norm_is_invariant_to_shift_and_positive_scale(seed, rows, W, shift, scale):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, W)) + 0.5
    g, b = rng.standard_normal(W), rng.standard_normal(W)
    # eps = 0 makes the invariance exact (the epsilon only matters for near-constant rows)
    a = O.layer_norm(x, g, b, eps=0.0)
    assert np.allclose(O.layer_norm(x * scale + shift, g, b, eps=0.0), a, atol=1e-8)


@SET
@given(seeds, st.integers(1, 30), st.sampled_from([2, 8, 64, 128]), st.integers(0, 5000))
def test_rope_preserves_norms_and_depends_on_position_differences(seed, T, hd, offset):
    rng = np.random.default_rng(seed)
    q, k = rng.standard_normal((T, hd)), rng.standard_normal((T, hd))
    pos = np.arange(T)
    rq, rk = O.rope(q, pos), O.rope(k, pos)
    assert np.allclose(np.linalg.norm(rq, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-12)
    # shifting every position by the same offset leaves every q.k product unchanged
    sq, sk = O.rope(q, pos + offset), O.rope(k, pos + offset)
    assert np.allclose(rq @ rk.T, sq @ sk.T, atol=1e-9)


@SET
@given(seeds, st.integers(1, 4), st.integers(1, 300), st.floats(-1e3, 1e3))
def test_log_softmax_shift_invariance_and_normalisation(seed, rows, n, c):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((rows, n)) * 10
    a = O.log_softmax(z)
    assert np.allclose(O.log_softmax(z + c), a, atol=1e-9)
    assert np.allclose(np.exp(a).sum(axis=-1), 1.0, atol=1e-12)


@SET
@given(st.integers(0, 10000), st.integers(0, 600))
def test_chunk_bounds_partition_the_clip(T, chunk):
    bounds = O.chunk_bounds(T, chunk)
    covered = [t for a, b in bounds for t in range(a, b)]
    assert covered == list(range(T))
    if chunk > 0:
        assert all(b - a == chunk for a, b in bounds[:-1])
        assert all(0 < b - a <= chunk for a, b in bounds)


@SET
@given(seeds, st.integers(1, 12), st.integers(8, 40))
def test_speaker_fusion_depends_only_on_the_thresholded_activity(seed, T, W):
    rng = np.random.default_rng(seed)
    W -= W % 2
    H = rng.standard_normal((T, W))
    P = rng.uniform(0, 1, (T, 8))
    g, b = 1 + 0.1 * rng.standard_normal(8), 0.1 * rng.standard_normal(8)
    # moving activities without crossing 0.5 changes nothing
    Q = np.where(P > 0.5, np.maximum(P, 0.5 + 1e-9) + 0.4 * (1 - P), 0.5 * P)
    assert np.array_equal((P > 0.5), (Q > 0.5))
    assert np.allclose(O.speaker_fuse(H, P, g, b), O.speaker_fuse(H, Q, g, b), atol=1e-12)
