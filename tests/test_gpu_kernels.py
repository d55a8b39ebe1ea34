"""GPU parity of the single-step entry points (LayerNorm, tensor-core linear layers with
each epilogue, QKV + QK-norm + RoPE, attention) against the fp64 oracle.

Inputs are bf16 values; the oracle takes the same values upcast to float64, so the only
differences are the kernels' fp32 accumulation and their final rounding. Tolerances,
from that arithmetic:
  * bf16 outputs: |err| <= 2^-8 |ref| + 2e-3 rms(ref)   (one bf16 rounding is <= 2^-9 |ref|;
    fp32 sums over K <= 5120 products add ~1e-6 relative)
  * fp32 outputs: |err| <= 1e-4 rms(ref) + 1e-5 |ref|
  * attention: P is rounded to bf16 before P V, so rel-L2 <= 1e-2 and every element
    within 2^-7 |ref| + 2e-2 rms(ref).
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import rand_bf16, rel_l2, to64, weights

pytestmark = pytest.mark.gpu


def _api():
    from speech_audio_encoder_b200 import api
    return api


def _rms(a):
    return float(np.sqrt(np.mean(np.square(a))))


def _assert_bf16_close(got, ref, what):
    err = np.abs(got - ref)
    tol = 2.0 ** -8 * np.abs(ref) + 2e-3 * _rms(ref)
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, max err {err.max()}"


def _assert_f32_close(got, ref, what):
    err = np.abs(got - ref)
    tol = 1e-4 * _rms(ref) + 1e-5 * np.abs(ref)
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, max err {err.max()}"


# ---------------------------------------------------------------- LayerNorm

@pytest.mark.parametrize("rows", [1, 7, 1000])
def test_layernorm(rows):
    api = _api()
    rng = np.random.default_rng(rows)
    x = (rng.standard_normal((rows, 1280)) * 2 + 0.5).astype(np.float32)
    g, g64 = rand_bf16((1280,), 1, 0.5)
    b, b64 = rand_bf16((1280,), 2, 0.5)
    y = api.sal_layernorm(torch.from_numpy(x).cuda(), g.data_ptr(), b.data_ptr())
    _assert_bf16_close(to64(y), O.layer_norm(x, g64, b64), "layernorm")


# ---------------------------------------------------------------- linear layers

SHAPES = [
    # M, K, N : small M (narrow tiles, split-K), ragged tails, and M large enough for 256-wide tiles
    (1, 1280, 1280), (127, 1024, 1280), (129, 1280, 3840), (300, 5120, 1280),
    (1000, 1280, 5120), (4100, 1280, 1280), (4100, 5120, 1280),
]


@pytest.mark.parametrize("M,K,N", SHAPES)
@pytest.mark.parametrize("epi", ["f32", "bf16", "gelu", "resid"])
def test_linear(M, K, N, epi):
    api = _api()
    A, A64 = rand_bf16((M, K), 10 + M, 1.0)
    W, W64 = rand_bf16((N, K), 20 + K, 0.02)
    bias, b64 = rand_bf16((N,), 30 + N, 0.02)
    ref = A64 @ W64.T + b64
    if epi == "f32":
        out = api.sal_linear(api.SAL_EPI_STORE_F32, A, W, bias)
        _assert_f32_close(to64(out), ref, "linear f32")
    elif epi == "bf16":
        out = api.sal_linear(api.SAL_EPI_STORE_BF16, A, W, bias)
        _assert_bf16_close(to64(out), ref, "linear bf16")
    elif epi == "gelu":
        out = api.sal_linear(api.SAL_EPI_GELU_BF16, A, W, bias)
        _assert_bf16_close(to64(out), O.gelu(ref), "linear gelu")
    else:
        rng = np.random.default_rng(M + N)
        x0 = rng.standard_normal((M, N)).astype(np.float32)
        x = torch.from_numpy(x0).cuda()
        api.sal_linear(api.SAL_EPI_RESID_F32, A, W, bias, out=x)
        got = to64(x)
        _assert_f32_close(got - x0, ref, "linear residual (update)")


def test_linear_rejects_bad_shapes():
    api = _api()
    A, _ = rand_bf16((4, 100), 1)
    W, _ = rand_bf16((64, 100), 2)
    bias, _ = rand_bf16((64,), 3)
    out = torch.empty((4, 64), device="cuda")
    st = api.lib().sal_linear(0, A.data_ptr(), 4, 100, W.data_ptr(), 64, bias.data_ptr(), out.data_ptr(), 0)
    assert st == 2  # K not a multiple of 64


# ---------------------------------------------------------------- QKV + QK-norm + RoPE

# (2, 700) and (1, 3000) fill the SMs with two-head (256-wide) tiles; (2, 700) also puts
# a clip boundary inside a tile.
@pytest.mark.parametrize("batch,T", [(1, 1), (2, 7), (1, 129), (3, 300), (2, 700), (1, 3000)])
def test_qkv_rope(batch, T):
    api = _api()
    w, wf, dw = weights(1)
    lw = {k: v.astype(np.float64) for k, v in wf["layers"][0].items()}
    h, h64 = rand_bf16((batch * T, 1280), 40 + T, 1.0)
    q, k, v = api.sal_qkv_rope(h, batch, T, dw.layer(0))
    qkv = O.linear(h64, lw["w_qkv"], lw["b_qkv"]).reshape(batch, T, 3, 10, 128)
    pos = np.arange(T)
    for b in range(batch):
        qr = O.rope(O.rms_norm(qkv[b, :, 0].transpose(1, 0, 2), lw["qn_g"]), pos)
        kr = O.rope(O.rms_norm(qkv[b, :, 1].transpose(1, 0, 2), lw["kn_g"]), pos)
        vr = qkv[b, :, 2].transpose(1, 0, 2)
        _assert_bf16_close(to64(q[b]), qr, "q")
        _assert_bf16_close(to64(k[b]), kr, "k")
        _assert_bf16_close(to64(v[b]), vr, "v")


# ---------------------------------------------------------------- attention

def _pairs_for_two_tile_kernel(batch, T, sms=148, rho=1.35):
    """Query-tile pairs per (clip, head) that the library gives the two-tile kernel (the
    remaining tiles go to split-mode CTAs of the same launch), 0 also when the one-tile
    kernel takes every tile: the choice among one-tile only, all pairs, no pairs and (from
    16 query tiles up) the largest counts of pairs filling whole waves whose greedy
    schedule ends first; at least 120 two-tile CTAs when there are pairs. The schedule
    places, for every (clip, head) in launch order, its pairs (rho one-tile CTAs each) and
    then its split tiles (0.74 + 1.09 / query tiles each); one-tile CTAs cost 1."""
    import heapq

    bh, n_qt = 10 * batch, -(-T // 128)
    sigma = 0.74 + 1.09 / n_qt

    def makespan(P):
        h = [0.0] * sms
        end = 0.0
        jobs = [(n_qt, 1.0)] if P < 0 else [(P, rho), (max(n_qt - 2 * P, 0), sigma)]
        for _ in range(bh):
            for n, c in jobs:
                for _ in range(n):
                    t = heapq.heappop(h) + c
                    heapq.heappush(h, t)
                    end = max(end, t)
        return end

    everything = (n_qt + 1) // 2
    cands = [everything, 0]
    if n_qt >= 16:  # shorter clips: one-tile, all pairs or every tile split
        cands += [w * sms // bh for w in range(1, everything * bh // sms + 1)]
    best, best_t = -1, makespan(-1)
    for P in cands:
        if P > 0 and P * bh < 120:
            continue
        t = makespan(P)
        if t < best_t - 1e-9:
            best, best_t = P, t
    return max(best, 0), n_qt


# The first five cases run the one-tile kernel; (1, 749) and (1, 2000) the two-tile kernel
# with every query tile in split mode (the keys split between its warpgroups); (30, 129),
# (8, 1000), (1, 3000) and (16, 749) the two-tile kernel in pairs only; (1, 4000) 14 pairs
# and 4 split-mode tiles. T = 129: a second query tile with one valid row and a last key
# tile with one valid column.
@pytest.mark.parametrize("batch,T,scale", [(1, 1, 1.0), (2, 7, 1.0), (1, 128, 1.0), (1, 129, 1.0),
                                           (2, 383, 1.0), (1, 749, 1.0), (1, 749, 8.0), (1, 2000, 3.0),
                                           (30, 129, 1.0), (8, 1000, 1.0), (1, 3000, 8.0), (16, 749, 1.0),
                                           (1, 4000, 2.0)])
def test_attention(batch, T, scale):
    api = _api()
    expect = {(30, 129): (1, 2), (1, 3000): (12, 24), (8, 1000): (4, 8), (16, 749): (3, 6), (1, 4000): (14, 32)}
    n_qt = -(-T // 128)
    assert api.attention_plan(batch, T) == expect.get((batch, T), (0, n_qt))
    q, q64 = rand_bf16((batch, 10, T, 128), 50 + T, scale)
    k, k64 = rand_bf16((batch, 10, T, 128), 60 + T, 1.0)
    v, v64 = rand_bf16((batch, 10, T, 128), 70 + T, 1.0)
    n0 = api.sal_launch_count()
    o = api.sal_attention(q, k, v)
    # one launch: the two-tile kernel (its pairs, then any split-mode tiles) or, with no
    # pairs, the one-tile kernel
    assert api.sal_launch_count() - n0 == 1
    got = to64(o).reshape(batch, T, 10, 128)
    for b in range(batch):
        ref = O.attention(q64[b], k64[b], v64[b]).transpose(1, 0, 2)
        assert rel_l2(got[b], ref) < 1e-2
        # Per element: each weight p_s enters the PV product rounded to bf16 (2^-9 relative),
        # the row sum uses the unrounded weights, and O is rounded to bf16 on output, so
        # |error| <= 2^-9 sum_s p_s |v_s| + 2^-8 |O| plus fp32 noise; checked with a factor 2
        # on the first term (sum_s p_s |v_s| is the oracle's attention over |v|).
        spv = O.attention(q64[b], k64[b], np.abs(v64[b])).transpose(1, 0, 2)
        err = np.abs(got[b] - ref)
        assert (err <= 2.0 ** -8 * (spv + np.abs(ref)) + 1e-5).all(), err.max()


def test_attention_dominant_key():
    """Sharp rows: one key aligned with each query selects its value row."""
    api = _api()
    T = 300
    rng = np.random.default_rng(9)
    qn = rng.standard_normal((1, 10, T, 128))
    kn = rng.standard_normal((1, 10, T, 128))
    perm = rng.permutation(T)
    kn[0][:, perm] = qn[0] * 4.0  # key perm[t] is 4 x query t
    from speech_audio_encoder_b200 import synth
    from gpu_util import bf16_tensor
    qb, kb = synth.bf16_bits(qn), synth.bf16_bits(kn)
    vb, v64 = rand_bf16((1, 10, T, 128), 11, 1.0)
    o = api.sal_attention(bf16_tensor(qb), bf16_tensor(kb), vb)
    ref = O.attention(synth.bf16_to_f32(qb)[0], synth.bf16_to_f32(kb)[0], v64[0]).transpose(1, 0, 2)
    got = to64(o).reshape(T, 10, 128)
    assert rel_l2(got, ref) < 1e-2
