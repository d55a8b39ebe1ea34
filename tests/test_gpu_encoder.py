"""GPU parity of the whole path (sal_stack_project, sal_encoder_forward, sal_encode)
against the fp64 oracle.

Bar: final embeddings within relative L2 2e-2 of the oracle (bf16 GEMM / attention
operands, fp32 accumulation and residual stream). The one-layer checks compare the
layer's update x1 - x0 (the part the kernels compute) at a tighter 1e-2.

For the long workloads (16 x 60 s, 10 minutes, one hour) the oracle cannot run 32 layers
over every position, so each check is teacher-forced: the GPU's residual stream after
layer l (fp32, upcast) is the oracle's input, and the oracle evaluates layer l only at
sampled positions (with keys and values from every position), which equals the same
rows of the full layer.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import rel_l2, to64, weights
from speech_audio_encoder_b200 import synth

pytestmark = pytest.mark.gpu

EMB_TOL = 2e-2


def _api():
    from speech_audio_encoder_b200 import api
    return api


def _layers64(wf, idx):
    return {k: v.astype(np.float64) for k, v in wf["layers"][idx].items()}


def _global64(wf):
    # float32 values of bf16 weights; the oracle upcasts each tensor to float64 exactly
    return wf


def test_stack_projection():
    api = _api()
    _, wf, dw = weights(2)
    wave = synth.WORKLOADS["tones_1s"].audio()
    lm, st = api.sal_frontend(torch.from_numpy(wave).cuda())
    x = api.sal_stack_project(st, dw)
    S = to64(st[0])  # the kernel's own bf16 stacked input
    ref = O.stack_project(S, _global64(wf))
    got = to64(x)
    assert np.abs(got - ref).max() <= 1e-4 * np.sqrt(np.mean(ref ** 2)) + 1e-5 * np.abs(ref).max()


@pytest.mark.parametrize("batch,T", [(1, 1), (2, 129), (1, 383)])
def test_one_layer(batch, T):
    api = _api()
    _, wf, dw = weights(2)
    rng = np.random.default_rng(T)
    x0 = rng.standard_normal((batch * T, 1280)).astype(np.float32)
    x = torch.from_numpy(x0).cuda()
    emb = api.sal_encoder_forward(x, batch, T, dw, 1)
    g = _global64(wf)
    for b in range(batch):
        xb = x0[b * T:(b + 1) * T].astype(np.float64)
        ref1 = O.encoder_layer(xb, g["layers"][0])
        got1 = to64(x[b * T:(b + 1) * T])
        assert rel_l2(got1 - xb, ref1 - xb) < 1e-2
        ref_emb = O.layer_norm(ref1, g["lnf_g"], g["lnf_b"])
        assert rel_l2(to64(emb[b * T:(b + 1) * T]), ref_emb) < 1e-2


def _bf16(a):
    return synth.bf16_to_f32(synth.bf16_bits(a)).astype(np.float64)


def _layer_bf16_operands(x, lw):
    """The oracle layer with every tensor-core operand rounded to bf16 where the GPU path
    rounds it (LN outputs, q / k / v after norm and RoPE, attention output, GELU output).
    What remains between this and the GPU is fp32 accumulation and the bf16 P."""
    T = x.shape[0]
    h = _bf16(O.layer_norm(x, lw["ln1_g"], lw["ln1_b"]))
    qkv = O.linear(h, lw["w_qkv"], lw["b_qkv"]).reshape(T, 3, 10, 128).transpose(1, 2, 0, 3)
    pos = np.arange(T)
    q = _bf16(O.rope(O.rms_norm(qkv[0], lw["qn_g"]), pos))
    k = _bf16(O.rope(O.rms_norm(qkv[1], lw["kn_g"]), pos))
    v = _bf16(qkv[2])
    o = _bf16(O.attention(q, k, v).transpose(1, 0, 2).reshape(T, 1280))
    x = x + O.linear(o, lw["w_o"], lw["b_o"])
    u = _bf16(O.gelu(O.linear(_bf16(O.layer_norm(x, lw["ln2_g"], lw["ln2_b"])), lw["w1"], lw["b1"])))
    return x + O.linear(u, lw["w2"], lw["b2"])


def test_sharp_attention_layer():
    """QK-norm gains of 8: logits with a standard deviation near 64, attention close to
    one-hot. Rounding q and k to bf16 (2^-9 relative) moves such logits by ~0.2, which
    reorders near-ties, so against the exact oracle the layer update is held to the
    embedding bar 2e-2 (rel-L2); against the oracle with the same bf16 operand roundings
    it is held to 1e-2."""
    api = _api()
    _, wf, dw = weights(1, seed=4242, qk_gain_scale=8.0)
    T = 300
    rng = np.random.default_rng(5)
    x0 = rng.standard_normal((T, 1280)).astype(np.float32)
    x = torch.from_numpy(x0).cuda()
    api.sal_encoder_forward(x, 1, T, dw, 1)
    lw = _layers64(wf, 0)
    got = to64(x) - x0
    exact = O.encoder_layer(x0.astype(np.float64), lw) - x0
    same_rounding = _layer_bf16_operands(x0.astype(np.float64), lw) - x0
    assert rel_l2(got, exact) < EMB_TOL
    assert rel_l2(got, same_rounding) < 1e-2


def test_tones_1s_end_to_end_host_buffers():
    """sal_encode with a pinned host waveform and a pinned host output."""
    api = _api()
    wl = synth.WORKLOADS["tones_1s"]
    _, wf, dw = weights(wl.n_layers)
    wave = torch.from_numpy(wl.audio()).pin_memory()
    T = O.position_count(wl.n_samples)
    emb = torch.empty((1, T, 1280), dtype=torch.bfloat16).pin_memory()
    api.sal_encode(wave, dw, wl.n_layers, emb=emb)
    torch.cuda.synchronize()
    ref = O.encode(wave.numpy()[0], _global64(wf), wl.n_layers)
    assert rel_l2(to64(emb[0]), ref) < EMB_TOL


def test_clip_30s_32_layers():
    api = _api()
    wl = synth.WORKLOADS["clip_30s"]
    _, wf, dw = weights(wl.n_layers)
    wave = wl.audio()
    emb = api.sal_encode(torch.from_numpy(wave).cuda(), dw, wl.n_layers)
    ref = O.encode(wave[0], _global64(wf), wl.n_layers)
    err = rel_l2(to64(emb[0]), ref)
    assert err < EMB_TOL, err


def _teacher_forced(name, layers, n_rows, seed):
    """Layers ``layers`` of workload ``name``, each teacher-forced: the GPU's residual
    stream before layer l (upcast) is the oracle's input, and the oracle's layer output on
    ``n_rows`` sampled positions of every clip (first and last included) is compared with
    the GPU's, as the update x_out - x_in at 1e-2 rel-L2. The embeddings the same call
    writes (the final LayerNorm of the GPU's stream after layer l) are compared on those
    rows with the final LayerNorm of the oracle's rows at the embedding bar 2e-2."""
    api = _api()
    wl = synth.WORKLOADS[name]
    _, wf, dw = weights(wl.n_layers)
    g = _global64(wf)
    wave = wl.audio()
    B, T = wl.batch, O.position_count(wl.n_samples)
    lm, st = api.sal_frontend(torch.from_numpy(wave).cuda())
    x = api.sal_stack_project(st, dw)
    ws = api.encoder_workspace(B, T)
    emb = torch.empty((B * T, 1280), dtype=torch.bfloat16, device="cuda")
    rng = np.random.default_rng(seed)
    done = 0  # layers applied to x so far
    for l in sorted(layers):
        if l > done:
            api.sal_encoder_forward(x, B, T, dw.sub(done, l - done), l - done, workspace=ws, emb=emb)
        x_in = to64(x)
        api.sal_encoder_forward(x, B, T, dw.sub(l, 1), 1, workspace=ws, emb=emb)
        done = l + 1
        x_out, e_out = to64(x), to64(emb)
        for b in range(B):
            rows = np.sort(rng.choice(np.arange(1, T - 1), size=min(n_rows, T) - 2, replace=False))
            rows = np.concatenate([[0], rows, [T - 1]])
            xin_b = x_in[b * T:(b + 1) * T]
            ref = O.encoder_layer_rows(xin_b, _layers64(wf, l), rows)
            got = x_out[b * T:(b + 1) * T][rows]
            err = rel_l2(got - xin_b[rows], ref - xin_b[rows])
            assert err < 1e-2, (name, l, b, err)
            e_err = rel_l2(e_out[b * T:(b + 1) * T][rows], O.layer_norm(ref, g["lnf_g"], g["lnf_b"]))
            assert e_err < EMB_TOL, (name, l, b, "embeddings", e_err)


def test_batch16_60s_teacher_forced():
    _teacher_forced("batch16_60s", [0, 15, 31], 256, 1)


def test_rec_10min_teacher_forced():
    _teacher_forced("rec_10min", [0, 15, 31], 256, 2)


def test_rec_1h_teacher_forced():
    _teacher_forced("rec_1h", [0, 15, 31], 256, 3)


def test_rec_10min_two_layers_end_to_end():
    """The whole path over ten minutes with two layers, against the oracle run end to end
    (front end, stacking, projection, layer 0 over every position, layer 1 and the final
    LayerNorm on 512 sampled positions including the first and the last). At one hour the
    oracle's full layer 0 takes minutes of host time; there the layers are teacher-forced."""
    api = _api()
    wl = synth.WORKLOADS["rec_10min"]
    _, wf, dw = weights(wl.n_layers)
    g = _global64(wf)
    wave = wl.audio()
    T = O.position_count(wl.n_samples)
    emb = api.sal_encode(torch.from_numpy(wave).cuda(), dw, 2)
    x1 = O.encoder_layer(O.stack_project(O.stack_frames(O.log_mel(wave[0])), g), g["layers"][0])
    rng = np.random.default_rng(11)
    rows = np.concatenate([[0], np.sort(rng.choice(np.arange(1, T - 1), size=510, replace=False)), [T - 1]])
    ref = O.layer_norm(O.encoder_layer_rows(x1, g["layers"][1], rows), g["lnf_g"], g["lnf_b"])
    err = rel_l2(to64(emb[0])[rows], ref)
    assert err < EMB_TOL, err


def test_encoder_rejects_bad_arguments():
    api = _api()
    _, _, dw = weights(2)
    lib = api.lib()
    import ctypes
    x = torch.empty((10, 1280), device="cuda")
    ws = api.encoder_workspace(1, 10)
    emb = torch.empty((10, 1280), dtype=torch.bfloat16, device="cuda")
    rec = ctypes.byref(dw.record)
    assert lib.sal_encoder_forward(x.data_ptr(), 1, 10, rec, 3, emb.data_ptr(), ws.data_ptr(), ws.numel(), 0) == 1
    assert lib.sal_encoder_forward(x.data_ptr(), 1, 10, rec, 1, emb.data_ptr(), ws.data_ptr(), 256, 0) == 3
    assert lib.sal_encoder_forward(x.data_ptr(), 1, 45001, rec, 1, emb.data_ptr(), ws.data_ptr(), ws.numel(), 0) == 2
