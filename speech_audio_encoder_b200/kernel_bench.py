"""Times one kernel of the path through the C-ABI on seeded random inputs.

    python -m speech_audio_encoder_b200.kernel_bench KIND [--batch B] [--T T] [--reps R]

KIND is one of frontend, stack_proj, layernorm, qkv, attention, out_proj, ffn_up, ffn_down,
speaker_fuse, connector, ctc (the whole CTC adapter), attention64 (its 16 heads of 64),
linear (any --N, --K, --epi).
Each repetition is one launch (qkv also launches the small RoPE-table kernel). The
repetitions are captured once as a CUDA graph and the replay is timed with CUDA events on
the launching stream after warm-up (eager launches from Python would measure the host). Prints one JSON line with the
average launch time and the achieved rate against the algorithmic flops or bytes. Small
cases of this command are what the committed ncu summaries capture.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import api, synth


def _bf16(shape, seed, std):
    bits, _ = synth.random_bf16(shape, seed, std)
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("kind")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--T", type=int, default=374)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--N", type=int, default=1280, help="linear: output width")
    ap.add_argument("--K", type=int, default=1280, help="linear: reduction length")
    ap.add_argument("--epi", type=int, default=1, help="linear: sal_epilogue value")
    a = ap.parse_args()
    B, T = a.batch, a.T
    M = B * T
    s = torch.cuda.current_stream()
    flops = bytes_ = 0.0
    if a.kind == "frontend":
        n = 160 * (8 * T - 1) + 400
        wave = torch.from_numpy(np.random.default_rng(0).standard_normal((B, n)).astype(np.float32)).cuda()
        F = api.frame_count(n)
        bytes_ = B * (4.0 * n + 512.0 * F + 256.0 * 8 * T)

        def run():
            api.sal_frontend(wave)
    elif a.kind == "layernorm":
        x = torch.randn((M, 1280), device="cuda")
        g, b = _bf16((1280,), 1, 1.0), _bf16((1280,), 2, 1.0)
        bytes_ = M * 1280 * 6.0

        def run():
            api.sal_layernorm(x, g.data_ptr(), b.data_ptr())
    elif a.kind in ("qkv",):
        w = synth.make_weights(1)
        dw = api.DeviceWeights(w)
        h = _bf16((M, 1280), 3, 1.0)
        flops = 2.0 * M * 1280 * 3840

        def run():
            api.sal_qkv_rope(h, B, T, dw.layer(0))
    elif a.kind == "attention":
        q, k, v = (_bf16((B, 10, T, 128), 10 + i, 1.0) for i in range(3))
        flops = 4.0 * T * T * 1280 * B

        def run():
            api.sal_attention(q, k, v)
    elif a.kind == "attention64":  # the CTC adapter's heads: 16 of width 64
        q, k, v = (_bf16((B, 16, T, 64), 20 + i, 1.0) for i in range(3))
        flops = 4.0 * T * T * 1024 * B

        def run():
            api.sal_attention_heads(q, k, v)
    elif a.kind == "speaker_fuse":
        H = _bf16((M, 1280), 7, 1.0)
        P = torch.from_numpy(synth.speaker_activity(M, 1)).cuda()
        g, b = _bf16((8,), 8, 1.0), _bf16((8,), 9, 0.1)
        out = torch.empty_like(H)
        bytes_ = M * (1280 * 2 * 2 + 8 * 4)

        def run():
            api.sal_speaker_fuse(H, P, g, b, out=out)
    elif a.kind == "connector":
        x = _bf16((M, 1280), 10, 1.0)
        W, bias = _bf16((2688, 1280), 11, 0.02), _bf16((2688,), 12, 0.02)
        flops = 2.0 * M * 2688 * 1280

        def run():
            api.sal_connector(x, W, bias)
    elif a.kind == "ctc":
        # the whole CTC timestamp adapter on B clips of T encoder positions (2T at 40 ms)
        dw = api.DeviceCtcWeights(synth.make_ctc_weights())
        h = _bf16((M, 1280), 13, 1.0)
        logp = torch.empty((2 * M, api.CTC_CLASSES), dtype=torch.float32, device="cuda")
        ws = api.ctc_workspace(B, T)
        M2, T2 = 2 * M, 2 * T
        flops = (2.0 * M * 1280 * 2048 + 2 * (2.0 * M2 * 1024 * (3072 + 1024 + 2 * 4096) + 4.0 * T2 * T2 * 1024 * B)
                 + 2.0 * M2 * 1024 * api.CTC_CLASSES)

        def run():
            api.sal_ctc_adapter(h, B, T, dw, logp=logp, workspace=ws)
    elif a.kind == "linear":
        K, N, epi = a.K, a.N, a.epi
        A = _bf16((M, K), 4, 1.0)
        W = _bf16((N, K), 5, 0.02)
        bias = _bf16((N,), 6, 0.02)
        out = torch.zeros((M, N), dtype=torch.float32 if epi in (0, 3) else torch.bfloat16, device="cuda")
        flops = 2.0 * M * N * K

        def run():
            api.sal_linear(epi, A, W, bias, out=out)
    else:
        K, N, epi = {"stack_proj": (1024, 1280, api.SAL_EPI_STORE_F32),
                     "out_proj": (1280, 1280, api.SAL_EPI_RESID_F32),
                     "ffn_up": (1280, 5120, api.SAL_EPI_GELU_BF16),
                     "ffn_down": (5120, 1280, api.SAL_EPI_RESID_F32)}[a.kind]
        A = _bf16((M, K), 4, 1.0)
        W = _bf16((N, K), 5, 0.02)
        bias = _bf16((N,), 6, 0.02)
        out = torch.zeros((M, N), dtype=torch.float32 if epi in (0, 3) else torch.bfloat16, device="cuda")
        flops = 2.0 * M * N * K

        def run():
            api.sal_linear(epi, A, W, bias, out=out)

    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(a.reps):
            run()
    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    graph.replay()
    e1.record(s)
    torch.cuda.synchronize()
    if api.sal_last_device_status() != 0:
        raise RuntimeError("a device wait timed out")
    ms = e0.elapsed_time(e1) / a.reps
    out = {"kind": a.kind, "batch": B, "T": T, "avg_ms": ms}
    if flops:
        out["tflops"] = flops / (ms / 1e3) / 1e12
    if bytes_:
        out["gbs"] = bytes_ / (ms / 1e3) / 1e9
    print(json.dumps(out))


if __name__ == "__main__":
    main()
