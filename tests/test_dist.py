"""Host-side multi-rank logic of bench.py, run as two gloo ranks on CPU.

bench.py shards by clip: every rank encodes its own clips (audio seeds offset per rank),
no data crosses ranks, and the job's time is the maximum over ranks. These tests check
that max reduction, the whole-job throughput arithmetic, and that ranks get distinct
inputs, with world size 2 over gloo.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from speech_audio_encoder_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, local = bench.dist_env()
        # each rank's own "timed region"
        mine = 1.5 + rank
        worst = bench.reduce_max(mine)
        wl = synth.WORKLOADS["tones_1s"]
        my = synth.Workload(wl.name, wl.batch, wl.n_samples, wl.n_layers, wl.kind,
                            wl.seed + bench.rank_seed_offset(r))
        audio = my.audio()
        value = bench.job_throughput(my.audio_seconds * 10, w, worst)
        out_q.put((r, w, local, worst, value, float(audio[0, :100].sum())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, l0, worst0, v0, a0), (r1, w1, l1, worst1, v1, a1) = res
    assert (r0, r1, w0, w1, l0, l1) == (0, 1, 2, 2, 0, 1)
    assert worst0 == worst1 == 2.5          # max over ranks, seen by both
    assert v0 == v1 == pytest.approx(2 * 10 * 1.0 / 2.5)  # 1 s of audio x 10 steps x 2 ranks
    assert a0 != a1                          # each rank encodes its own clip


def test_single_process_helpers():
    assert bench.reduce_max(3.0) == 3.0
    assert bench.job_throughput(30.0, 4, 2.0) == 60.0
    assert bench.positions(480000) == 374 and bench.frames(480000) == 2998
    assert bench.workload_flops(1, 374, 32) == pytest.approx(
        39321600 * 374 * 32 + 5120 * 374 * 374 * 32 + 2621440 * 374)
    assert bench.kernel_flops("ffn_up", 16, 749) == 2.0 * 16 * 749 * 1280 * 5120
    assert np.isclose(bench.kernel_flops("attention", 1, 100), 4 * 100 * 100 * 1280)
