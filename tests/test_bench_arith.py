"""The measurement arithmetic of bench.py against closed forms: algorithmic flops per
position and layer (two-matrix FFN, width 1280), attention flops 4 T^2 d per layer and clip,
the front end's algorithmic bytes, and the workload totals the baseline notes quote
(0.494 TFLOP at 30 s, 388.5 TFLOP at one hour)."""
import bench
import oracle as O


def test_per_unit_flops():
    assert bench.GEMM_FLOPS_PER_POS_LAYER == 2 * (4 * 1280 ** 2 + 2 * 1280 * 5120) == 39_321_600
    assert bench.ATTN_FLOPS_PER_T2_LAYER == 4 * 1280 == 5120
    assert bench.STACK_PROJ_FLOPS_PER_POS == 2 * 1024 * 1280


def test_kernel_flops_sum_to_the_layer():
    B, T = 2, 700
    gemm = sum(bench.kernel_flops(k, B, T) for k in ("qkv", "out_proj", "ffn_up", "ffn_down"))
    assert gemm == bench.GEMM_FLOPS_PER_POS_LAYER * B * T
    assert bench.kernel_flops("attention", B, T) == 4 * T * T * 1280 * B


def test_chunked_attention_pairs():
    assert bench.attention_pairs(1000, 0) == 1000 ** 2
    assert bench.attention_pairs(1000, 375) == 2 * 375 ** 2 + 250 ** 2
    assert bench.attention_pairs(1000, 5000) == 1000 ** 2


def test_workload_totals():
    t30 = O.position_count(480_000)
    t1h = O.position_count(57_600_000)
    assert abs(bench.workload_flops(1, t30, 32) / 1e12 - 0.494) < 0.001
    assert abs(bench.workload_flops(1, t1h, 32) / 1e12 - 388.5) < 0.1


def test_frontend_bytes():
    # one hour: 57.6 M samples read, 359,998 fp32 log-mel rows, 44,999 bf16 stacked rows
    assert bench.frontend_bytes(1, 57_600_000) == 4 * 57_600_000 + 512 * 359_998 + 2048 * 44_999
    assert bench.frontend_bytes(3, 16_000) == 3 * (4 * 16_000 + 512 * 98 + 2048 * 12)
    assert bench.frontend_bytes(1, 399) == 4 * 399


def test_serving_window_work():
    """Serving windows: every window's own positions and pairs, context included; the
    lengths agree with the oracle's window bounds."""
    T = O.position_count(57_600_000)
    lens = bench.window_lengths(T, 500, 50)
    assert lens == [hi - lo for lo, _, _, hi in O.window_bounds(T, 500, 50)]
    assert len(lens) == 90 and lens[0] == 550 and lens[1] == 600 and lens[-1] == 549
    rows, pairs = bench.layer_work(T, window=(500, 50))
    assert rows == sum(lens) == T + 2 * 50 * 89
    assert pairs == sum(n * n for n in lens)
    assert bench.layer_work(T) == (T, T * T)
    assert bench.kernel_flops("attention", 1, T, window=(500, 50)) == 5120 * pairs


def test_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    """The bench reports a stored DRAM figure only for the workload it was captured on and
    only while the kernel's source hashes as it did then."""
    import hashlib
    import json
    import os

    src = tmp_path / "kernel.cu"
    src.write_text("// v1\n")
    (tmp_path / "profiles").mkdir()
    rec = {"attention": {"workload": "rec_1h", "dram_bytes_per_launch": 123, "source": "kernel.cu",
                         "sha256_16": hashlib.sha256(b"// v1\n").hexdigest()[:16]}}
    (tmp_path / "profiles" / "roofline_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("attention", "rec_1h") == 123
    assert bench._traffic("attention", "rec_10min") is None  # another workload
    assert bench._traffic("qkv", "rec_1h") is None  # no record
    src.write_text("// v2\n")
    assert bench._traffic("attention", "rec_1h") is None  # the kernel changed since the capture
    os.remove(tmp_path / "profiles" / "roofline_traffic.json")
    assert bench._traffic("attention", "rec_1h") is None

