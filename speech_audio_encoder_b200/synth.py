"""Seeded synthetic inputs: audio clips and random-init encoder weights.

This module is the only code that both the CUDA path and the fp64 oracle consume. It
holds input recipes only (random draws, a one-pole lowpass, tone bursts, bf16 rounding
of the weights) and none of the encoder's own arithmetic.

Audio recipes (the pages publish no audio; these stand in for the clip lengths they
discuss: 30 s chunks, 10-minute and one-hour recordings):

* ``tones``: 0.5 sin(2 pi 440 t) + 0.2 sin(2 pi 1000 t) + N(0, 0.01^2).
* ``bursts``: white N(0, 0.1^2) through y[n] = 0.95 y[n-1] + 0.05 w[n], plus 20 tone
  bursts (frequency U(100, 4000) Hz, amplitude U(0.05, 0.3), length U(0.1, 1.0) s,
  start U(0, D - length), Hann-tapered), optionally multiplied by the 4 Hz envelope
  0.55 + 0.45 sin(2 pi 4 t).

Weights: every matrix and bias N(0, 0.02); LayerNorm and QK-norm gains 1 + N(0, 0.02);
LayerNorm betas N(0, 0.02). Drawn in float64 with one PCG64 stream per tensor, rounded
once to bf16 (round to nearest even), and returned both as bf16 bit patterns (uint16)
and as the float32 values those bits encode.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
from scipy.signal import lfilter

SAMPLE_RATE = 16000


# ----------------------------------------------------------------------------- audio

def tones_clip(n_samples: int = 16000, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    t = np.arange(n_samples, dtype=np.float64) / SAMPLE_RATE
    x = 0.5 * np.sin(2 * np.pi * 440.0 * t) + 0.2 * np.sin(2 * np.pi * 1000.0 * t)
    x += rng.normal(0.0, 0.01, n_samples)
    return x.astype(np.float32)


def bursts_clip(n_samples: int, seed: int, envelope: bool = False,
                n_bursts: int = 20) -> np.ndarray:
    rng = np.random.default_rng(seed)
    w = rng.normal(0.0, 0.1, n_samples)
    x = lfilter([0.05], [1.0, -0.95], w)
    dur = n_samples / SAMPLE_RATE
    for _ in range(n_bursts):
        f = rng.uniform(100.0, 4000.0)
        amp = rng.uniform(0.05, 0.3)
        length = min(rng.uniform(0.1, 1.0), dur)
        start = rng.uniform(0.0, dur - length)
        i0 = int(start * SAMPLE_RATE)
        n = min(int(length * SAMPLE_RATE), n_samples - i0)
        if n <= 1:
            continue
        k = np.arange(n, dtype=np.float64)
        taper = 0.5 - 0.5 * np.cos(2 * np.pi * k / (n - 1))
        x[i0:i0 + n] += amp * taper * np.sin(2 * np.pi * f * k / SAMPLE_RATE)
    if envelope:
        t = np.arange(n_samples, dtype=np.float64) / SAMPLE_RATE
        x *= 0.55 + 0.45 * np.sin(2 * np.pi * 4.0 * t)
    return x.astype(np.float32)


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_samples: int
    n_layers: int
    kind: str          # "tones" | "bursts" | "bursts_env"
    seed: int

    @property
    def audio_seconds(self) -> float:
        return self.batch * self.n_samples / SAMPLE_RATE

    def audio(self) -> np.ndarray:
        """[batch, n_samples] float32, one seed per clip (seed + clip index)."""
        out = np.empty((self.batch, self.n_samples), dtype=np.float32)
        for b in range(self.batch):
            if self.kind == "tones":
                out[b] = tones_clip(self.n_samples, self.seed + b)
            else:
                out[b] = bursts_clip(self.n_samples, self.seed + b,
                                     envelope=(self.kind == "bursts_env"))
        return out


# The five workloads: a 1 s tone clip (2 layers), a 30 s clip, 16 x 60 s clips, a
# 10-minute recording and a one-hour recording (32 layers each).
WORKLOADS = {
    "tones_1s": Workload("tones_1s", 1, 16_000, 2, "tones", 0),
    "clip_30s": Workload("clip_30s", 1, 480_000, 32, "bursts", 1),
    "batch16_60s": Workload("batch16_60s", 16, 960_000, 32, "bursts", 100),
    "rec_10min": Workload("rec_10min", 1, 9_600_000, 32, "bursts_env", 2),
    "rec_1h": Workload("rec_1h", 1, 57_600_000, 32, "bursts_env", 3),
}
WORKLOAD_ORDER = ["tones_1s", "clip_30s", "batch16_60s", "rec_10min", "rec_1h"]


# ----------------------------------------------------------------------------- weights

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64/float32 values to bf16 (nearest even); return the uint16 bit patterns."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


LAYER_TENSORS = [
    # name, shape (as a function of width W, ffn Fd, head dim hd), init kind
    ("ln1_g", lambda W, Fd, hd: (W,), "gain"),
    ("ln1_b", lambda W, Fd, hd: (W,), "normal"),
    ("w_qkv", lambda W, Fd, hd: (3 * W, W), "normal"),
    ("b_qkv", lambda W, Fd, hd: (3 * W,), "normal"),
    ("qn_g", lambda W, Fd, hd: (hd,), "gain"),
    ("kn_g", lambda W, Fd, hd: (hd,), "gain"),
    ("w_o", lambda W, Fd, hd: (W, W), "normal"),
    ("b_o", lambda W, Fd, hd: (W,), "normal"),
    ("ln2_g", lambda W, Fd, hd: (W,), "gain"),
    ("ln2_b", lambda W, Fd, hd: (W,), "normal"),
    ("w1", lambda W, Fd, hd: (Fd, W), "normal"),
    ("b1", lambda W, Fd, hd: (Fd,), "normal"),
    ("w2", lambda W, Fd, hd: (W, Fd), "normal"),
    ("b2", lambda W, Fd, hd: (W,), "normal"),
]
GLOBAL_TENSORS = [
    ("w_proj", lambda W, S: (W, S), "normal"),
    ("b_proj", lambda W, S: (W,), "normal"),
    ("lnf_g", lambda W, S: (W,), "gain"),
    ("lnf_b", lambda W, S: (W,), "normal"),
]


def _draw(shape, kind: str, seed: int, std: float, gain_std: float) -> np.ndarray:
    rng = np.random.default_rng(seed)
    z = rng.standard_normal(shape)
    if kind == "gain":
        return 1.0 + gain_std * z
    return std * z


def make_weights(n_layers: int, seed: int = 1000, width: int = 1280, ffn: int = 5120,
                 head_dim: int = 128, stack_in: int = 1024, std: float = 0.02,
                 gain_std: float = 0.02, qk_gain_scale: float = 1.0) -> dict:
    """Random-init weights, bf16-rounded. Returns a nested dict of

    ``{"w_proj": (bits, f32), ..., "layers": [{"ln1_g": (bits, f32), ...}, ...]}``.
    Tensor i of the flat order (globals first, then layer by layer) uses seed + i.
    ``qk_gain_scale`` multiplies the q/k norm gains (a sharp-attention test case).
    """
    out: dict = {"layers": []}
    idx = 0
    for name, shp, kind in GLOBAL_TENSORS:
        v = _draw(shp(width, stack_in), kind, seed + idx, std, gain_std)
        b = bf16_bits(v)
        out[name] = (b, bf16_to_f32(b))
        idx += 1
    for _ in range(n_layers):
        lw = {}
        for name, shp, kind in LAYER_TENSORS:
            v = _draw(shp(width, ffn, head_dim), kind, seed + idx, std, gain_std)
            if name in ("qn_g", "kn_g"):
                v = v * qk_gain_scale
            b = bf16_bits(v)
            lw[name] = (b, bf16_to_f32(b))
            idx += 1
        out["layers"].append(lw)
    return out


def weights_f32(w: dict) -> dict:
    """The float32 values of :func:`make_weights` output, in the same nesting."""
    out = {k: v[1] for k, v in w.items() if k != "layers"}
    out["layers"] = [{k: v[1] for k, v in lw.items()} for lw in w["layers"]]
    return out


# ----------------------------------------------------------------------------- weight file
# The library's flat weight file (include/sal.h, "Flat weight file"): a 256-byte header,
# then every tensor as row-major bf16 on a 256-byte boundary, globals first, then layer by
# layer in LAYER_TENSORS order. The generator writes it; the oracle's tests and the
# library (sal_weights_file_load) read it.

WEIGHT_FILE_MAGIC = b"SALENCW1"
WEIGHT_FILE_ORDER_GLOBAL = ("w_proj", "b_proj", "lnf_g", "lnf_b")


def _padded_bytes(n_elems: int) -> int:
    return (2 * n_elems + 255) // 256 * 256


def _weight_file_tensors(w: dict):
    """(name, layer or None, bf16 bits) in file order."""
    for k in WEIGHT_FILE_ORDER_GLOBAL:
        yield k, None, w[k][0]
    for i, lw in enumerate(w["layers"]):
        for name, _, _ in LAYER_TENSORS:
            yield name, i, lw[name][0]


def write_weight_file(w: dict, path: str, width: int = 1280, heads: int = 10, head_dim: int = 128,
                      ffn: int = 5120, stack_in: int = 1024) -> int:
    """Writes :func:`make_weights` output to `path`; returns the data size D in bytes."""
    data = sum(_padded_bytes(b.size) for _, _, b in _weight_file_tensors(w))
    header = bytearray(256)
    header[0:8] = WEIGHT_FILE_MAGIC
    fields = [1, 256, 1, width, heads, head_dim, ffn, stack_in, len(w["layers"]), 256]
    header[8:48] = np.asarray(fields, dtype="<u4").tobytes()
    header[48:56] = np.asarray([data], dtype="<u8").tobytes()
    with open(path, "wb") as f:
        f.write(bytes(header))
        for _, _, bits in _weight_file_tensors(w):
            raw = np.ascontiguousarray(bits, dtype="<u2").tobytes()
            f.write(raw)
            f.write(bytes(_padded_bytes(bits.size) - len(raw)))
    return data


def read_weight_file(path: str, width: int = 1280, ffn: int = 5120, head_dim: int = 128,
                     stack_in: int = 1024) -> dict:
    """Reads a weight file back into the :func:`make_weights` form ``(bits, f32)``."""
    raw = np.fromfile(path, dtype=np.uint8)
    if raw[:8].tobytes() != WEIGHT_FILE_MAGIC:
        raise ValueError(f"{path}: not a weight file")
    fields = raw[8:48].view("<u4")
    n_layers = int(fields[8])
    if tuple(int(v) for v in fields[3:8]) != (width, 10, head_dim, ffn, stack_in):
        raise ValueError(f"{path}: sizes {tuple(fields[3:8])} differ")
    data = int(raw[48:56].view("<u8")[0])
    if raw.size != 256 + data:
        raise ValueError(f"{path}: {raw.size} bytes, header says {256 + data}")
    out: dict = {"layers": [{} for _ in range(n_layers)]}
    shapes = {name: shp(width, stack_in) for name, shp, _ in GLOBAL_TENSORS}
    layer_shapes = {name: shp(width, ffn, head_dim) for name, shp, _ in LAYER_TENSORS}
    off = 256
    order = [(k, None) for k in WEIGHT_FILE_ORDER_GLOBAL]
    order += [(name, i) for i in range(n_layers) for name, _, _ in LAYER_TENSORS]
    for name, i in order:
        shape = shapes[name] if i is None else layer_shapes[name]
        n = int(np.prod(shape))
        bits = raw[off:off + 2 * n].view("<u2").reshape(shape).astype(np.uint16)
        off += _padded_bytes(n)
        (out if i is None else out["layers"][i])[name] = (bits, bf16_to_f32(bits))
    return out


def random_bf16(shape, seed: int, std: float = 1.0):
    """N(0, std^2) values rounded to bf16: (bits, float32 values)."""
    b = bf16_bits(np.random.default_rng(seed).normal(0.0, std, shape))
    return b, bf16_to_f32(b)


# ----------------------------------------------------------------------------- speaker fusion inputs

def speaker_activity(T: int, seed: int, n_slots: int = 8, n_speakers: int = 3) -> np.ndarray:
    """[T, n_slots] float32 activities on the 80 ms grid: speakers take turns of 1-10 s
    (12-125 positions) with some overlap, plus N(0, 0.2) noise clipped to [0, 1]; unused
    slots stay near 0. A few entries are exactly 0.5 (the threshold)."""
    rng = np.random.default_rng(seed)
    P = np.zeros((T, n_slots))
    t = 0
    while t < T:
        n = int(rng.integers(12, 126))
        spk = int(rng.integers(0, n_speakers))
        P[t:t + n, spk] = 1.0
        if rng.uniform() < 0.2:  # an overlapping second speaker
            P[t + n // 2:t + n, (spk + 1) % n_speakers] = 1.0
        t += n
    P = np.clip(P + rng.normal(0.0, 0.2, P.shape), 0.0, 1.0)
    P[rng.integers(0, T, max(1, T // 50)), rng.integers(0, n_slots, max(1, T // 50))] = 0.5
    return P.astype(np.float32)


def make_fusion_weights(seed: int = 5000, width: int = 1280, llm_width: int = 2688, n_slots: int = 8,
                        std: float = 0.02, gain_std: float = 0.02) -> dict:
    """Speaker LayerNorm (gain 1 + N(0, 0.02), bias N(0, 0.02)) and the connector
    (N(0, 0.02) weights and bias), bf16-rounded: {name: (bits, float32)}."""
    out = {}
    for i, (name, shape, kind) in enumerate([("spk_g", (n_slots,), "gain"), ("spk_b", (n_slots,), "normal"),
                                              ("w_conn", (llm_width, width), "normal"),
                                              ("b_conn", (llm_width,), "normal")]):
        b = bf16_bits(_draw(shape, kind, seed + i, std, gain_std))
        out[name] = (b, bf16_to_f32(b))
    return out


# ----------------------------------------------------------------------------- CTC adapter weights

def make_ctc_weights(seed: int = 7000, in_width: int = 1280, width: int = 1024, ffn: int = 4096,
                     head_dim: int = 64, n_layers: int = 2, classes: int = 23863, std: float = 0.02,
                     gain_std: float = 0.02) -> dict:
    """Random-init weights of the CTC timestamp adapter, bf16-rounded, as {name: (bits, f32)}
    with "layers" a list of per-layer dicts (the encoder's layer tensors at this width).
    w_up [2, width, in_width] holds the two taps of the transposed convolution; w_out
    [classes, width]. Tensor i of the flat order uses seed + i."""
    out: dict = {"layers": []}
    idx = 0

    def put(d, name, shape, kind):
        nonlocal idx
        b = bf16_bits(_draw(shape, kind, seed + idx, std, gain_std))
        d[name] = (b, bf16_to_f32(b))
        idx += 1

    put(out, "w_up", (2, width, in_width), "normal")
    put(out, "b_up", (width,), "normal")
    for _ in range(n_layers):
        lw: dict = {}
        for name, shp, kind in LAYER_TENSORS:
            put(lw, name, shp(width, ffn, head_dim), kind)
        out["layers"].append(lw)
    put(out, "lnf_g", (width,), "gain")
    put(out, "lnf_b", (width,), "normal")
    put(out, "w_out", (classes, width), "normal")
    put(out, "b_out", (classes,), "normal")
    return out
