"""fp64 oracle: log-mel front end, 8-frame stacking and the bidirectional Transformer encoder.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
legs of ``bench.py`` may call this module. The product path never routes through it.

The arithmetic is the plain C++ of ``sal_oracle.cpp`` (``liboracle.so``, textbook loops in
double precision: an explicit DFT sum, explicit Slaney mel rows, triple-loop matrix
products, two-pass LayerNorm, max-subtracted softmax, ``std::erf`` GELU and fp64 RoPE).
This module marshals numpy arrays to it and composes its steps in the page's order;
integer bookkeeping (frame counts, chunk and window bounds, parameter counts) is written
here directly.

Sources (all on the page "Nemotron 3.5 Transcribe: From Recorded Speech to Dataset
Audits", flozi.net):

* [ARCH]  section "How audio and speakers reach the language model", the paragraph on
  the exported frontend: 16 kHz mono input, 128 log-mel features, 25 ms Hann window,
  512-point FFT, 10 ms hop; eight stacked frames projected to width 1,280; 32 Transformer
  layers, ten heads, QK normalization, feed-forward expansion four, rotary position
  embeddings; 12.5 embeddings per second (80 ms per position).
* [ARCH-600M] same section, the ASR Transformer is "roughly 600M" parameters.
* [POS]   section "How one hour fits into 65,536 positions": 12.5 D positions per D
  seconds, nominally 375 per 30 s and 45,000 per hour, ignoring rounding at the ends.
* [SERVE] section "Serving choices that change the audit": an hour of 16 kHz mono audio
  decodes to about 230.4 MB of float32.
* [FUSE]  section "How audio and speakers reach the language model", the paragraphs after
  the frontend one: speaker activity for eight slots, aligned to the ASR grid, thresholded
  at 0.5, a learned LayerNorm over the speaker dimension, a fixed sinusoidal speaker kernel
  (scale 1) mapping the eight slot indicators to width 1,280, summed into the ASR states;
  then one learned linear projection (the identity connector) to the language width 2,688
  (the width of the language backbone's block input, section on the released backbone).
  The fusion equation itself is missing from the page text; readings 13-16 below.
* [CHUNK] section "Local encoder windows, recording-wide language context": in training the
  encoder runs on independent 30-second post-feature chunks with no attention across
  their borders, and the chunk outputs are concatenated in order; pairs scale as T w.
* [WINDOW] section "Local encoder windows, recording-wide language context", the
  paragraph on the serving path: the encoder runs on context-extended windows, the outputs
  at overlap (context) positions are discarded and the core outputs concatenated; the
  defaults are 500 encoded core positions with 50 context positions on each side (80 ms
  per position). Edge handling is not given; reading 22 below.
* [CTC]   section "Use alignment and audio questions as supporting evidence": a CTC
  timestamp adapter of about 50M parameters takes the unfused ASR states (width 1,280),
  upsamples their 80 ms grid to 40 ms with a stride-two transposed convolution, runs two
  Transformer layers with 16 heads, and projects to a 23,862-token vocabulary plus the
  CTC blank. Widths and kernel size are not given; readings 17-21 below.

Readings where the pages are silent (each one is listed in the design notes):

1. frames F = 1 + floor((N - 400) / 160) for N >= 400 else 0; positions T = floor(F / 8);
   no centre or tail padding; remainder frames are dropped.
2. periodic Hann window of length 400, w[n] = 0.5 - 0.5 cos(2 pi n / 400).
3. power spectrum |X_k|^2 of the 400 windowed samples zero-padded to 512, k = 0..256.
4. Slaney mel scale and Slaney area normalisation, 130 points equally spaced in mel
   over 0..8000 Hz, 128 triangular filters on the bin frequencies 31.25 k Hz.
5. natural log with a clamp at 1e-10: ln(max(e, 1e-10)).
6. frame-major stacking S[t, 128 j + m] = M[8 t + j, m].
7. every linear layer has a bias; weights are [out, in].
8. pre-norm LayerNorm (eps 1e-5) before attention and before the FFN, plus a final
   LayerNorm after the last layer.
9. QK normalisation is RMS over head_dim 128 (eps 1e-6) with one gain vector for q and
   one for k, shared by the heads, applied before RoPE.
10. RoPE rotates the pairs (i, i + 64) by t * 10000^(-2 i / 128), t = 0..T-1 per clip.
11. attention is softmax(q k^T / sqrt(128)) v over the whole clip, no mask.
12. GELU is the exact erf form; the FFN has two matrices (1280 -> 5120 -> 1280).
13. speaker activity arrives already on the 80 ms ASR grid, P [T, 8] in [0, 1]; the
    indicator is P > 0.5 (strict).
14. the speaker LayerNorm normalises the 8 indicators of a position (eps 1e-5, gain and
    bias of length 8).
15. the speaker kernel is the sinusoidal table K[s, 2i] = sin(s w_i), K[s, 2i+1] = cos(s w_i),
    w_i = 10000^(-2i/1280), s = 0..7; fused = H + 1 * LN(indicators) K.
16. the connector is x W^T + b with W [2688, 1280].
17. the adapter's transposed convolution has kernel size 2 (equal to its stride), so each
    80 ms state gives two 40 ms states with no overlap: U[2t + j] = h[t] W_j^T + b,
    j in {0, 1}, one bias per output channel.
18. the adapter width is 1,024 (16 heads of 64): with the encoder's layer recipe and an
    FFN of 4,096, it is the width that gives about 50M parameters (52.3M; 768 gives 35M,
    1,280 gives 73M).
19. the adapter layers follow the encoder's recipe (readings 8-12) at that width; RoPE
    positions count 40 ms steps from the clip start.
20. a final LayerNorm precedes the projection (as after the encoder); the projection has a
    bias and 23,863 outputs, the blank last.
21. the adapter's output is the frame log-probabilities, log_softmax over the 23,863
    classes.
22. serving windows: the cores are consecutive runs of ``core`` positions from the clip
    start (the last may be shorter); a window is its core extended by ``context``
    positions on each side, clipped to the clip, so the first window has no left context
    and the last no right context beyond the clip end. Each window is encoded as an
    independent sequence (all layers and the final LayerNorm, attention inside the window,
    RoPE positions from 0 at the window start); its core outputs are kept in order.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

SAMPLE_RATE = 16000  # [ARCH]
WIN = 400            # 25 ms at 16 kHz [ARCH]
HOP = 160            # 10 ms at 16 kHz [ARCH]
NFFT = 512           # [ARCH]
NBINS = NFFT // 2 + 1
NMEL = 128           # [ARCH]
STACK = 8            # [ARCH]
LOG_FLOOR = 1e-10    # reading 5
LN_EPS = 1e-5        # reading 8
QK_EPS = 1e-6        # reading 9
ROPE_BASE = 10000.0  # reading 10
MAX_POSITIONS = 45000  # one hour at 12.5 positions/s [POS]
WINDOW_CORE = 500      # serving window core positions [WINDOW]
WINDOW_CONTEXT = 50    # serving window context positions on each side [WINDOW]
N_SLOTS = 8            # speaker slots [FUSE]
LLM_WIDTH = 2688       # language width [FUSE]

__all__ = [
    "SAMPLE_RATE", "WIN", "HOP", "NFFT", "NBINS", "NMEL", "STACK", "LOG_FLOOR",
    "LN_EPS", "QK_EPS", "ROPE_BASE", "MAX_POSITIONS",
    "EncoderDims", "DIMS", "frame_count", "position_count", "hann_window",
    "frame_signal", "power_spectrum", "hz_to_mel", "mel_to_hz", "mel_filterbank",
    "log_mel", "stack_frames", "linear", "layer_norm", "rms_norm", "rope_angles",
    "rope", "attention_probs", "attention", "gelu", "encoder_layer",
    "encoder_layer_rows", "encoder_forward", "stack_project", "encode",
    "param_count", "rel_l2", "chunk_bounds", "encoder_layer_chunked",
    "encoder_layer_rows_chunked", "encoder_forward_chunked", "window_bounds",
    "encoder_forward_windowed", "WINDOW_CORE", "WINDOW_CONTEXT", "N_SLOTS", "LLM_WIDTH",
    "speaker_kernel", "speaker_fuse", "connector", "CtcDims", "CTC", "ctc_upsample",
    "log_softmax", "ctc_logits", "ctc_adapter", "ctc_param_count", "threads", "LIB_PATH",
]

# ----------------------------------------------------------------------------- the C++ library

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "sal_oracle.cpp")
LIB_PATH = os.path.join(_HERE, "liboracle.so")
# x86-64-v3 (AVX2, FMA): a target every current server CPU runs, here and on other hosts
CXX_FLAGS = ["-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared", "-std=c++17"]

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source with g++ (when missing or older)."""
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SOURCE):
        return LIB_PATH
    tmp = LIB_PATH + f".{os.getpid()}.tmp"
    r = subprocess.run(["g++", *CXX_FLAGS, SOURCE, "-o", tmp], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"building the oracle failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64


class _Layer(ctypes.Structure):
    _fields_ = [(n, _D) for n in ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "qn_g", "kn_g", "w_o", "b_o",
                                  "ln2_g", "ln2_b", "w1", "b1", "w2", "b2")]


_SIGS = {
    "oc_threads": (ctypes.c_int, []),
    "oc_frame_count": (_I64, [_I64]),
    "oc_hann": (None, [_D]),
    "oc_hz_to_mel": (ctypes.c_double, [ctypes.c_double]),
    "oc_mel_to_hz": (ctypes.c_double, [ctypes.c_double]),
    "oc_mel_filterbank": (None, [_D]),
    "oc_linear": (None, [_D, _I64, _I64, _D, _I64, _D, _D]),
    "oc_power_spectrum": (None, [_D, _I64, _I64, _D]),
    "oc_log_mel": (None, [ctypes.POINTER(ctypes.c_float), _I64, _I64, _I64, _D]),
    "oc_layer_norm": (None, [_D, _I64, _I64, _D, _D, ctypes.c_double, _D]),
    "oc_rms_norm": (None, [_D, _I64, _I64, _D, ctypes.c_double, _D]),
    "oc_rope": (None, [_D, _I64, _I64, _D, _D]),
    "oc_attention_probs": (None, [_D, _I64, _D, _I64, _I64, _D]),
    "oc_attention": (None, [_D, _I64, _I64, _D, _D, _I64, _I64, _D]),
    "oc_gelu": (None, [_D, _I64, _D]),
    "oc_encoder_layer_rows": (None, [_D, _I64, _I64, _I64, _I64, _I64, ctypes.POINTER(_Layer),
                                     ctypes.POINTER(_I64), _I64, _D]),
    "oc_speaker_kernel": (None, [_I64, _I64, _D]),
    "oc_log_softmax": (None, [_D, _I64, _I64, _D]),
}


def _load():
    global _lib
    with _lock:
        if _lib is None:
            l = ctypes.CDLL(build())
            for name, (res, args) in _SIGS.items():
                f = getattr(l, name)
                f.restype = res
                f.argtypes = args
            _lib = l
    return _lib


def threads() -> int:
    """Threads the C++ oracle runs on (OpenMP)."""
    return _load().oc_threads()


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(_D)


# ----------------------------------------------------------------------------- counts

@dataclass(frozen=True)
class EncoderDims:
    """Encoder shape. The defaults are the published ones [ARCH]; tests shrink them."""
    width: int = 1280
    heads: int = 10
    head_dim: int = 128
    ffn: int = 5120          # expansion four [ARCH]
    stack_in: int = NMEL * STACK  # 1024


DIMS = EncoderDims()


def frame_count(n_samples: int) -> int:
    """Number of 400-sample frames at a 160-sample hop (reading 1, [ARCH])."""
    n = int(n_samples)
    return 0 if n < WIN else 1 + (n - WIN) // HOP


def position_count(n_samples: int) -> int:
    """Encoder positions after stacking eight frames; the remainder is dropped [ARCH]."""
    return frame_count(n_samples) // STACK


# ----------------------------------------------------------------------------- front end

def hann_window() -> np.ndarray:
    """Periodic Hann window of length 400 (reading 2)."""
    w = np.empty(WIN)
    _load().oc_hann(_p(w))
    return w


def frame_signal(wave: np.ndarray, first: int = 0, count: int | None = None) -> np.ndarray:
    """Windowed frames y_f[n] = w[n] x[160 f + n], n < 400, for f in [first, first+count)."""
    x = np.asarray(wave, dtype=np.float64)
    F = frame_count(x.shape[0])
    if count is None:
        count = F - first
    idx = (first + np.arange(count))[:, None] * HOP + np.arange(WIN)[None, :]
    return x[idx] * hann_window()[None, :]


def power_spectrum(y: np.ndarray) -> np.ndarray:
    """|X_k|^2 for k = 0..256 of frames zero-padded to 512 samples (reading 3), by the
    explicit DFT sum over the frame's own samples."""
    y = _f64(y)
    shape = y.shape[:-1]
    y2 = y.reshape(-1, y.shape[-1])
    P = np.empty((y2.shape[0], NBINS))
    _load().oc_power_spectrum(_p(y2), y2.shape[0], y2.shape[1], _p(P))
    return P.reshape(shape + (NBINS,))


def hz_to_mel(f):
    """Slaney mel scale: linear 3 f / 200 below 1 kHz, logarithmic above (reading 4)."""
    l = _load()
    return np.vectorize(l.oc_hz_to_mel, otypes=[np.float64])(np.asarray(f, dtype=np.float64))


def mel_to_hz(m):
    """Inverse of :func:`hz_to_mel`."""
    l = _load()
    return np.vectorize(l.oc_mel_to_hz, otypes=[np.float64])(np.asarray(m, dtype=np.float64))


def mel_filterbank() -> np.ndarray:
    """128 x 257 Slaney-normalised triangular filters over 0..8 kHz (reading 4)."""
    W = np.empty((NMEL, NBINS))
    _load().oc_mel_filterbank(_p(W))
    return W


def log_mel(wave: np.ndarray, chunk: int = 8192, first: int = 0,
            count: int | None = None) -> np.ndarray:
    """[F, 128] natural-log mel energies of one clip ([ARCH], readings 1-5).

    ``first``/``count`` select a range of frames; frames are independent, so the range
    is only a way to sample long clips. (``chunk`` is kept for callers; the C++ side
    takes frames 8,192 at a time.)
    """
    x = np.ascontiguousarray(wave, dtype=np.float32)
    F = frame_count(x.shape[0])
    if count is None:
        count = F - first
    if first < 0 or count < 0 or first + count > F:
        raise ValueError("frame range outside the clip")
    out = np.empty((count, NMEL))
    if count:
        _load().oc_log_mel(x.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), x.shape[0], first, count, _p(out))
    return out


def stack_frames(logmel: np.ndarray) -> np.ndarray:
    """S[t, 128 j + m] = M[8 t + j, m] for t < floor(F / 8) ([ARCH], reading 6)."""
    M = np.asarray(logmel)
    T = M.shape[0] // STACK
    S = np.empty((T, STACK * M.shape[1]), dtype=np.float64)
    for j in range(STACK):
        S[:, j * M.shape[1]:(j + 1) * M.shape[1]] = M[j:T * STACK:STACK]
    return S


# ----------------------------------------------------------------------------- encoder pieces

def linear(x, w, b):
    """x W^T + b with W stored [out, in] (reading 7)."""
    x, w = _f64(x), _f64(w)
    lead = x.shape[:-1]
    x2 = x.reshape(-1, x.shape[-1])
    out = np.empty((x2.shape[0], w.shape[0]))
    bb = None if b is None else _f64(b)
    _load().oc_linear(_p(x2), x2.shape[0], x2.shape[1], _p(w), w.shape[0], None if bb is None else _p(bb), _p(out))
    return out.reshape(lead + (w.shape[0],))


def layer_norm(x, g, b, eps: float = LN_EPS):
    """Per-row LayerNorm with two-pass mean and variance (reading 8)."""
    x = _f64(x)
    x2 = x.reshape(-1, x.shape[-1])
    y = np.empty_like(x2)
    _load().oc_layer_norm(_p(x2), x2.shape[0], x2.shape[1], _p(_f64(np.broadcast_to(g, x.shape[-1:]))),
                          _p(_f64(np.broadcast_to(b, x.shape[-1:]))), eps, _p(y))
    return y.reshape(x.shape)


def rms_norm(x, g, eps: float = QK_EPS):
    """x / sqrt(mean(x^2) + eps) * g over the last axis (reading 9)."""
    x = _f64(x)
    x2 = x.reshape(-1, x.shape[-1])
    y = np.empty_like(x2)
    _load().oc_rms_norm(_p(x2), x2.shape[0], x2.shape[1], _p(_f64(np.broadcast_to(g, x.shape[-1:]))), eps, _p(y))
    return y.reshape(x.shape)


def rope_angles(positions, head_dim: int):
    """t * base^(-2 i / head_dim) for i < head_dim / 2 (reading 10)."""
    half = head_dim // 2
    inv = ROPE_BASE ** (-2.0 * np.arange(half, dtype=np.float64) / head_dim)
    return _f64(positions)[:, None] * inv[None, :]


def rope(x, positions):
    """Rotate the pairs (i, i + hd/2) of x [..., T, hd] by the angles of ``positions``."""
    x = _f64(x)
    T, hd = x.shape[-2], x.shape[-1]
    pos = _f64(positions)
    x3 = x.reshape(-1, T, hd)
    y = np.empty_like(x3)
    for i in range(x3.shape[0]):
        _load().oc_rope(_p(np.ascontiguousarray(x3[i])), T, hd, _p(pos), _p(y[i]))
    return y.reshape(x.shape)


def attention_probs(q, k):
    """softmax(q k^T / sqrt(hd)) over keys, with the row maximum subtracted (reading 11)."""
    q, k = _f64(q), _f64(k)
    P = np.empty((q.shape[0], k.shape[0]))
    _load().oc_attention_probs(_p(q), q.shape[0], _p(k), k.shape[0], q.shape[1], _p(P))
    return P


def attention(q, k, v, chunk: int = 2048):
    """Per head: softmax(q k^T / sqrt(hd)) v. q [H, Tq, hd], k and v [H, Tk, hd].
    (``chunk`` is kept for callers; the C++ side walks query rows one at a time.)"""
    q, k, v = _f64(q), _f64(k), _f64(v)
    out = np.empty(q.shape[:-1] + (v.shape[-1],))
    _load().oc_attention(_p(q), q.shape[0], q.shape[1], _p(k), _p(v), k.shape[1], q.shape[2], _p(out))
    return out


def gelu(x):
    """Exact GELU 0.5 x (1 + erf(x / sqrt 2)) (reading 12)."""
    x = _f64(x)
    y = np.empty_like(x)
    _load().oc_gelu(_p(x), x.size, _p(y))
    return y


_LAYER_KEYS = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "qn_g", "kn_g", "w_o", "b_o",
               "ln2_g", "ln2_b", "w1", "b1", "w2", "b2")


def encoder_layer_rows(x, lw, rows, dims: EncoderDims = DIMS):
    """One pre-norm bidirectional Transformer layer on one clip x [T, width] ([ARCH]),
    evaluated only at the positions ``rows``: x + Attn(LN1(x)), then + FFN(LN2(.)), with
    keys and values from every position (so the rows equal the same rows of the full
    layer)."""
    x = _f64(x)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    T = x.shape[0]
    if rows.size and (rows.min() < 0 or rows.max() >= T):
        raise IndexError("row outside the clip")
    keep = {k: _f64(lw[k]) for k in _LAYER_KEYS}
    L = _Layer(*[_p(keep[k]) for k in _LAYER_KEYS])
    out = np.empty((len(rows), dims.width))
    if len(rows):
        _load().oc_encoder_layer_rows(_p(x), T, dims.width, dims.heads, dims.head_dim, dims.ffn, ctypes.byref(L),
                                      rows.ctypes.data_as(ctypes.POINTER(_I64)), len(rows), _p(out))
    return out


def encoder_layer(x, lw, dims: EncoderDims = DIMS):
    """One pre-norm bidirectional Transformer layer on one clip x [T, width] ([ARCH]),
    with the attention over all T positions."""
    return encoder_layer_rows(x, lw, np.arange(_f64(x).shape[0]), dims)


def chunk_bounds(T: int, chunk: int):
    """[(start, end)] of consecutive chunks of ``chunk`` positions (``chunk`` <= 0: one chunk,
    the whole clip); the last may be shorter; an empty clip has none."""
    if T <= 0:
        return []
    chunk = T if chunk <= 0 else chunk
    return [(s, min(s + chunk, T)) for s in range(0, T, chunk)]


def encoder_layer_chunked(x, lw, chunk: int, dims: EncoderDims = DIMS):
    """One layer where each chunk of ``chunk`` positions is an independent sequence
    ([CHUNK]): attention stays inside the chunk and RoPE positions restart at its start."""
    x = _f64(x)
    return np.concatenate([encoder_layer(x[a:b], lw, dims) for a, b in chunk_bounds(len(x), chunk)])


def encoder_layer_rows_chunked(x, lw, rows, chunk: int, dims: EncoderDims = DIMS):
    """:func:`encoder_layer_chunked` evaluated only at the positions ``rows``."""
    x = _f64(x)
    rows = np.asarray(rows)
    out = np.empty((len(rows), x.shape[1]))
    for a, b in chunk_bounds(len(x), chunk):
        sel = np.nonzero((rows >= a) & (rows < b))[0]
        if len(sel):
            out[sel] = encoder_layer_rows(x[a:b], lw, rows[sel] - a, dims)
    return out


def encoder_forward_chunked(x0, weights, n_layers: int, chunk: int, dims: EncoderDims = DIMS):
    """Chunked encoder: every chunk runs all layers on its own; final LayerNorm per position."""
    x = _f64(x0)
    for i in range(n_layers):
        x = encoder_layer_chunked(x, weights["layers"][i], chunk, dims)
    return layer_norm(x, weights["lnf_g"], weights["lnf_b"])


def window_bounds(T: int, core: int = WINDOW_CORE, context: int = WINDOW_CONTEXT):
    """[(lo, c0, c1, hi)] per serving window ([WINDOW], reading 22): the core [c0, c1) of
    ``core`` positions (the last may be shorter) and the window [lo, hi) that extends it by
    ``context`` positions on each side, clipped to [0, T). An empty clip has none."""
    out = []
    for c0 in range(0, max(T, 0), core):
        c1 = min(c0 + core, T)
        out.append((max(0, c0 - context), c0, c1, min(T, c1 + context)))
    return out


def encoder_forward_windowed(x0, weights, n_layers: int, core: int = WINDOW_CORE,
                             context: int = WINDOW_CONTEXT, dims: EncoderDims = DIMS):
    """Serving-window encoder ([WINDOW], reading 22): every window runs ``n_layers`` layers
    and the final LayerNorm on its own positions as an independent sequence; the outputs
    at its context positions are discarded and the core outputs concatenated in order."""
    x = _f64(x0)
    parts = [encoder_forward(x[lo:hi], weights, n_layers, dims)[c0 - lo:c1 - lo]
             for lo, c0, c1, hi in window_bounds(len(x), core, context)]
    return np.concatenate(parts) if parts else np.empty((0, x.shape[1]))


def speaker_kernel(n_slots: int = N_SLOTS, width: int = 1280) -> np.ndarray:
    """Fixed sinusoidal speaker kernel K [n_slots, width] (reading 15)."""
    K = np.empty((n_slots, width))
    _load().oc_speaker_kernel(n_slots, width, _p(K))
    return K


def speaker_fuse(H, P, g, b, scale: float = 1.0):
    """H + scale * LN_slots(P > 0.5) K ([FUSE], readings 13-15). H [T, 1280], P [T, 8]."""
    A = (np.asarray(P, dtype=np.float64) > 0.5).astype(np.float64)
    H = _f64(H)
    K = speaker_kernel(A.shape[1], H.shape[1])
    return H + scale * linear(layer_norm(A, g, b), np.ascontiguousarray(K.T), None)


def connector(x, w, b):
    """The identity connector: one linear projection to the language width ([FUSE], 16)."""
    return linear(x, w, b)


# ----------------------------------------------------------------------------- CTC timestamp adapter

@dataclass(frozen=True)
class CtcDims:
    """Shape of the CTC timestamp adapter ([CTC], readings 17-21)."""
    in_width: int = 1280   # the unfused ASR states [CTC]
    width: int = 1024      # reading 18
    heads: int = 16        # [CTC]
    head_dim: int = 64
    ffn: int = 4096        # expansion four, as in the encoder (reading 19)
    layers: int = 2        # [CTC]
    classes: int = 23863   # 23,862 tokens + the CTC blank [CTC]

    @property
    def layer_dims(self) -> EncoderDims:
        return EncoderDims(width=self.width, heads=self.heads, head_dim=self.head_dim, ffn=self.ffn)


CTC = CtcDims()


def ctc_upsample(h, w_up, b_up):
    """Stride-two transposed convolution with kernel 2 ([CTC], reading 17): the state of
    position t gives the states 2t and 2t + 1, U[2t + j] = h[t] W_j^T + b, with
    w_up [2, width, in_width] holding W_0 and W_1 and b_up [width]."""
    h, w = _f64(h), _f64(w_up)
    U = np.empty((2 * h.shape[0], w.shape[1]), dtype=np.float64)
    for j in range(2):
        U[j::2] = linear(h, w[j], b_up)
    return U


def log_softmax(z):
    """log(softmax(z)) over the last axis, with the row maximum subtracted (reading 21)."""
    z = _f64(z)
    z2 = z.reshape(-1, z.shape[-1])
    y = np.empty_like(z2)
    _load().oc_log_softmax(_p(z2), z2.shape[0], z2.shape[1], _p(y))
    return y.reshape(z.shape)


def ctc_logits(h, cw, dims: CtcDims = CTC):
    """Class scores [2T, classes] of the adapter on one clip's unfused states h [T, in_width]:
    upsampling, the Transformer layers, the final LayerNorm and the projection."""
    x = ctc_upsample(h, cw["w_up"], cw["b_up"])
    for lw in cw["layers"][:dims.layers]:
        x = encoder_layer(x, lw, dims.layer_dims)
    return linear(layer_norm(x, cw["lnf_g"], cw["lnf_b"]), cw["w_out"], cw["b_out"])


def ctc_adapter(h, cw, dims: CtcDims = CTC):
    """Frame log-probabilities [2T, classes] on the 40 ms grid ([CTC], reading 21)."""
    return log_softmax(ctc_logits(h, cw, dims))


def ctc_param_count(dims: CtcDims = CTC) -> int:
    """Parameters of the adapter: transposed convolution, layers, final LN, projection."""
    W = dims.width
    up = 2 * W * dims.in_width + W
    layers = param_count(dims.layers, dims.layer_dims) - (dims.layer_dims.stack_in * W + W + 2 * W)
    return up + layers + 2 * W + dims.classes * W + dims.classes


def stack_project(stacked, weights):
    """x0 = S P^T + p: the 1024 -> 1280 projection of the stacked frames [ARCH]."""
    return linear(stacked, weights["w_proj"], weights["b_proj"])


def encoder_forward(x0, weights, n_layers: int, dims: EncoderDims = DIMS):
    """``n_layers`` encoder layers on one clip, then the final LayerNorm (reading 8)."""
    x = _f64(x0)
    for i in range(n_layers):
        x = encoder_layer(x, weights["layers"][i], dims)
    return layer_norm(x, weights["lnf_g"], weights["lnf_b"])


def encode(wave, weights, n_layers: int, dims: EncoderDims = DIMS):
    """Whole path for one clip: log-mel -> stack -> projection -> encoder -> final LN."""
    return encoder_forward(stack_project(stack_frames(log_mel(wave)), weights), weights,
                           n_layers, dims)


# ----------------------------------------------------------------------------- helpers

def param_count(n_layers: int = 32, dims: EncoderDims = DIMS) -> int:
    """Parameters of the projection, the layers and the final LayerNorm ([ARCH-600M])."""
    W, Fd, hd = dims.width, dims.ffn, dims.head_dim
    per_layer = (2 * W                    # LN1
                 + 3 * W * W + 3 * W      # QKV
                 + 2 * hd                 # q and k norm gains
                 + W * W + W              # output projection
                 + 2 * W                  # LN2
                 + W * Fd + Fd + Fd * W + W)  # FFN
    return dims.stack_in * W + W + n_layers * per_layer + 2 * W


def rel_l2(a, ref) -> float:
    """||a - ref|| / ||ref|| in float64."""
    a, ref = _f64(a), _f64(ref)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-300))
