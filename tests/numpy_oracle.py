"""A second fp64 formulation of the oracle in numpy, used only by the tests to
cross-check the C++ oracle (``oracle/sal_oracle.cpp``) function by function.

TEST INFRASTRUCTURE: nothing outside ``tests/`` imports it.

Every function is the plain definition of one step, written in numpy float64. Library
primitives (matrix product, ``erf``, ``exp``) are used as single steps; there is no
blocking or reordering beyond chunking over independent frames or query rows to bound
memory. It shares no code with the C++ oracle: a mistake would have to be made twice,
in two languages and two styles, to pass the cross-check.

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

import math
from dataclasses import dataclass

import numpy as np
from scipy.special import erf as _erf

SAMPLE_RATE = 16000  # [ARCH]
WIN = 400            # 25 ms at 16 kHz [ARCH]
HOP = 160            # 10 ms at 16 kHz [ARCH]
NFFT = 512           # [ARCH]
NBINS = NFFT // 2 + 1
NMEL = 128           # [ARCH]
STACK = 8            # [ARCH]
MEL_FMIN = 0.0       # reading 4
MEL_FMAX = 8000.0    # reading 4
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
    "log_softmax", "ctc_logits", "ctc_adapter", "ctc_param_count",
]


@dataclass(frozen=True)
class EncoderDims:
    """Encoder shape. The defaults are the published ones [ARCH]; tests shrink them."""
    width: int = 1280
    heads: int = 10
    head_dim: int = 128
    ffn: int = 5120          # expansion four [ARCH]
    stack_in: int = NMEL * STACK  # 1024


DIMS = EncoderDims()


# ----------------------------------------------------------------------------- counts

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
    n = np.arange(WIN, dtype=np.float64)
    return 0.5 - 0.5 * np.cos(2.0 * math.pi * n / WIN)


def frame_signal(wave: np.ndarray, first: int = 0, count: int | None = None) -> np.ndarray:
    """Windowed frames y_f[n] = w[n] x[160 f + n], n < 400, for f in [first, first+count)."""
    x = np.asarray(wave, dtype=np.float64)
    F = frame_count(x.shape[0])
    if count is None:
        count = F - first
    idx = (first + np.arange(count))[:, None] * HOP + np.arange(WIN)[None, :]
    return x[idx] * hann_window()[None, :]


def power_spectrum(y: np.ndarray) -> np.ndarray:
    """|X_k|^2 for k = 0..256 of frames zero-padded to 512 samples (reading 3).

    The DFT is the explicit sum X_k = sum_n y[n] exp(-2 pi i k n / 512); the zero padding
    contributes nothing, so the sum runs over the frame's own samples.
    """
    y = np.asarray(y, dtype=np.float64)
    n = np.arange(y.shape[-1], dtype=np.float64)[:, None]
    k = np.arange(NBINS, dtype=np.float64)[None, :]
    ang = 2.0 * math.pi * ((k * n) % NFFT) / NFFT
    re = y @ np.cos(ang)
    im = -(y @ np.sin(ang))
    return re * re + im * im


def hz_to_mel(f):
    """Slaney mel scale: linear 3 f / 200 below 1 kHz, logarithmic above (reading 4)."""
    f = np.asarray(f, dtype=np.float64)
    lin = f * 3.0 / 200.0
    logstep = math.log(6.4) / 27.0
    with np.errstate(divide="ignore"):
        lg = 15.0 + np.log(np.maximum(f, 1e-300) / 1000.0) / logstep
    return np.where(f >= 1000.0, lg, lin)


def mel_to_hz(m):
    """Inverse of :func:`hz_to_mel`."""
    m = np.asarray(m, dtype=np.float64)
    logstep = math.log(6.4) / 27.0
    return np.where(m >= 15.0, 1000.0 * np.exp(logstep * (m - 15.0)), m * 200.0 / 3.0)


def mel_filterbank() -> np.ndarray:
    """128 x 257 Slaney-normalised triangular filters over 0..8 kHz (reading 4)."""
    pts = mel_to_hz(np.linspace(hz_to_mel(MEL_FMIN), hz_to_mel(MEL_FMAX), NMEL + 2))
    fk = np.arange(NBINS, dtype=np.float64) * SAMPLE_RATE / NFFT
    W = np.zeros((NMEL, NBINS), dtype=np.float64)
    for m in range(NMEL):
        rise = (fk - pts[m]) / (pts[m + 1] - pts[m])
        fall = (pts[m + 2] - fk) / (pts[m + 2] - pts[m + 1])
        W[m] = np.maximum(0.0, np.minimum(rise, fall)) * (2.0 / (pts[m + 2] - pts[m]))
    return W


def log_mel(wave: np.ndarray, chunk: int = 8192, first: int = 0,
            count: int | None = None) -> np.ndarray:
    """[F, 128] natural-log mel energies of one clip ([ARCH], readings 1-5).

    ``first``/``count`` select a range of frames; frames are independent, so the range
    is only a way to sample long clips.
    """
    x = np.asarray(wave, dtype=np.float32)
    F = frame_count(x.shape[0])
    if count is None:
        count = F - first
    W = mel_filterbank()
    out = np.empty((count, NMEL), dtype=np.float64)
    for s in range(0, count, chunk):
        c = min(chunk, count - s)
        P = power_spectrum(frame_signal(x, first + s, c))
        out[s:s + c] = np.log(np.maximum(P @ W.T, LOG_FLOOR))
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

def _f64(a):
    return np.asarray(a, dtype=np.float64)


def linear(x, w, b):
    """x W^T + b with W stored [out, in] (reading 7)."""
    return _f64(x) @ _f64(w).T + _f64(b)


def layer_norm(x, g, b, eps: float = LN_EPS):
    """Per-row LayerNorm with two-pass mean and variance (reading 8)."""
    x = _f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    d = x - mu
    var = (d * d).mean(axis=-1, keepdims=True)
    return d / np.sqrt(var + eps) * _f64(g) + _f64(b)


def rms_norm(x, g, eps: float = QK_EPS):
    """x / sqrt(mean(x^2) + eps) * g over the last axis (reading 9)."""
    x = _f64(x)
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * _f64(g)


def rope_angles(positions, head_dim: int):
    """t * base^(-2 i / head_dim) for i < head_dim / 2 (reading 10)."""
    half = head_dim // 2
    inv = ROPE_BASE ** (-2.0 * np.arange(half, dtype=np.float64) / head_dim)
    return _f64(positions)[:, None] * inv[None, :]


def rope(x, positions):
    """Rotate the pairs (i, i + hd/2) of x [..., T, hd] by the angles of ``positions``."""
    x = _f64(x)
    hd = x.shape[-1]
    half = hd // 2
    ang = rope_angles(positions, hd)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def attention_probs(q, k):
    """softmax(q k^T / sqrt(hd)) over keys, with the row maximum subtracted (reading 11)."""
    q, k = _f64(q), _f64(k)
    s = q @ k.T / math.sqrt(q.shape[-1])
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def attention(q, k, v, chunk: int = 2048):
    """Per head: softmax(q k^T / sqrt(hd)) v. q [H, Tq, hd], k and v [H, Tk, hd].

    Query rows are independent, so they are taken ``chunk`` at a time to bound memory.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    out = np.empty(q.shape[:-1] + (v.shape[-1],), dtype=np.float64)
    for h in range(q.shape[0]):
        for s in range(0, q.shape[1], chunk):
            out[h, s:s + chunk] = attention_probs(q[h, s:s + chunk], k[h]) @ v[h]
    return out


def gelu(x):
    """Exact GELU 0.5 x (1 + erf(x / sqrt 2)) (reading 12)."""
    x = _f64(x)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def _split_heads(y, dims: EncoderDims):
    # y [T, width] -> [heads, T, head_dim]
    return y.reshape(y.shape[0], dims.heads, dims.head_dim).transpose(1, 0, 2)


def _qkv(h, lw, dims: EncoderDims, positions):
    """Q, K, V [heads, T, hd] after QK normalisation and RoPE (readings 9, 10)."""
    qkv = linear(h, lw["w_qkv"], lw["b_qkv"])
    W = dims.width
    q = _split_heads(qkv[:, :W], dims)
    k = _split_heads(qkv[:, W:2 * W], dims)
    v = _split_heads(qkv[:, 2 * W:], dims)
    q = rope(rms_norm(q, lw["qn_g"]), positions)
    k = rope(rms_norm(k, lw["kn_g"]), positions)
    return q, k, v


def encoder_layer(x, lw, dims: EncoderDims = DIMS):
    """One pre-norm bidirectional Transformer layer on one clip x [T, width] ([ARCH]).

    x + Attn(LN1(x)), then + FFN(LN2(.)), with the attention over all T positions.
    """
    x = _f64(x)
    T = x.shape[0]
    q, k, v = _qkv(layer_norm(x, lw["ln1_g"], lw["ln1_b"]), lw, dims, np.arange(T))
    o = attention(q, k, v).transpose(1, 0, 2).reshape(T, dims.width)
    x = x + linear(o, lw["w_o"], lw["b_o"])
    u = gelu(linear(layer_norm(x, lw["ln2_g"], lw["ln2_b"]), lw["w1"], lw["b1"]))
    return x + linear(u, lw["w2"], lw["b2"])


def encoder_layer_rows(x, lw, rows, dims: EncoderDims = DIMS):
    """:func:`encoder_layer` evaluated only at the positions ``rows`` of one clip.

    Keys and values still come from every position; everything after attention is
    per position, so the selected rows equal the same rows of the full layer.
    """
    x = _f64(x)
    rows = np.asarray(rows)
    T = x.shape[0]
    h = layer_norm(x, lw["ln1_g"], lw["ln1_b"])
    _, k, v = _qkv(h, lw, dims, np.arange(T))
    q, _, _ = _qkv(h[rows], lw, dims, rows)
    o = attention(q, k, v).transpose(1, 0, 2).reshape(len(rows), dims.width)
    xr = x[rows] + linear(o, lw["w_o"], lw["b_o"])
    u = gelu(linear(layer_norm(xr, lw["ln2_g"], lw["ln2_b"]), lw["w1"], lw["b1"]))
    return xr + linear(u, lw["w2"], lw["b2"])


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
    s = np.arange(n_slots, dtype=np.float64)[:, None]
    w = ROPE_BASE ** (-2.0 * np.arange(width // 2, dtype=np.float64) / width)[None, :]
    K = np.empty((n_slots, width), dtype=np.float64)
    K[:, 0::2] = np.sin(s * w)
    K[:, 1::2] = np.cos(s * w)
    return K


def speaker_fuse(H, P, g, b, scale: float = 1.0):
    """H + scale * LN_slots(P > 0.5) K ([FUSE], readings 13-15). H [T, 1280], P [T, 8]."""
    A = (np.asarray(P, dtype=np.float64) > 0.5).astype(np.float64)
    return _f64(H) + scale * layer_norm(A, g, b) @ speaker_kernel(A.shape[1], H.shape[1])


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
        U[j::2] = h @ w[j].T + _f64(b_up)
    return U


def log_softmax(z):
    """log(softmax(z)) over the last axis, with the row maximum subtracted (reading 21)."""
    z = _f64(z)
    m = z.max(axis=-1, keepdims=True)
    return z - m - np.log(np.exp(z - m).sum(axis=-1, keepdims=True))


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
