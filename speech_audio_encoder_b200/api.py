"""Thin Python binding of libsal (include/sal.h): argument marshalling over ctypes.

Every computation runs in the CUDA library; this module only allocates output buffers
with PyTorch (device memory and streams are PyTorch's), passes raw pointers, and turns
status codes into exceptions. There is no CPU fallback: if libsal.so is missing or the
device is not an sm_100 GPU, the calls raise.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsal.so")
# The bounds-checked build (sal.h, "Bounds-checked build"): same calls, every kernel's
# plain global accesses tested against the buffers it was given.
LIB_CHECKED_PATH = os.path.join(_HERE, "libsal_checked.so")

N_MELS, STACK, STACK_DIM, WIDTH, HEADS, HEAD_DIM, FFN = 128, 8, 1024, 1280, 10, 128, 5120
MAX_POSITIONS = 45000

SAL_EPI_STORE_F32, SAL_EPI_STORE_BF16, SAL_EPI_GELU_BF16, SAL_EPI_RESID_F32 = 0, 1, 2, 3

LAYER_FIELDS = ["ln1_g", "ln1_b", "w_qkv", "b_qkv", "qn_g", "kn_g", "w_o", "b_o",
                "ln2_g", "ln2_b", "w1", "b1", "w2", "b2"]


class SalError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


class sal_layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in LAYER_FIELDS]


class sal_weights(ctypes.Structure):
    _fields_ = [("w_proj", ctypes.c_void_p), ("b_proj", ctypes.c_void_p),
                ("layers", ctypes.POINTER(sal_layer)), ("n_layers", ctypes.c_int),
                ("lnf_g", ctypes.c_void_p), ("lnf_b", ctypes.c_void_p)]


class sal_ctc_weights(ctypes.Structure):
    _fields_ = [("w_up", ctypes.c_void_p), ("b_up", ctypes.c_void_p),
                ("layers", ctypes.POINTER(sal_layer)), ("n_layers", ctypes.c_int),
                ("lnf_g", ctypes.c_void_p), ("lnf_b", ctypes.c_void_p),
                ("w_out", ctypes.c_void_p), ("b_out", ctypes.c_void_p)]


class sal_trace(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("events", ctypes.POINTER(ctypes.c_void_p)),
                ("n_events", ctypes.c_int)]


class sal_forward_options(ctypes.Structure):
    _fields_ = [("chunk", ctypes.c_int64), ("trace", ctypes.POINTER(sal_trace)),
                ("window_core", ctypes.c_int64), ("window_context", ctypes.c_int64)]


WINDOW_CORE, WINDOW_CONTEXT = 500, 50  # the serving-window defaults (sal.h)


KIND_NAMES = ["rope_table", "layernorm", "qkv", "attention", "out_proj", "ffn_up", "ffn_down"]

EXPORTS = {
    # name: (restype, argtypes)
    "sal_frame_count": (ctypes.c_int64, [ctypes.c_int64]),
    "sal_position_count": (ctypes.c_int64, [ctypes.c_int64]),
    "sal_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sal_frontend": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p]),
    "sal_stack_project": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                          ctypes.POINTER(sal_weights), ctypes.c_void_p, ctypes.c_void_p]),
    "sal_encoder_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int64]),
    "sal_encoder_workspace_bytes_ex": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int64,
                                                         ctypes.POINTER(sal_forward_options)]),
    "sal_encoder_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                            ctypes.POINTER(sal_weights), ctypes.c_int, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "sal_encoder_forward_ex": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                               ctypes.POINTER(sal_weights), ctypes.c_int, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                               ctypes.POINTER(sal_forward_options)]),
    "sal_launch_count": (ctypes.c_uint64, []),
    "sal_encode_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int64]),
    "sal_encode": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.POINTER(sal_weights),
                                   ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                   ctypes.c_void_p]),
    "sal_last_device_status": (ctypes.c_int, [ctypes.c_void_p]),
    "sal_weights_file_info": (ctypes.c_int, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_int),
                                              ctypes.POINTER(ctypes.c_size_t)]),
    "sal_weights_file_load": (ctypes.c_int, [ctypes.c_char_p, ctypes.c_void_p, ctypes.c_size_t,
                                              ctypes.POINTER(sal_layer), ctypes.c_int, ctypes.POINTER(sal_weights),
                                              ctypes.c_void_p]),
    "sal_checked_build": (ctypes.c_int, []),
    "sal_check_report": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64),
                                         ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                                         ctypes.POINTER(ctypes.c_uint64)]),
    "sal_check_shrink_writable": (None, [ctypes.c_uint64]),
    "sal_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "sal_layernorm": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p]),
    "sal_linear": (ctypes.c_int, [ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                                   ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "sal_qkv_rope": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.POINTER(sal_layer),
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p]),
    "sal_qkv_rope_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                             ctypes.POINTER(sal_layer), ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p]),
    "sal_speaker_fuse": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "sal_connector": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p]),
    "sal_attention": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                      ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]),
    "sal_attention_chunked": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                              ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]),
    "sal_attention_heads": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                            ctypes.c_void_p]),
    "sal_log_softmax": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p]),
    "sal_attention_plan": (ctypes.c_int, [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "sal_attention_withhold": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                               ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                               ctypes.c_void_p]),
    "sal_ctc_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int64]),
    "sal_ctc_adapter": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                        ctypes.POINTER(sal_ctc_weights), ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_size_t, ctypes.c_void_p]),
}

_libs: dict = {}
# SAL_LIB=checked routes every call of this module through the bounds-checked build.
_active = LIB_CHECKED_PATH if os.environ.get("SAL_LIB") == "checked" else LIB_PATH


def _load(path: str) -> ctypes.CDLL:
    if path not in _libs:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run `python -m speech_audio_encoder_b200.build`")
        l = ctypes.CDLL(path)
        for name, (res, args) in EXPORTS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _libs[path] = l
    return _libs[path]


def lib() -> ctypes.CDLL:
    """The loaded library (libsal.so, or libsal_checked.so inside `checked_library()` or
    with SAL_LIB=checked). Raises if it has not been built."""
    return _load(_active)


@contextlib.contextmanager
def checked_library():
    """Calls made inside this block go through libsal_checked.so."""
    global _active
    prev, _active = _active, LIB_CHECKED_PATH
    try:
        yield lib()
    finally:
        _active = prev


def status_string(status: int) -> str:
    return lib().sal_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise SalError(fn, status)


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensors passed to libsal must be contiguous")
        return t.data_ptr()
    return int(t)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ----------------------------------------------------------------------------- counts

def frame_count(n_samples: int) -> int:
    return lib().sal_frame_count(int(n_samples))


def position_count(n_samples: int) -> int:
    return lib().sal_position_count(int(n_samples))


# ----------------------------------------------------------------------------- weights

class DeviceWeights:
    """Encoder parameters in one device buffer, plus the sal_weights record that points into it.

    ``w`` is the nested dict of (bf16 bits, float32) pairs from ``synth.make_weights``.
    """

    def __init__(self, w: dict, device="cuda"):
        names, arrays = [], []
        for k in ("w_proj", "b_proj", "lnf_g", "lnf_b"):
            names.append((None, k))
            arrays.append(w[k][0])
        for i, lw in enumerate(w["layers"]):
            for k in LAYER_FIELDS:
                names.append((i, k))
                arrays.append(lw[k][0])
        offsets, off = [], 0
        for a in arrays:
            offsets.append(off)
            off += (a.size + 127) // 128 * 128  # 256-byte aligned bf16 offsets
        host = np.zeros(off, dtype=np.uint16)
        for a, o in zip(arrays, offsets):
            host[o:o + a.size] = a.reshape(-1)
        self.buffer = torch.from_numpy(host.view(np.int16)).to(device).view(torch.bfloat16)
        base = self.buffer.data_ptr()
        self.n_layers = len(w["layers"])
        self._layers = (sal_layer * max(self.n_layers, 1))()
        self.ptr = {}
        for (i, k), o in zip(names, offsets):
            p = base + 2 * o
            self.ptr[(i, k)] = p
            if i is not None:
                setattr(self._layers[i], k, p)
        self.record = sal_weights(self.ptr[(None, "w_proj")], self.ptr[(None, "b_proj")],
                                  self._layers, self.n_layers, self.ptr[(None, "lnf_g")],
                                  self.ptr[(None, "lnf_b")])

    @classmethod
    def from_file(cls, path: str, device="cuda", stream=None) -> "DeviceWeights":
        """Loads a flat weight file (sal_weights_file_load) into one device buffer."""
        n_layers, nbytes = ctypes.c_int(), ctypes.c_size_t()
        _check("sal_weights_file_info", lib().sal_weights_file_info(os.fsencode(path), ctypes.byref(n_layers),
                                                                    ctypes.byref(nbytes)))
        self = cls.__new__(cls)
        self.buffer = torch.empty(nbytes.value, dtype=torch.uint8, device=device)
        self.n_layers = n_layers.value
        self._layers = (sal_layer * max(self.n_layers, 1))()
        self.record = sal_weights()
        _check("sal_weights_file_load",
               lib().sal_weights_file_load(os.fsencode(path), self.buffer.data_ptr(), nbytes.value, self._layers,
                                           self.n_layers, ctypes.byref(self.record), _stream(stream)))
        self.ptr = {(None, k): getattr(self.record, k) for k in ("w_proj", "b_proj", "lnf_g", "lnf_b")}
        for i in range(self.n_layers):
            for k in LAYER_FIELDS:
                self.ptr[(i, k)] = getattr(self._layers[i], k)
        return self

    def layer(self, i: int) -> sal_layer:
        return self._layers[i]

    def sub(self, first: int, count: int) -> sal_weights:
        """A sal_weights record over layers [first, first + count) (shares this buffer)."""
        arr = ctypes.cast(ctypes.byref(self._layers, first * ctypes.sizeof(sal_layer)),
                          ctypes.POINTER(sal_layer))
        rec = sal_weights(self.record.w_proj, self.record.b_proj, arr, count,
                          self.record.lnf_g, self.record.lnf_b)
        rec._keep = self  # keep the layer array alive
        return rec


class DeviceCtcWeights:
    """CTC adapter parameters in one device buffer, plus the sal_ctc_weights record.

    ``w`` is the dict of (bf16 bits, float32) pairs from ``synth.make_ctc_weights``; w_up
    [2, 1024, 1280] is laid out as the [2048, 1280] the library reads.
    """

    GLOBALS = ("w_up", "b_up", "lnf_g", "lnf_b", "w_out", "b_out")

    def __init__(self, w: dict, device="cuda"):
        names, arrays = [], []
        for k in self.GLOBALS:
            names.append((None, k))
            arrays.append(w[k][0])
        for i, lw in enumerate(w["layers"]):
            for k in LAYER_FIELDS:
                names.append((i, k))
                arrays.append(lw[k][0])
        offsets, off = [], 0
        for a in arrays:
            offsets.append(off)
            off += (a.size + 127) // 128 * 128
        host = np.zeros(off, dtype=np.uint16)
        for a, o in zip(arrays, offsets):
            host[o:o + a.size] = a.reshape(-1)
        self.buffer = torch.from_numpy(host.view(np.int16)).to(device).view(torch.bfloat16)
        base = self.buffer.data_ptr()
        self.n_layers = len(w["layers"])
        self._layers = (sal_layer * max(self.n_layers, 1))()
        ptr = {}
        for (i, k), o in zip(names, offsets):
            ptr[(i, k)] = base + 2 * o
            if i is not None:
                setattr(self._layers[i], k, base + 2 * o)
        g = {k: ptr[(None, k)] for k in self.GLOBALS}
        self.record = sal_ctc_weights(g["w_up"], g["b_up"], self._layers, self.n_layers, g["lnf_g"], g["lnf_b"],
                                      g["w_out"], g["b_out"])


# ----------------------------------------------------------------------------- calls

def sal_frontend(wave: torch.Tensor, stacked: bool = True, stream=None):
    """wave [batch, n] float32 (device) -> (logmel [batch, F, 128] f32, stacked [batch, T, 1024] bf16)."""
    batch, n = wave.shape
    F, T = frame_count(n), position_count(n)
    logmel = torch.empty((batch, F, N_MELS), dtype=torch.float32, device=wave.device)
    st = torch.empty((batch, T, STACK_DIM), dtype=torch.bfloat16, device=wave.device) if stacked else None
    _check("sal_frontend", lib().sal_frontend(_ptr(wave), n, batch, _ptr(logmel), _ptr(st), _stream(stream)))
    return logmel, st


def sal_stack_project(stacked: torch.Tensor, weights: DeviceWeights, stream=None) -> torch.Tensor:
    """stacked [batch, T, 1024] bf16 -> x [batch * T, 1280] float32."""
    batch, T, _ = stacked.shape
    x = torch.empty((batch * T, WIDTH), dtype=torch.float32, device=stacked.device)
    _check("sal_stack_project", lib().sal_stack_project(_ptr(stacked), batch, T, ctypes.byref(weights.record),
                                                        _ptr(x), _stream(stream)))
    return x


def encoder_workspace(batch: int, T: int, device="cuda") -> torch.Tensor:
    n = lib().sal_encoder_workspace_bytes(batch, T)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def sal_encoder_forward(x: torch.Tensor, batch: int, T: int, weights, n_layers: int,
                        workspace: torch.Tensor | None = None, emb: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """x [batch * T, 1280] f32 (clobbered: the residual stream after n_layers) -> emb bf16."""
    rec = weights.record if isinstance(weights, DeviceWeights) else weights
    if workspace is None:
        workspace = encoder_workspace(batch, T, x.device)
    if emb is None:
        emb = torch.empty((batch * T, WIDTH), dtype=torch.bfloat16, device=x.device)
    _check("sal_encoder_forward", lib().sal_encoder_forward(
        _ptr(x), batch, T, ctypes.byref(rec), n_layers, _ptr(emb), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return emb


def encoder_workspace_ex(batch: int, T: int, chunk: int = 0, window_core: int = 0, window_context: int = 0,
                         device="cuda") -> torch.Tensor:
    opts = sal_forward_options(chunk, None, window_core, window_context)
    n = lib().sal_encoder_workspace_bytes_ex(batch, T, ctypes.byref(opts))
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def sal_encoder_forward_ex(x: torch.Tensor, batch: int, T: int, weights, n_layers: int,
                           workspace: torch.Tensor | None = None, emb: torch.Tensor | None = None,
                           chunk: int = 0, kind: int | None = None, events=None, stream=None,
                           window_core: int = 0, window_context: int = 0) -> torch.Tensor:
    """sal_encoder_forward with chunked attention (``chunk`` positions per chunk, 0 = whole
    clip) or serving windows (``window_core`` core positions with ``window_context`` context
    positions on each side, 0 = none) and, optionally, torch.cuda.Event pairs recorded
    around each launch of ``kind``."""
    rec = weights.record if isinstance(weights, DeviceWeights) else weights
    if workspace is None:
        workspace = encoder_workspace_ex(batch, T, chunk, window_core, window_context, x.device)
    if emb is None:
        emb = torch.empty((batch * T, WIDTH), dtype=torch.bfloat16, device=x.device)
    trace_p = None
    if events:
        if any(e.cuda_event == 0 for e in events):
            raise ValueError("record each torch.cuda.Event once before tracing (its handle is created lazily)")
        handles = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        tr = sal_trace(kind, ctypes.cast(handles, ctypes.POINTER(ctypes.c_void_p)), len(events))
        trace_p = ctypes.pointer(tr)
    opts = sal_forward_options(chunk, trace_p, window_core, window_context)
    _check("sal_encoder_forward_ex", lib().sal_encoder_forward_ex(
        _ptr(x), batch, T, ctypes.byref(rec), n_layers, _ptr(emb), _ptr(workspace), workspace.numel(),
        _stream(stream), ctypes.byref(opts)))
    return emb


def sal_launch_count() -> int:
    return int(lib().sal_launch_count())


def encode_workspace(batch: int, n_samples: int, device="cuda") -> torch.Tensor:
    n = lib().sal_encode_workspace_bytes(batch, n_samples)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def sal_encode(wave: torch.Tensor, weights: DeviceWeights, n_layers: int, emb: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Whole path; ``wave`` and ``emb`` may live on the host (pinned or not) or the device."""
    batch, n = wave.shape
    T = position_count(n)
    if workspace is None:
        workspace = encode_workspace(batch, n)
    if emb is None:
        emb = torch.empty((batch, T, WIDTH), dtype=torch.bfloat16, device=wave.device)
    _check("sal_encode", lib().sal_encode(_ptr(wave), n, batch, ctypes.byref(weights.record), n_layers,
                                          _ptr(emb), _ptr(workspace), workspace.numel(), _stream(stream)))
    return emb


def sal_layernorm(x: torch.Tensor, g: int, b: int, stream=None) -> torch.Tensor:
    y = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    _check("sal_layernorm", lib().sal_layernorm(_ptr(x), x.shape[0], g, b, _ptr(y), _stream(stream)))
    return y


def sal_linear(epilogue: int, A: torch.Tensor, W: torch.Tensor, bias: torch.Tensor,
               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    M, K = A.shape
    N = W.shape[0]
    if out is None:
        dt = torch.float32 if epilogue in (SAL_EPI_STORE_F32, SAL_EPI_RESID_F32) else torch.bfloat16
        out = torch.empty((M, N), dtype=dt, device=A.device)
    _check("sal_linear", lib().sal_linear(epilogue, _ptr(A), M, K, _ptr(W), N, _ptr(bias), _ptr(out),
                                          _stream(stream)))
    return out


def sal_qkv_rope(h: torch.Tensor, batch: int, T: int, layer: sal_layer, stream=None):
    shape = (batch, HEADS, T, HEAD_DIM)
    q = torch.empty(shape, dtype=torch.bfloat16, device=h.device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    cs = torch.empty((2, T, 64), dtype=torch.float32, device=h.device)
    _check("sal_qkv_rope", lib().sal_qkv_rope(_ptr(h), batch, T, ctypes.byref(layer), _ptr(q), _ptr(k), _ptr(v),
                                              _ptr(cs), _stream(stream)))
    return q, k, v


def sal_qkv_rope_noalloc(h: torch.Tensor, batch: int, T: int, layer: sal_layer, q: torch.Tensor,
                         k: torch.Tensor, v: torch.Tensor, stream=None):
    """sal_qkv_rope into caller-provided q, k, v [batch, 10, T, 128] bf16; allocates nothing."""
    _check("sal_qkv_rope_noalloc", lib().sal_qkv_rope_noalloc(_ptr(h), batch, T, ctypes.byref(layer), _ptr(q),
                                                              _ptr(k), _ptr(v), _stream(stream)))
    return q, k, v


def sal_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream=None) -> torch.Tensor:
    batch, H, T, hd = q.shape
    o = torch.empty((batch * T, H * hd), dtype=torch.bfloat16, device=q.device)
    _check("sal_attention", lib().sal_attention(_ptr(q), _ptr(k), _ptr(v), batch, T, _ptr(o), _stream(stream)))
    return o


def sal_attention_withhold(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, kernel: int, tile: int,
                           stream=None) -> torch.Tensor:
    """Test hook: sal_attention with key/value tile ``tile`` of every CTA never loaded, so a
    bounded wait gives up (read the outcome with sal_last_device_status)."""
    batch, H, T, hd = q.shape
    o = torch.empty((batch * T, H * hd), dtype=torch.bfloat16, device=q.device)
    _check("sal_attention_withhold", lib().sal_attention_withhold(_ptr(q), _ptr(k), _ptr(v), batch, T, kernel, tile,
                                                                  _ptr(o), _stream(stream)))
    return o


def sal_attention_chunked(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, chunk: int, stream=None) -> torch.Tensor:
    batch, H, T, hd = q.shape
    o = torch.empty((batch * T, H * hd), dtype=torch.bfloat16, device=q.device)
    _check("sal_attention_chunked", lib().sal_attention_chunked(_ptr(q), _ptr(k), _ptr(v), batch, T, chunk,
                                                                _ptr(o), _stream(stream)))
    return o


def sal_speaker_fuse(H: torch.Tensor, P: torch.Tensor, g: torch.Tensor, b: torch.Tensor,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """H [rows, 1280] bf16, P [rows, 8] f32 -> H + LN_8(P > 0.5) K (bf16)."""
    if out is None:
        out = torch.empty_like(H)
    _check("sal_speaker_fuse", lib().sal_speaker_fuse(_ptr(H), _ptr(P), H.shape[0], _ptr(g), _ptr(b), _ptr(out),
                                                      _stream(stream)))
    return out


def sal_connector(x: torch.Tensor, W: torch.Tensor, bias: torch.Tensor, stream=None) -> torch.Tensor:
    """x [rows, 1280] bf16 -> [rows, 2688] bf16."""
    out = torch.empty((x.shape[0], 2688), dtype=torch.bfloat16, device=x.device)
    _check("sal_connector", lib().sal_connector(_ptr(x), x.shape[0], _ptr(W), _ptr(bias), _ptr(out),
                                                _stream(stream)))
    return out


def sal_last_device_status(stream=None) -> int:
    return lib().sal_last_device_status(_stream(stream))


def sal_set_wait_limit_ns(ns: int) -> None:
    lib().sal_set_wait_limit_ns(int(ns))


FILE_IDS = {1: "frontend.cu", 2: "rowops.cu", 3: "gemm.cu", 4: "attention.cu", 5: "ctc.cu"}


def check_report() -> dict:
    """Reads and clears the checked build's record of refused accesses (sal_check_report)."""
    count, addr, seq = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
    f, ln = ctypes.c_int(), ctypes.c_int()
    _check("sal_check_report", lib().sal_check_report(ctypes.byref(count), ctypes.byref(addr), ctypes.byref(f),
                                                       ctypes.byref(ln), ctypes.byref(seq)))
    return {"count": count.value, "first_address": addr.value, "file": FILE_IDS.get(f.value, f.value),
            "line": ln.value, "first_launch": seq.value}


def check_shrink_writable(nbytes: int) -> None:
    """Test hook of the checked build: writable ranges declared from now on end nbytes early."""
    lib().sal_check_shrink_writable(int(nbytes))


CTC_CLASSES = 23863


def ctc_workspace(batch: int, T: int, device="cuda") -> torch.Tensor:
    n = lib().sal_ctc_workspace_bytes(batch, T)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def sal_ctc_adapter(h: torch.Tensor, batch: int, T: int, weights: DeviceCtcWeights,
                    logp: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """Unfused encoder states h [batch * T, 1280] bf16 -> log-probabilities
    [batch * 2T, 23863] float32 on the 40 ms grid."""
    if logp is None:
        logp = torch.empty((batch * 2 * T, CTC_CLASSES), dtype=torch.float32, device=h.device)
    if workspace is None:
        workspace = ctc_workspace(batch, T, h.device)
    _check("sal_ctc_adapter", lib().sal_ctc_adapter(_ptr(h), batch, T, ctypes.byref(weights.record), _ptr(logp),
                                                    _ptr(workspace), workspace.numel(), _stream(stream)))
    return logp


def sal_attention_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream=None) -> torch.Tensor:
    """q, k, v [batch, heads, T, head_dim] bf16 (head_dim 64 or 128) -> o [batch, T, heads * head_dim]."""
    B, H, T, hd = q.shape
    o = torch.empty((B, T, H * hd), dtype=torch.bfloat16, device=q.device)
    _check("sal_attention_heads", lib().sal_attention_heads(_ptr(q), _ptr(k), _ptr(v), B, T, H, hd, _ptr(o),
                                                            _stream(stream)))
    return o


def sal_log_softmax(z: torch.Tensor, n: int | None = None, stream=None) -> torch.Tensor:
    """Row log-softmax of the first n columns of z [rows, ld] float32 -> [rows, n]."""
    rows, ld = z.shape
    n = ld if n is None else n
    out = torch.empty((rows, n), dtype=torch.float32, device=z.device)
    _check("sal_log_softmax", lib().sal_log_softmax(_ptr(z), rows, n, ld, _ptr(out), _stream(stream)))
    return out


def attention_plan(batch: int, T: int, heads: int = 10, head_dim: int = 128, sms: int = 148) -> tuple[int, int]:
    """(pairs for the two-tile kernel, query tiles per clip) that sal_attention would use."""
    p, q = ctypes.c_int(), ctypes.c_int()
    _check("sal_attention_plan", lib().sal_attention_plan(batch, T, heads, head_dim, sms, ctypes.byref(p),
                                                          ctypes.byref(q)))
    return p.value, q.value
