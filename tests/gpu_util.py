"""Helpers shared by the GPU parity tests (no test functions here)."""
from __future__ import annotations

import functools

import numpy as np
import torch

from speech_audio_encoder_b200 import synth


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def rand_bf16(shape, seed, std=1.0, device="cuda"):
    """(device bf16 tensor, float64 numpy copy of the same values)."""
    bits, vals = synth.random_bf16(shape, seed, std)
    return bf16_tensor(bits, device), vals.astype(np.float64)


@functools.lru_cache(maxsize=4)
def weights(n_layers: int, seed: int = 1000, qk_gain_scale: float = 1.0):
    """(synth weights dict, float64-ready dict, DeviceWeights) cached per process."""
    from speech_audio_encoder_b200 import api
    w = synth.make_weights(n_layers, seed=seed, qk_gain_scale=qk_gain_scale)
    return w, synth.weights_f32(w), api.DeviceWeights(w)


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
