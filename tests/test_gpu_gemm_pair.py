"""The two-SM GEMM (clusters of two CTAs, tcgen05.mma.cta_group::2, 256 x 256 work units)
against the oracle, for every epilogue, forced on in a child process.

SAL_GEMM_PAIR is read once per process, so a child runs the kernels with it set to 1 and
saves the outputs; this process draws the same seeded bf16 inputs and compares them with
the oracle at the bounds of test_gpu_kernels (one bf16 rounding, fp32 sums). Shapes:
ragged last row blocks (M = 1000 ends with 232 rows, so the odd CTA of the last pair has
104; M = 4100 ends with 4, so that odd CTA has none), K of 1024, 1280 and 5120, and the
QKV epilogue (QK-norm, RoPE, head scatter) over two clips of 700.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle as O
from speech_audio_encoder_b200 import synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [(1000, 1280, 5120), (4100, 1280, 1280), (4100, 5120, 1280), (1400, 1024, 1280)]

CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
from gpu_util import rand_bf16, weights
from speech_audio_encoder_b200 import api
out = {{}}
for (M, K, N) in {shapes!r}:
    A, _ = rand_bf16((M, K), 10 + M, 1.0)
    W, _ = rand_bf16((N, K), 20 + K, 0.02)
    b, _ = rand_bf16((N,), 30 + N, 0.02)
    out[f"f32_{{M}}_{{K}}_{{N}}"] = api.sal_linear(api.SAL_EPI_STORE_F32, A, W, b).cpu().numpy()
    out[f"bf16_{{M}}_{{K}}_{{N}}"] = api.sal_linear(api.SAL_EPI_STORE_BF16, A, W, b).float().cpu().numpy()
    out[f"gelu_{{M}}_{{K}}_{{N}}"] = api.sal_linear(api.SAL_EPI_GELU_BF16, A, W, b).float().cpu().numpy()
    x = torch.from_numpy(np.random.default_rng(M + N).standard_normal((M, N)).astype(np.float32)).cuda()
    api.sal_linear(api.SAL_EPI_RESID_F32, A, W, b, out=x)
    out[f"resid_{{M}}_{{K}}_{{N}}"] = x.cpu().numpy()
_, _, dw = weights(1)
h, _ = rand_bf16((1400, 1280), 41, 1.0)
q, k, v = api.sal_qkv_rope(h, 2, 700, dw.layer(0))
out["q"], out["k"], out["v"] = (t.float().cpu().numpy() for t in (q, k, v))
torch.cuda.synchronize()
assert api.sal_last_device_status() == 0
np.savez({path!r}, **out)
"""


def _vals(shape, seed, std):
    """The float64 values of the child's seeded bf16 inputs (gpu_util.rand_bf16)."""
    return synth.random_bf16(shape, seed, std)[1].astype(np.float64)


def _rms(a):
    return float(np.sqrt(np.mean(np.square(a))))


def _bf16_close(got, ref, what):
    err = np.abs(got - ref)
    bad = err > 2.0 ** -8 * np.abs(ref) + 2e-3 * _rms(ref)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, max err {err.max()}"


def _f32_close(got, ref, what):
    err = np.abs(got - ref)
    bad = err > 1e-4 * _rms(ref) + 1e-5 * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, max err {err.max()}"


@pytest.fixture(scope="module")
def pair_outputs(tmp_path_factory):
    path = str(tmp_path_factory.mktemp("pair") / "out.npz")
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), shapes=SHAPES, path=path)
    env = dict(os.environ, SAL_GEMM_PAIR="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return dict(np.load(path))


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_pair_linear_epilogues(pair_outputs, M, K, N):
    A64 = _vals((M, K), 10 + M, 1.0)
    W64 = _vals((N, K), 20 + K, 0.02)
    b64 = _vals((N,), 30 + N, 0.02)
    ref = O.linear(A64, W64, b64)
    tag = f"{M}_{K}_{N}"
    _f32_close(pair_outputs["f32_" + tag].astype(np.float64), ref, "f32")
    _bf16_close(pair_outputs["bf16_" + tag].astype(np.float64), ref, "bf16")
    _bf16_close(pair_outputs["gelu_" + tag].astype(np.float64), O.gelu(ref), "gelu")
    x0 = np.random.default_rng(M + N).standard_normal((M, N)).astype(np.float32)
    _f32_close(pair_outputs["resid_" + tag].astype(np.float64) - x0, ref, "residual (update)")


def test_pair_qkv_rope(pair_outputs):
    from gpu_util import weights
    _, wf, _ = weights(1)
    lw = {k: v.astype(np.float64) for k, v in wf["layers"][0].items()}
    h64 = _vals((1400, 1280), 41, 1.0)
    qkv = O.linear(h64, lw["w_qkv"], lw["b_qkv"]).reshape(2, 700, 3, 10, 128)
    pos = np.arange(700)
    for b in range(2):
        qr = O.rope(O.rms_norm(qkv[b, :, 0].transpose(1, 0, 2), lw["qn_g"]), pos)
        kr = O.rope(O.rms_norm(qkv[b, :, 1].transpose(1, 0, 2), lw["kn_g"]), pos)
        vr = qkv[b, :, 2].transpose(1, 0, 2)
        _bf16_close(pair_outputs["q"][b].astype(np.float64), qr, "q")
        _bf16_close(pair_outputs["k"][b].astype(np.float64), kr, "k")
        _bf16_close(pair_outputs["v"][b].astype(np.float64), vr, "v")
