"""The fixed-scratch Hessian entry point, for callers that cannot give the library a
device workspace: a C program that links only this library and has no device allocator
of its own, or a plug-in running inside a host application whose memory pool owns the
device and forbids further cudaMalloc calls.  It runs the same kernels as the workspace
entry point (scratch in a fixed array inside the library instead of the caller's
workspace), so it must return the same H, bit for bit, on consecutive calls that reuse
the library's one scratch array, and that H must meet the 1e-5 Hessian gate against
the fp64 oracle, including on activations whose Hessian nearly cancels (ReLU^2-like,
all non-negative) and on long fp32 batches (many accumulation steps).

Collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test.
"""

import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_14_b200 import gptq as G
from post_weight_quantization_14_b200 import inputs as I

pytestmark = pytest.mark.gpu

FIXED_SCRATCH_BYTES = 16 << 20
H_TOL = 1e-5


@pytest.fixture(autouse=True)
def _need_cuda(cuda_dev):
    yield


def _fixed(X: torch.Tensor, H: torch.Tensor, xt: int, accumulate: bool) -> int:
    n, d_in = X.shape
    return G.lib().gptq_hessian_accumulate_fixed_scratch(
        X.data_ptr(), xt, n, d_in, H.data_ptr(), int(accumulate), torch.cuda.current_stream().cuda_stream or None)


def _rel(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a.astype(np.float64) - b) / np.linalg.norm(b))


def _batches():
    """(name, X on the device, dtype code, the exact fp64 values of X)."""
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(123)
    out = []
    # bf16, the largest batch the scratch holds: 2048 tokens x 4096 lognormal-scaled channels
    Xf = (rng.standard_normal((2048, 4096)) * np.exp(rng.standard_normal(4096))[None, :]).astype(np.float32)
    bits = I.bf16_bits_from_f32(Xf)
    out.append(("bf16 lognormal 2048x4096", torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16),
                G.GPTQ_BF16, I.f32_from_bf16_bits(bits).astype(np.float64)))
    # bf16 ReLU^2-like activations (60 % zeros, the rest half-normal): a near-cancelling Hessian
    Xr = I._x_relu2(rng, 1024, 4096)
    bits = I.bf16_bits_from_f32(Xr.astype(np.float32))
    out.append(("bf16 relu2 1024x4096", torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16),
                G.GPTQ_BF16, I.f32_from_bf16_bits(bits).astype(np.float64)))
    # fp32, narrow and long: 16384 tokens x 64 channels (3xTF32 path, many k-steps)
    X3 = (np.abs(rng.standard_normal((16384, 64))) * np.exp(rng.standard_normal(64))[None, :]).astype(np.float32)
    out.append(("fp32 16384x64", torch.from_numpy(X3).to(dev), G.GPTQ_F32, X3.astype(np.float64)))
    # fp32, an odd shape
    X4 = rng.standard_normal((300, 264)).astype(np.float32)
    out.append(("fp32 300x264", torch.from_numpy(X4).to(dev), G.GPTQ_F32, X4.astype(np.float64)))
    return out


@pytest.mark.parametrize("case", range(4))
def test_fixed_scratch_matches_workspace_entry_point_on_consecutive_calls(case):
    name, X, xt, X64 = _batches()[case]
    dev = X.device
    d = X.shape[1]
    ref = torch.zeros((d, d), dtype=torch.float32, device=dev)
    G.gptq_hessian_accumulate(X, ref, accumulate=False)
    G.gptq_hessian_accumulate(X, ref, accumulate=True)
    got = torch.full((d, d), float("nan"), dtype=torch.float32, device=dev)
    assert _fixed(X, got, xt, False) == G.GPTQ_OK, G.lib().gptq_last_error()
    assert _fixed(X, got, xt, True) == G.GPTQ_OK, G.lib().gptq_last_error()
    G.gptq_sync_status()
    assert torch.isfinite(got).all(), name
    # the same kernels: the same bits as the workspace entry point
    assert torch.equal(got, ref), name
    # and the Hessian gate against the oracle (two batches accumulated: 2 * 2 X^T X)
    H = 2.0 * O.hessian(X64)
    assert _rel(got.cpu().numpy(), H) <= H_TOL, (name, _rel(got.cpu().numpy(), H))


def test_fixed_scratch_rejects_a_batch_larger_than_the_scratch():
    dev = torch.device("cuda:0")
    X = torch.zeros((2112, 4096), dtype=torch.bfloat16, device=dev)   # 4096 * 2112 * 2 > 16 MiB
    H = torch.zeros((4096, 4096), dtype=torch.float32, device=dev)
    st = _fixed(X, H, G.GPTQ_BF16, False)
    assert st == G.GPTQ_ERR_INVALID_ARG
    msg = G.lib().gptq_last_error().decode()
    assert str(FIXED_SCRATCH_BYTES) in msg
