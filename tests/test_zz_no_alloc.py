"""The fixed-scratch Hessian entry point, for callers that cannot give the library a
device workspace (a C program with no device allocator of its own, or a plug-in whose
host application owns all device memory).  It must produce the same H as the
workspace entry point, on consecutive calls that reuse the library's one scratch array.

Collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from post_weight_quantization_14_b200 import gptq as G
from post_weight_quantization_14_b200.inputs import bf16_bits_from_f32

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


def _rel(a, b):
    return float(torch.linalg.norm((a - b).double()) / torch.linalg.norm(b.double()))


def test_fixed_scratch_matches_workspace_entry_point_on_consecutive_calls():
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(123)
    # call 1: bf16 batch of the largest size the scratch holds (4096 x 2048 tokens)
    Xf = (rng.standard_normal((2048, 4096)) * np.exp(rng.standard_normal(4096))[None, :]).astype(np.float32)
    X1 = torch.from_numpy(bf16_bits_from_f32(Xf).view(np.int16)).to(dev).view(torch.bfloat16)
    # call 2: fp32 batch of a different shape, accumulated onto a fresh H
    X2 = torch.from_numpy(rng.standard_normal((300, 264)).astype(np.float32)).to(dev)
    for X, xt in ((X1, G.GPTQ_BF16), (X2, G.GPTQ_F32)):
        d = X.shape[1]
        ref = torch.zeros((d, d), dtype=torch.float32, device=dev)
        G.gptq_hessian_accumulate(X, ref, accumulate=False)
        G.gptq_hessian_accumulate(X, ref, accumulate=True)
        got = torch.full((d, d), float("nan"), dtype=torch.float32, device=dev)
        assert _fixed(X, got, xt, False) == G.GPTQ_OK, G.lib().gptq_last_error()
        assert _fixed(X, got, xt, True) == G.GPTQ_OK, G.lib().gptq_last_error()
        G.gptq_sync_status()
        assert torch.isfinite(got).all()
        assert _rel(got, ref) <= H_TOL


def test_fixed_scratch_rejects_a_batch_larger_than_the_scratch():
    dev = torch.device("cuda:0")
    X = torch.zeros((2112, 4096), dtype=torch.bfloat16, device=dev)   # 4096 * 2112 * 2 > 16 MiB
    H = torch.zeros((4096, 4096), dtype=torch.float32, device=dev)
    st = _fixed(X, H, G.GPTQ_BF16, False)
    assert st == G.GPTQ_ERR_INVALID_ARG
    msg = G.lib().gptq_last_error().decode()
    assert str(FIXED_SCRATCH_BYTES) in msg
