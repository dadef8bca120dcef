"""GPU parity of the dequantizing GEMM Y = X W_hat^T on the packed format against the fp64
oracle, from packed arrays built by the oracle's packers (codes, fp16 scales and zero
points drawn at random).

Tolerance, from the arithmetic: the products x * (q - z) are exact (bf16 times a small
integer), each group's partial sum is accumulated in fp32 on the tensor pipe (K = group
size), scaled once in fp32 and summed over the groups in fp32.  So every output stays
within a small multiple of the fp32 unit roundoff times the absolute-value product
sum_k |x_k| |w_hat_k|; the test allows 2e-5 of that bound, elementwise.
"""

import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_14_b200 import gptq as G
from post_weight_quantization_14_b200.inputs import bf16_bits_from_f32, f32_from_bf16_bits

from . import gpu_util as U_

pytestmark = pytest.mark.gpu

REL_BOUND = 2e-5


@pytest.fixture(autouse=True)
def _need_cuda(cuda_dev):
    yield


def _packed_layer(rng, d_out, d_in, bits, g, sym):
    ng = O.n_groups(d_in, g)
    codes = rng.integers(0, 1 << bits, size=(d_out, d_in))
    scales = rng.uniform(1e-3, 5e-2, size=(ng, d_out)).astype(np.float16)
    zeros = rng.integers(0, 1 << bits, size=(ng, d_out))
    qw = O.pack_qweight(codes, bits)
    qz = None if sym else O.pack_qzeros(zeros, bits)
    return qw, scales, qz


def _run(X_bits, qw, scales, qz, d_out, d_in, bits, g, sym):
    M = X_bits.shape[0]
    cfg = G.make_config(bits, g, sym)
    Y = torch.full((M, d_out), np.nan, dtype=torch.float32, device=U_.dev())
    Xt = U_.t(X_bits.view(np.int16)).view(torch.bfloat16)
    G.gptq_dequant_gemm(Xt, U_.t(qw), U_.t(scales), None if sym else U_.t(qz), d_out, d_in, cfg, Y)
    G.gptq_sync_status()
    return Y.cpu().numpy().astype(np.float64)


def _check(Y, X, qw, scales, qz, d_out, d_in, bits, g, sym, rows=None):
    What = O.dequant_packed(qw, scales, qz, d_out, d_in, bits, g, sym)
    Xs = X if rows is None else X[rows]
    Ys = Y if rows is None else Y[rows]
    ref = Xs @ What.T
    bound = np.abs(Xs) @ np.abs(What).T
    err = np.abs(Ys - ref)
    assert np.all(np.isfinite(Ys))
    assert np.all(err <= REL_BOUND * bound + 1e-30), float(np.max(err / np.maximum(bound, 1e-30)))
    # and the rounding-level agreement is typical, not just within the bound
    assert float(np.median(err / np.maximum(bound, 1e-30))) < 1e-6


CASES = [
    (1, 256, 512, 4, 128, False),      # one token (decode)
    (130, 384, 1024, 4, 128, False),   # ragged M over two tile rows
    (64, 256, 512, 8, 64, True),
    (200, 136, 256, 2, -1, False),     # ragged N, one group per row
    (77, 520, 640, 4, 64, True),
    (300, 1024, 2048, 4, 128, False),
    (16, 4096, 4096, 4, 128, False),   # decode batch at the attention layer's size
]


@pytest.mark.parametrize("M,d_out,d_in,bits,g,sym", CASES)
def test_dequant_gemm_matches_fp64(M, d_out, d_in, bits, g, sym):
    rng = np.random.default_rng(M * 31 + d_out + d_in + bits)
    qw, scales, qz = _packed_layer(rng, d_out, d_in, bits, g, sym)
    Xf = (rng.standard_normal((M, d_in)) * np.exp(rng.standard_normal(d_in))[None, :]).astype(np.float32)
    X_bits = bf16_bits_from_f32(Xf)
    X = f32_from_bf16_bits(X_bits).astype(np.float64)
    Y = _run(X_bits, qw, scales, qz, d_out, d_in, bits, g, sym)
    _check(Y, X, qw, scales, qz, d_out, d_in, bits, g, sym)


def test_dequant_gemm_zero_weights_and_zero_activations():
    # codes equal to their zero points give W_hat = 0 exactly, so Y = 0 exactly; zero X
    # rows give zero Y rows
    rng = np.random.default_rng(4)
    d_out, d_in, bits, g = 128, 256, 4, 128
    zeros = rng.integers(0, 16, size=(2, d_out))
    codes = np.repeat(zeros.T, g, axis=1)
    scales = np.full((2, d_out), 0.01, dtype=np.float16)
    X_bits = bf16_bits_from_f32(rng.standard_normal((40, d_in)).astype(np.float32))
    Y = _run(X_bits, O.pack_qweight(codes, bits), scales, O.pack_qzeros(zeros, bits), d_out, d_in, bits, g, False)
    assert np.all(Y == 0.0)
    X_bits[:] = 0
    qw, sc, qz = _packed_layer(rng, d_out, d_in, bits, g, False)
    assert np.all(_run(X_bits, qw, sc, qz, d_out, d_in, bits, g, False) == 0.0)


@pytest.mark.slow
def test_dequant_gemm_prefill_4096():
    # the attention layer's shape with 2048 tokens (the bench's dequant-GEMM workload)
    rng = np.random.default_rng(2048)
    d_out = d_in = 4096
    qw, scales, qz = _packed_layer(rng, d_out, d_in, 4, 128, False)
    Xf = (rng.standard_normal((2048, d_in)) * np.exp(rng.standard_normal(d_in))[None, :]).astype(np.float32)
    X_bits = bf16_bits_from_f32(Xf)
    X = f32_from_bf16_bits(X_bits).astype(np.float64)
    Y = _run(X_bits, qw, scales, qz, d_out, d_in, 4, 128, False)
    rows = np.sort(rng.choice(2048, 256, replace=False))
    _check(Y, X, qw, scales, qz, d_out, d_in, 4, 128, False, rows=rows)
