"""GPU parity of gptq_layer_loss against the fp64 oracle's layer_loss / row_losses
(E = ||(W - W_hat) X^T||_F^2, tutorial "阶段一").

The kernel splits D = W - W_hat and X into bf16 pairs and forms Y = D X^T as three bf16
products with fp32 accumulation.  Each operand's pair represents it to 2^-18 relative
(hi and lo both rounded to nearest), the dropped lo lo product is below 2^-18 relative,
and fp32 accumulation of K terms adds at most (K + 2) 2^-23 relative (truncating adds
allowed).  So |Y_gpu - Y| <= delta = (3 2^-18 + (K + 2) 2^-23) sum_k |D_ok| |X_tk|, and
each row's loss lies within sum_t (2 |Y_ot| delta_ot + delta_ot^2) of the oracle's: the
test computes that bound from the inputs in fp64 and checks every row and the total
against it (plus the fp64 summation's own rounding, far smaller).
"""

import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_14_b200 import gptq as G

from . import gpu_util as U_

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_dev):
    yield


def _inputs(seed, d_out, d_in, n, x_bf16):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((n, d_in)) * np.exp(0.7 * rng.standard_normal(d_in))[None, :]).astype(np.float32)
    if x_bf16:
        X = torch.from_numpy(X).to(torch.bfloat16).float().numpy()   # bf16-representable values
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    s = 0.004
    W_hat = (s * np.rint(W / s)).astype(np.float32)
    return X, W, W_hat


def _bound(X, W, W_hat):
    D = W.astype(np.float64) - W_hat.astype(np.float64)
    K = X.shape[1]
    Y = D @ X.astype(np.float64).T
    delta = (3 * 2.0 ** -18 + (K + 2) * 2.0 ** -23) * (np.abs(D) @ np.abs(X.astype(np.float64)).T)
    rows = np.sum(2 * np.abs(Y) * delta + delta * delta, axis=1)
    return rows


def _gpu(X, W, W_hat, x_bf16):
    Xd = U_.t(X).to(torch.bfloat16) if x_bf16 else U_.t(X)
    row = torch.empty((W.shape[0],), dtype=torch.float64, device=U_.dev())
    loss = G.gptq_layer_loss(U_.t(W), U_.t(W_hat), Xd, row_loss=row)
    G.gptq_sync_status()
    return float(loss.item()), row.cpu().numpy()


@pytest.mark.parametrize("d_out,d_in,n,x_bf16", [(200, 384, 300, False), (200, 384, 300, True), (1, 8, 1, False),
                                                 (130, 136, 5, True), (1024, 1024, 512, True)])
def test_layer_loss_matches_the_oracle_within_its_bound(d_out, d_in, n, x_bf16):
    X, W, W_hat = _inputs(d_out + n, d_out, d_in, n, x_bf16)
    total, rows = _gpu(X, W, W_hat, x_bf16)
    ref_rows = O.row_losses(W, W_hat, X)
    ref = O.layer_loss(W, W_hat, X)
    bound = _bound(X, W, W_hat)
    slack = 1e-12 * np.abs(ref_rows) + 1e-300
    assert np.all(np.abs(rows - ref_rows) <= bound + slack)
    assert abs(total - ref) <= bound.sum() + 1e-12 * abs(ref)
    assert abs(total - ref) <= 1e-4 * ref


def test_layer_loss_is_deterministic_and_zero_for_equal_weights():
    X, W, W_hat = _inputs(3, 300, 256, 200, False)
    a = _gpu(X, W, W_hat, False)
    b = _gpu(X, W, W_hat, False)
    assert a[0] == b[0] and np.array_equal(a[1], b[1])
    z, zr = _gpu(X, W, W.copy(), False)
    assert z == 0.0 and not zr.any()


def test_layer_loss_of_a_quantized_layer():
    """The loss of a GPU-quantized layer (dequantized W_hat) equals the oracle's loss of that W_hat."""
    d_out, d_in, n = 256, 512, 640
    rng = np.random.default_rng(9)
    X = (rng.standard_normal((n, d_in)) * np.exp(0.7 * rng.standard_normal(d_in))[None, :]).astype(np.float32)
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    q = G.quantize_layer(U_.t(W.copy()), U_.t(X), 4, 128, False, 0.01, 0)
    What = torch.empty((d_out, d_in), dtype=torch.float32, device=U_.dev())
    G.gptq_dequant(q.qweight, q.scales, q.qzeros, d_out, d_in, G.make_config(4, 128, False), What)
    W_hat = What.cpu().numpy()
    total, rows = _gpu(X, W, W_hat, False)
    ref = O.layer_loss(W, W_hat, X)
    assert abs(total - ref) <= _bound(X, W, W_hat).sum() + 1e-12 * ref


def test_layer_loss_rejects_bad_shapes():
    X, W, W_hat = _inputs(1, 16, 64, 8, False)
    with pytest.raises(ValueError):
        G.gptq_layer_loss(U_.t(W), U_.t(W_hat[:, :32].copy()), U_.t(X))
    with pytest.raises(ValueError):
        G.gptq_layer_loss(U_.t(W), U_.t(W_hat), U_.t(X[:, :32].copy()))
