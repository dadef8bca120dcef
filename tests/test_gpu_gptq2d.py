"""GPU parity of the GPTQ-2D two-sided rounding (GPTQ-2D summary, "方法" steps 1-3): the
kernel's integers against the oracle's quartic vectorized definition on small matrices and
against the oracle's anti-diagonal route (pinned to the definition on the CPU) on larger
ones, in both kernel paths (error sums in shared memory or in the workspace), and on a
batch.  Both sides round fp64 values, so the integers must agree exactly."""

import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_14_b200 import gptq as G

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_dev):
    yield


def _spd(rng, k):
    A = rng.standard_normal((k, k)) + 2.0 * np.eye(k)
    return A.T @ A + 0.1 * np.eye(k)


def _problem(seed, m, n, batch=None):
    rng = np.random.default_rng(seed)
    UL = O.hinv_upper_cholesky(_spd(rng, m))
    UR = O.hinv_upper_cholesky(_spd(rng, n))
    shape = (m, n) if batch is None else (batch, m, n)
    X = rng.standard_normal(shape) * 3.0
    return X, UL, UR


def _gpu(X, UL, UR):
    dev = torch.device("cuda:0")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    Z = G.gptq_2d_round(t(X), t(UL), t(UR))
    G.gptq_sync_status()
    return Z.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("seed,m,n", [(1, 5, 7), (2, 8, 3), (3, 1, 9), (4, 9, 1), (5, 16, 16), (6, 24, 20),
                                      (7, 33, 31)])
def test_gptq2d_matches_the_vectorized_definition(seed, m, n):
    X, UL, UR = _problem(seed, m, n)
    G_left, G_right = np.linalg.inv(UL.T @ UL), np.linalg.inv(UR.T @ UR)
    ref = O.gptq2d_vectorized(X, G_left, G_right)
    np.testing.assert_array_equal(_gpu(X, UL, UR), ref)


@pytest.mark.parametrize("seed,m,n", [(10, 64, 96), (11, 128, 128), (12, 200, 150), (13, 3, 500)])
def test_gptq2d_matches_the_antidiagonal_route(seed, m, n):
    # 128 x 128 keeps its error sums in shared memory, 200 x 150 in the workspace
    X, UL, UR = _problem(seed, m, n)
    np.testing.assert_array_equal(_gpu(X, UL, UR), O.gptq2d_antidiagonal(X, UL, UR))


def test_gptq2d_batch_shares_the_bases():
    X, UL, UR = _problem(20, 40, 24, batch=6)
    got = _gpu(X, UL, UR)
    for b in range(6):
        np.testing.assert_array_equal(got[b], O.gptq2d_antidiagonal(X[b], UL, UR))


def test_gptq2d_identity_bases_round_to_nearest():
    rng = np.random.default_rng(30)
    X = rng.standard_normal((17, 23)) * 5.0
    np.testing.assert_array_equal(_gpu(X, np.eye(17), np.eye(23)), np.rint(X))


def test_gptq2d_nonfinite_input_is_reported():
    X, UL, UR = _problem(31, 8, 8)
    X[3, 4] = np.nan
    dev = torch.device("cuda:0")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    G.gptq_2d_round(t(X), t(UL), t(UR))
    with pytest.raises(G.GPTQError) as ei:
        G.gptq_sync_status()
    assert ei.value.status == G.GPTQ_ERR_NONFINITE
