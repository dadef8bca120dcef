"""GPU parity of each C-ABI stage against the fp64 oracle, at small and ragged sizes
(several tiles plus a ragged tail), plus the error paths."""

import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_14_b200 import gptq as G
from post_weight_quantization_14_b200.inputs import bf16_bits_from_f32, f32_from_bf16_bits

from . import gpu_util as U_

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_dev):
    yield


# ---------------------------------------------------------------- packing / dequant

@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("layout", [0, 1])
def test_pack_int_bit_exact(bits, layout):
    rng = np.random.default_rng(bits * 10 + layout)
    rows, cols = 37, 1001
    codes = rng.integers(0, 1 << bits, size=(rows, cols)).astype(np.uint8)
    nw = (cols * bits + 31) // 32
    out = torch.full((rows * nw,), -1, dtype=torch.int32, device=U_.dev())
    G.gptq_pack_int(U_.t(codes), bits, layout, out)
    got = out.cpu().numpy().view(np.uint32)
    ref = O.pack_bitstream(codes, bits)
    if layout == 1:
        ref = ref.T
    np.testing.assert_array_equal(got, ref.reshape(-1))


@pytest.mark.parametrize("bits,g,sym", [(4, 128, False), (3, 64, True), (2, 32, False), (4, -1, False), (8, 16, True)])
def test_dequant_bit_exact(bits, g, sym):
    rng = np.random.default_rng(bits + g)
    d_out, d_in = 70, 256
    codes = rng.integers(0, 1 << bits, size=(d_out, d_in))
    ng = O.n_groups(d_in, g)
    scales = rng.uniform(1e-3, 1e-1, size=(ng, d_out)).astype(np.float16)
    zeros = rng.integers(0, 1 << bits, size=(ng, d_out))
    qw = O.pack_qweight(codes, bits)
    qz = None if sym else O.pack_qzeros(zeros, bits)
    cfg = G.make_config(bits, g, sym)
    out = torch.empty((d_out, d_in), dtype=torch.float32, device=U_.dev())
    G.gptq_dequant(U_.t(qw), U_.t(scales), None if sym else U_.t(qz), d_out, d_in, cfg, out)
    ref = O.dequant_packed(qw, scales, qz, d_out, d_in, bits, g, sym)
    np.testing.assert_array_equal(out.cpu().numpy().astype(np.float64), ref)


# ---------------------------------------------------------------- Hessian

@pytest.mark.parametrize("dtype,n,d_in", [("bf16", 300, 200), ("bf16", 2048, 512), ("bf16", 64, 8),
                                          ("f32", 512, 256), ("f32", 77, 136)])
def test_hessian_matches_fp64(dtype, n, d_in):
    rng = np.random.default_rng(n + d_in)
    Xf = (rng.standard_normal((n, d_in)) * np.exp(rng.standard_normal(d_in))[None, :]).astype(np.float32)
    if dtype == "bf16":
        bits = bf16_bits_from_f32(Xf)
        X = f32_from_bf16_bits(bits)
        Xt = U_.t(bits.view(np.int16)).view(torch.bfloat16)
    else:
        X = Xf
        Xt = U_.t(Xf)
    H = U_.gpu_hessian(Xt)
    ref = O.hessian(X)
    assert U_.rel_fro(H, ref) <= U_.H_TOL
    np.testing.assert_array_equal(H, H.T)   # both triangles written, mirrored exactly


def test_hessian_accumulates_over_batches():
    rng = np.random.default_rng(3)
    X1 = rng.standard_normal((128, 264)).astype(np.float32)
    X2 = rng.standard_normal((200, 264)).astype(np.float32)
    H = torch.zeros((264, 264), dtype=torch.float32, device=U_.dev())
    G.gptq_hessian_accumulate(U_.t(X1), H, accumulate=False)
    G.gptq_hessian_accumulate(U_.t(X2), H, accumulate=True)
    ref = O.hessian(np.concatenate([X1, X2]))
    assert U_.rel_fro(H.cpu().numpy(), ref) <= U_.H_TOL


# ---------------------------------------------------------------- inverse-Hessian factor

@pytest.mark.parametrize("d", [256, 200, 640, 1024, 1152])
def test_prepare_hinv_matches_oracle(d):
    rng = np.random.default_rng(d)
    n = max(64, d // 2)
    X = rng.standard_normal((n, d)) * np.exp(rng.standard_normal(d))[None, :]
    X[:, rng.choice(d, 3, replace=False)] *= 30.0
    H32 = O.hessian(X).astype(np.float32)
    Ug, lam = U_.gpu_hinv(H32)
    Hd, lam_ref = O.damp(H32.astype(np.float64), 0.01)
    Uref = O.hinv_upper_cholesky(Hd)
    assert lam == pytest.approx(lam_ref, rel=1e-6)
    assert np.all(np.tril(Ug, -1) == 0.0)
    assert np.all(np.isfinite(Ug))
    assert U_.rel_fro(Ug, Uref) <= U_.U_TOL


# ---------------------------------------------------------------- column loop given U

CASES = [
    (100, 200, 4, 128, False),
    (256, 256, 4, 128, False),
    (64, 384, 3, 64, True),
    (130, 256, 2, 32, False),
    (48, 512, 4, -1, False),
    (33, 256, 8, 16, False),
    (64, 1024, 4, 128, True),
    (17, 136, 4, 32, False),
    (96, 1152, 4, 128, False),   # a full superblock of deferred updates, then one more block
    (40, 2200, 3, 64, True),     # three superblocks, the last one ragged
]


@pytest.mark.parametrize("d_out,d_in,bits,g,sym", CASES)
def test_quantize_given_U(d_out, d_in, bits, g, sym):
    rng = np.random.default_rng(d_out * 7 + d_in)
    X = rng.standard_normal((max(2 * d_in, 64), d_in)) * np.exp(0.5 * rng.standard_normal(d_in))[None, :]
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    W.reshape(-1)[rng.choice(W.size, max(1, W.size // 1000), replace=False)] *= 10
    Hd, _ = O.damp(O.hessian(X), 0.01)
    U32 = O.hinv_upper_cholesky(Hd).astype(np.float32)
    gpu = U_.gpu_quantize(W, U32, bits, g, sym)
    U_.check_quant(W, U32.astype(np.float64), gpu, bits, g, sym)


def test_identity_hessian_gives_round_to_nearest():
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((96, 384)) * 0.05).astype(np.float32)
    Ug, _ = U_.gpu_hinv(np.eye(384, dtype=np.float32) * 3.0)
    assert np.count_nonzero(Ug - np.diag(np.diag(Ug))) == 0
    gpu = U_.gpu_quantize(W, Ug, 4, 64, False)
    ref = O.rtn(W, 4, 64, False)
    rr = U_.check_quant(W, Ug.astype(np.float64), gpu, 4, 64, False)
    assert rr.forced_codes <= 2
    assert np.count_nonzero(gpu["codes"] != ref.codes) <= 2


def test_degenerate_zero_rows_and_tiny_groups():
    W = np.zeros((20, 256), dtype=np.float32)
    W[3, :] = 1e-12
    W[5, 128:] = np.linspace(-0.5, 0.5, 128, dtype=np.float32)
    U32 = O.hinv_upper_cholesky(np.eye(256) + 0.1 * np.ones((256, 256)) / 256).astype(np.float32)
    for sym in (False, True):
        gpu = U_.gpu_quantize(W, U32, 4, 128, sym)
        U_.check_quant(W, U32.astype(np.float64), gpu, 4, 128, sym)
        assert np.all(gpu["What"][0] == 0.0)
        assert gpu["scales"][0, 0] == 1.0


# ---------------------------------------------------------------- error paths (no device fault)

def test_not_positive_definite_reports_column():
    d = 256
    H = np.eye(d, dtype=np.float32)
    H[200, 200] = -5.0
    U = torch.empty((d, d), dtype=torch.float32, device=U_.dev())
    with pytest.raises(G.GPTQError) as ei:
        G.gptq_prepare_hinv(U_.t(H), U, damp_rel=0.0)
    assert ei.value.status == G.GPTQ_ERR_NOT_PD
    assert ei.value.index == 200


def test_nonfinite_hessian_reported():
    H = np.eye(128, dtype=np.float32)
    H[3, 90] = np.nan
    U = torch.empty((128, 128), dtype=torch.float32, device=U_.dev())
    with pytest.raises(G.GPTQError) as ei:
        G.gptq_prepare_hinv(U_.t(H), U)
    assert ei.value.status == G.GPTQ_ERR_NONFINITE


def test_zero_hessian_is_invalid():
    U = torch.empty((64, 64), dtype=torch.float32, device=U_.dev())
    with pytest.raises(G.GPTQError) as ei:
        G.gptq_prepare_hinv(torch.zeros((64, 64), dtype=torch.float32, device=U_.dev()), U)
    assert ei.value.status == G.GPTQ_ERR_INVALID_ARG


def test_nonfinite_weight_reported_by_sync_status():
    W = np.zeros((16, 128), dtype=np.float32)
    W[7, 9] = np.inf
    U32 = np.eye(128, dtype=np.float32)
    with pytest.raises(G.GPTQError) as ei:
        U_.gpu_quantize(W, U32, 4, 128, False)
    assert ei.value.status == G.GPTQ_ERR_NONFINITE


def test_bounded_wait_times_out_without_hanging():
    G.gptq_selftest_bounded_wait(2_000_000)        # 2 ms limit, nobody arrives
    with pytest.raises(G.GPTQError) as ei:
        G.gptq_sync_status()
    assert ei.value.status == G.GPTQ_ERR_TIMEOUT
    G.gptq_sync_status()                            # cleared; the context stays usable
    x = torch.ones(4, device=U_.dev())
    assert float(x.sum()) == 4.0
