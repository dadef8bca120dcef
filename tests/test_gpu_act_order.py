"""GPU parity of activation ordering (desc_act) against the fp64 oracle.

Stages: the per-column activation statistic, the ranking (bit-exact permutation,
ties by column index), the permuted factorization, the column loop in that order
(codes replayed against the oracle in quantization order, g_idx bit-exact), the
g_idx dequantization, and the whole layer through ``quantize_layer(desc_act=...)``
at a small size and at 4096 x 4096 (sampled rows).  Invalid permutations come back
as GPTQ_ERR_INVALID_ARG without any out-of-range access.
"""

import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_14_b200 import gptq as G
from post_weight_quantization_14_b200 import inputs as I
from post_weight_quantization_14_b200.inputs import bf16_bits_from_f32, f32_from_bf16_bits

from . import gpu_util as U_

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_dev):
    yield


def _i32(a):
    return U_.t(np.asarray(a, dtype=np.int32))


def _gpu_order(act: np.ndarray, desc: int):
    d = act.size
    perm = torch.full((d,), -7, dtype=torch.int32, device=U_.dev())
    rank = torch.full((d,), -7, dtype=torch.int32, device=U_.dev())
    G.gptq_act_order(U_.t(act.astype(np.float64)), desc, perm, rank)
    G.gptq_sync_status()
    return perm.cpu().numpy().astype(np.int64), rank.cpu().numpy().astype(np.int64)


def _assert_unique_order(a: np.ndarray):
    # the oracle's sums have no near-ties, so the order is the same on both sides
    s = np.sort(a)
    gaps = np.diff(s) / np.maximum(np.abs(s[1:]), 1e-300)
    assert gaps.min() > 1e-9


# ---------------------------------------------------------------- statistic

@pytest.mark.parametrize("dtype,n,d_in", [("bf16", 300, 200), ("bf16", 2048, 4096), ("f32", 77, 136),
                                          ("f32", 513, 1032), ("bf16", 1, 8)])
def test_act_sum_matches_fp64(dtype, n, d_in):
    rng = np.random.default_rng(n * 3 + d_in)
    Xf = (rng.standard_normal((n, d_in)) * np.exp(rng.standard_normal(d_in))[None, :]).astype(np.float32)
    if dtype == "bf16":
        bits = bf16_bits_from_f32(Xf)
        X = f32_from_bf16_bits(bits)
        Xt = U_.t(bits.view(np.int16)).view(torch.bfloat16)
    else:
        X, Xt = Xf, U_.t(Xf)
    act = torch.full((d_in,), np.nan, dtype=torch.float64, device=U_.dev())
    G.gptq_act_sum_accumulate(Xt, act)
    G.gptq_sync_status()
    np.testing.assert_allclose(act.cpu().numpy(), O.act_abs_sum(X), rtol=1e-13, atol=0)


def test_act_sum_accumulates_over_batches():
    rng = np.random.default_rng(5)
    X1 = rng.standard_normal((100, 264)).astype(np.float32)
    X2 = rng.standard_normal((37, 264)).astype(np.float32)
    act = torch.zeros((264,), dtype=torch.float64, device=U_.dev())
    G.gptq_act_sum_accumulate(U_.t(X1), act, accumulate=False)
    G.gptq_act_sum_accumulate(U_.t(X2), act, accumulate=True)
    np.testing.assert_allclose(act.cpu().numpy(), O.act_abs_sum(np.concatenate([X1, X2])), rtol=1e-13)


def test_act_sum_reports_nonfinite():
    X = np.ones((16, 64), dtype=np.float32)
    X[3, 17] = np.inf
    act = torch.zeros((64,), dtype=torch.float64, device=U_.dev())
    G.gptq_act_sum_accumulate(U_.t(X), act)
    with pytest.raises(G.GPTQError) as ei:
        G.gptq_sync_status()
    assert ei.value.status == G.GPTQ_ERR_NONFINITE
    assert "index 17" in str(ei.value)


# ---------------------------------------------------------------- ranking

@pytest.mark.parametrize("desc", [1, 2])
@pytest.mark.parametrize("d,levels", [(5000, 40), (4096, 0), (1, 0), (1025, 3), (65536, 1000)])
def test_act_order_bit_exact_with_ties(desc, d, levels):
    rng = np.random.default_rng(d + desc)
    # integer levels give many exact ties; levels = 0 gives distinct values
    a = rng.integers(0, levels, d).astype(np.float64) if levels else rng.random(d) * 100
    if d > 3:
        a[:3] = [0.0, -0.0, 0.0]   # both zeros compare equal
    perm, rank = _gpu_order(a, desc)
    ref = O.act_order(a, desc)
    np.testing.assert_array_equal(perm, ref)
    np.testing.assert_array_equal(rank[perm], np.arange(d))


# ---------------------------------------------------------------- permuted factorization

@pytest.mark.parametrize("d", [256, 200, 1152])
def test_prepare_hinv_permuted_matches_oracle(d):
    rng = np.random.default_rng(d + 9)
    X = rng.standard_normal((max(64, d // 2), d)) * np.exp(rng.standard_normal(d))[None, :]
    X[:, rng.choice(d, 3, replace=False)] *= 30.0
    H32 = O.hessian(X).astype(np.float32)
    H32 = np.triu(H32) + np.triu(H32, 1).T            # exactly symmetric, both triangles
    perm = rng.permutation(d)
    U = torch.full((d, d), np.nan, dtype=torch.float32, device=U_.dev())
    lam = G.gptq_prepare_hinv_permuted(U_.t(H32), _i32(perm), U)
    Hd, lam_ref = O.damp(H32.astype(np.float64)[np.ix_(perm, perm)], 0.01)
    Uref = O.hinv_upper_cholesky(Hd)
    Ug = U.cpu().numpy()
    assert lam == pytest.approx(lam_ref, rel=1e-6)
    assert np.all(np.tril(Ug, -1) == 0.0)
    assert U_.rel_fro(Ug, Uref) <= U_.U_TOL


@pytest.mark.parametrize("bad", ["duplicate", "out_of_range", "negative"])
def test_invalid_permutation_is_reported(bad):
    d = 256
    perm = np.arange(d)
    if bad == "duplicate":
        perm[100] = 7
    elif bad == "out_of_range":
        perm[100] = d + 5
    else:
        perm[100] = -3
    H = np.eye(d, dtype=np.float32) * 2.0
    U = torch.empty((d, d), dtype=torch.float32, device=U_.dev())
    with pytest.raises(G.GPTQError) as ei:
        G.gptq_prepare_hinv_permuted(U_.t(H), _i32(perm), U)
    assert ei.value.status == G.GPTQ_ERR_INVALID_ARG
    # the column loop with the same permutation reports it too and leaves the context usable
    cfg = G.make_config(4, 128, False, desc_act=1)
    W = U_.t(np.ones((16, d), dtype=np.float32))
    qw = torch.empty(((d * 4 + 31) // 32, 16), dtype=torch.int32, device=U_.dev())
    sc = torch.empty((2, 16), dtype=torch.float16, device=U_.dev())
    qz = torch.empty((2, 2), dtype=torch.int32, device=U_.dev())
    gi = torch.empty((d,), dtype=torch.int32, device=U_.dev())
    G.gptq_quantize_layer_act_order(W, U_.t(np.eye(d, dtype=np.float32)), _i32(perm), cfg, qw, sc, qz, gi)
    with pytest.raises(G.GPTQError) as ei:
        G.gptq_sync_status()
    assert ei.value.status == G.GPTQ_ERR_INVALID_ARG
    G.gptq_sync_status()
    assert float(torch.ones(3, device=U_.dev()).sum()) == 3.0


# ---------------------------------------------------------------- column loop in a given order

def gpu_quantize_act(W32, U32, perm, bits, g, sym, desc=1) -> dict:
    d_out, d_in = W32.shape
    cfg = G.make_config(bits, g, sym, desc_act=desc)
    ng = G.n_groups(d_in, g)
    qw = torch.full(((d_in * bits + 31) // 32, d_out), -1, dtype=torch.int32, device=U_.dev())
    sc = torch.zeros((ng, d_out), dtype=torch.float16, device=U_.dev())
    qz = None if sym else torch.full((ng, (d_out * bits + 31) // 32), -1, dtype=torch.int32, device=U_.dev())
    gi = torch.full((d_in,), -1, dtype=torch.int32, device=U_.dev())
    es = torch.zeros((d_out,), dtype=torch.float32, device=U_.dev())
    W = U_.t(W32.astype(np.float32))
    G.gptq_quantize_layer_act_order(W, U_.t(U32.astype(np.float32)), _i32(perm), cfg, qw, sc, qz, gi, es)
    G.gptq_sync_status()
    assert np.array_equal(W.cpu().numpy(), W32.astype(np.float32))     # W is read only
    return _unpack_act(qw, sc, qz, gi, es, d_out, d_in, bits, g, sym)


def _unpack_act(qw, sc, qz, gi, es, d_out, d_in, bits, g, sym) -> dict:
    out = U_.unpack_outputs(qw, sc, qz, es, d_out, d_in, bits, g, sym)
    cfg = G.make_config(bits, g, sym)
    What = torch.empty((d_out, d_in), dtype=torch.float32, device=U_.dev())
    G.gptq_dequant_g_idx(qw, sc, qz, gi, d_out, d_in, cfg, What)
    G.gptq_sync_status()
    out["g_idx"] = gi.cpu().numpy().astype(np.int64)
    out["What"] = What.cpu().numpy().astype(np.float64)
    return out


def check_act(W0, U, perm, gpu: dict, bits, g, sym, rows=None):
    """Replay in quantization order: the GPU's codes, moved to that order, against the oracle."""
    np.testing.assert_array_equal(gpu["g_idx"], O.g_idx_of(perm, g))
    # dequantization through g_idx is s[g_idx[c]] * (q - z[g_idx[c]]), in the original order
    gi = gpu["g_idx"]
    What = gpu["scales"][gi, :].T * (gpu["codes"] - gpu["zeros"][gi, :].T)
    np.testing.assert_array_equal(gpu["What"], What)
    permuted = dict(gpu, codes=gpu["codes"][:, perm], What=gpu["What"][:, perm])
    return U_.check_quant(np.asarray(W0, dtype=np.float64)[:, perm], U, permuted, bits, g, sym, rows=rows)


CASES = [
    (100, 200, 4, 128, False),
    (64, 384, 3, 64, True),
    (130, 256, 2, 32, False),
    (48, 512, 4, -1, False),
    (33, 256, 8, 16, False),
    (96, 1152, 4, 128, False),
    (40, 2200, 3, 64, True),
]


@pytest.mark.parametrize("d_out,d_in,bits,g,sym", CASES)
def test_quantize_act_order_given_U(d_out, d_in, bits, g, sym):
    rng = np.random.default_rng(d_out * 11 + d_in)
    X = rng.standard_normal((max(2 * d_in, 64), d_in)) * np.exp(0.5 * rng.standard_normal(d_in))[None, :]
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    perm = O.act_order(O.act_abs_sum(X), 2 if (d_out + bits) % 2 else 1)
    Hd, _ = O.damp(O.hessian(X)[np.ix_(perm, perm)], 0.01)
    U32 = O.hinv_upper_cholesky(Hd).astype(np.float32)
    gpu = gpu_quantize_act(W, U32, perm, bits, g, sym)
    check_act(W, U32.astype(np.float64), perm, gpu, bits, g, sym)


# ---------------------------------------------------------------- whole layer

def _run_layer_act(layer, spec, desc):
    W = U_.t(layer.W)
    X = U_.x_tensor(layer)
    cfg = G.make_config(spec.bits, spec.group_size, spec.sym, 128, spec.damp_rel, desc)
    bufs = G.LayerBuffers(layer.d_out, layer.d_in, layer.n, X.dtype, cfg, U_.dev())
    q = G.quantize_layer(W, X, buffers=bufs)
    G.gptq_sync_status()
    out = _unpack_act(q.qweight, q.scales, q.qzeros, q.g_idx, q.err_sq, layer.d_out, layer.d_in, spec.bits,
                      spec.group_size, spec.sym)
    out["perm"] = q.perm.cpu().numpy().astype(np.int64)
    out["act"] = bufs.act.cpu().numpy()
    out["U"] = bufs.U.cpu().numpy()
    out["lam"] = q.lam
    return out


@pytest.mark.parametrize("desc", [1, 2])
def test_tiny_layer_act_order_end_to_end(desc):
    layer = I.make_layer("tiny", seed=3)
    spec = layer.spec
    gpu = _run_layer_act(layer, spec, desc)
    a = O.act_abs_sum(layer.X)
    np.testing.assert_allclose(gpu["act"], a, rtol=1e-13)
    _assert_unique_order(a)
    perm = O.act_order(a, desc)
    np.testing.assert_array_equal(gpu["perm"], perm)
    ref = O.gptq_act_order(layer.W, O.hessian(layer.X), perm, spec.bits, spec.group_size, spec.sym, 128,
                           spec.damp_rel)
    assert U_.rel_fro(gpu["U"], ref.U) <= U_.U_TOL
    assert gpu["lam"] == pytest.approx(ref.lam, rel=1e-5)
    check_act(layer.W, ref.U, perm, gpu, spec.bits, spec.group_size, spec.sym)
    l_gpu = O.layer_loss(layer.W, gpu["What"], layer.X)
    l_ref = O.layer_loss(layer.W, ref.what, layer.X)
    assert abs(l_gpu - l_ref) <= U_.LOSS_TOL * l_ref


@pytest.mark.slow
def test_attention_projection_4096_act_order():
    layer = I.make_layer("attn", seed=0)
    spec = layer.spec
    gpu = _run_layer_act(layer, spec, 1)
    X = layer.X.astype(np.float64)
    a = O.act_abs_sum(X)
    np.testing.assert_allclose(gpu["act"], a, rtol=1e-13)
    _assert_unique_order(a)
    perm = O.act_order(a, 1)
    np.testing.assert_array_equal(gpu["perm"], perm)
    Hd, lam = O.damp(O.hessian(X)[np.ix_(perm, perm)], spec.damp_rel)
    Uo = O.hinv_upper_cholesky(Hd)
    assert U_.rel_fro(gpu["U"], Uo) <= U_.U_TOL
    rows = np.sort(np.random.default_rng(2).choice(layer.d_out, 256, replace=False))
    check_act(layer.W, Uo, perm, gpu, spec.bits, spec.group_size, spec.sym, rows=rows)
    own = O.gptq(layer.W[rows][:, perm], Uo, spec.bits, spec.group_size, spec.sym, 128)
    l_gpu = O.row_losses(layer.W[rows], gpu["What"][rows], X).sum()
    what = np.empty_like(own.what)
    what[:, perm] = own.what
    l_ref = O.row_losses(layer.W[rows], what, X).sum()
    assert abs(l_gpu - l_ref) <= U_.LOSS_TOL * l_ref
