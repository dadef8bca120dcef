"""Helpers shared by the GPU parity tests: run each C-ABI stage from numpy inputs
and apply the parity gates against the fp64 oracle.

Gates (per the benchmark's parity contract):
  H        relative Frobenius error <= 1e-5
  U        relative Frobenius error <= 1e-4
  codes    every mismatch within 1e-5 (weight units) of a rounding boundary, and
           mismatches <= 0.01 % of the weights (teacher-forced replay of the oracle)
  scales   relative error <= 1e-3
  loss     ||(W - W_hat) X^T||_F^2 relative error <= 0.5 %
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_14_b200 import gptq as G

H_TOL = 1e-5
U_TOL = 1e-4
CODE_TOL = 1e-5
CODE_FRAC = 1e-4
SCALE_TOL = 1e-3
LOSS_TOL = 5e-3


def dev():
    return torch.device("cuda:0")


def t(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev())


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def x_tensor(layer) -> torch.Tensor:
    if layer.x_dtype == "bf16":
        return t(layer.X_bits.view(np.int16)).view(torch.bfloat16)
    return t(layer.X)


def gpu_hessian(X: torch.Tensor) -> np.ndarray:
    d = X.shape[1]
    H = torch.empty((d, d), dtype=torch.float32, device=dev())
    G.gptq_hessian_accumulate(X, H)
    torch.cuda.synchronize()
    return H.cpu().numpy()


def gpu_hinv(H32: np.ndarray, damp_rel=0.01):
    d = H32.shape[0]
    U = torch.full((d, d), float("nan"), dtype=torch.float32, device=dev())
    lam = G.gptq_prepare_hinv(t(H32.astype(np.float32)), U, damp_rel)
    return U.cpu().numpy(), lam


def gpu_quantize(W32: np.ndarray, U32: np.ndarray, bits: int, g: int, sym: bool) -> dict:
    d_out, d_in = W32.shape
    cfg = G.make_config(bits, g, sym)
    ng = G.n_groups(d_in, g)
    qw = torch.full(((d_in * bits + 31) // 32, d_out), -1, dtype=torch.int32, device=dev())
    sc = torch.zeros((ng, d_out), dtype=torch.float16, device=dev())
    qz = None if sym else torch.full((ng, (d_out * bits + 31) // 32), -1, dtype=torch.int32, device=dev())
    es = torch.zeros((d_out,), dtype=torch.float32, device=dev())
    W = t(W32.astype(np.float32))
    G.gptq_quantize_layer(W, t(U32.astype(np.float32)), cfg, qw, sc, qz, es)
    G.gptq_sync_status()
    return unpack_outputs(qw, sc, qz, es, d_out, d_in, bits, g, sym)


def unpack_outputs(qw, sc, qz, es, d_out, d_in, bits, g, sym) -> dict:
    qwn = qw.cpu().numpy()
    codes = O.unpack_bitstream(qwn.view(np.uint32).T, bits, d_in)
    scales = sc.cpu().numpy().astype(np.float64)
    ng = scales.shape[0]
    if sym:
        zeros = np.full((ng, d_out), 1 << (bits - 1), dtype=np.int64)
        qzn = None
    else:
        qzn = qz.cpu().numpy()
        zeros = O.unpack_bitstream(qzn.view(np.uint32), bits, d_out)
    cfg = G.make_config(bits, g, sym)
    What = torch.empty((d_out, d_in), dtype=torch.float32, device=dev())
    G.gptq_dequant(qw, sc, qz, d_out, d_in, cfg, What)
    torch.cuda.synchronize()
    return dict(codes=codes, scales=scales, zeros=zeros, err_sq=es.cpu().numpy().astype(np.float64),
                qweight=qwn, qzeros=qzn, What=What.cpu().numpy().astype(np.float64))


def check_quant(W0, U, gpu: dict, bits, g, sym, rows=None):
    """Teacher-forced replay of the oracle against the GPU's codes/scales/zeros."""
    W0 = np.asarray(W0, dtype=np.float64)
    sel = slice(None) if rows is None else rows
    Wr = W0[sel]
    codes = gpu["codes"][sel]
    scales = gpu["scales"][:, sel]
    zeros = gpu["zeros"][:, sel]
    rr = O.gptq_replay(Wr, U, codes, scales, zeros, bits, g, sym, 128, CODE_TOL)
    assert rr.hard_params == 0, f"scale/zero decisions differ away from rounding boundaries: {rr.hard_params}"
    assert rr.hard_codes == 0, f"codes differ away from rounding boundaries: {rr.hard_codes}"
    assert rr.forced_codes <= CODE_FRAC * Wr.size, f"too many near-boundary mismatches {rr.forced_codes}"
    rel = np.abs(scales - rr.own_scales) / np.abs(rr.own_scales)
    assert rel.max() <= SCALE_TOL, rel.max()
    # dequantized weights of the GPU agree with s*(q-z) of its own packed outputs
    g_eff = W0.shape[1] if g == -1 else g
    gi = np.arange(W0.shape[1]) // g_eff
    What = scales[gi, :].T * (codes - zeros[gi, :].T)
    np.testing.assert_array_equal(gpu["What"][sel], What)
    # err_sq identity: sum_c e_c^2 of the GPU equals the replayed oracle's
    np.testing.assert_allclose(gpu["err_sq"][sel], np.sum(rr.err ** 2, axis=1), rtol=2e-3, atol=1e-12)
    return rr
