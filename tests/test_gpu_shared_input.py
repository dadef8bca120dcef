"""GPU parity of quantize_layers_shared_input: several weights reading one input X (the q,
k and v projections of an attention block, or gate and up) share one H, one activation
order and one U; every weight must still meet the parity gates against the fp64 oracle
for that X, in natural and in activation order."""

import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_14_b200 import gptq as G

from . import gpu_util as U_
from .test_gpu_act_order import check_act

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_dev):
    yield


def _inputs(seed, d_outs, d_in, n):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((n, d_in)) * np.exp(0.7 * rng.standard_normal(d_in))[None, :]).astype(np.float32)
    Ws = [(rng.standard_normal((d, d_in)) * 0.02).astype(np.float32) for d in d_outs]
    return X, Ws


@pytest.mark.parametrize("desc_act", [0, 1])
def test_shared_input_layers_meet_the_gates(desc_act):
    d_outs, d_in, n, bits, g = [128, 64, 192], 384, 768, 4, 128
    X, Ws = _inputs(7 + desc_act, d_outs, d_in, n)
    res = G.quantize_layers_shared_input([U_.t(W.copy()) for W in Ws], U_.t(X), bits, g, False, 0.01, desc_act)
    G.gptq_sync_status()
    assert len(res) == 3
    H = O.hessian(X.astype(np.float64))
    if desc_act:
        perm = O.act_order(O.act_abs_sum(X), desc_act)
        Hd, lam = O.damp(H[np.ix_(perm, perm)], 0.01)
    else:
        Hd, lam = O.damp(H, 0.01)
    Uo = O.hinv_upper_cholesky(Hd)
    for W, q in zip(Ws, res):
        assert q.lam == pytest.approx(lam, rel=1e-5)
        out = U_.unpack_outputs(q.qweight, q.scales, q.qzeros, q.err_sq, W.shape[0], d_in, bits, g, False)
        if desc_act:
            np.testing.assert_array_equal(q.perm.cpu().numpy(), perm)
            out["g_idx"] = q.g_idx.cpu().numpy().astype(np.int64)
            What = torch.empty((W.shape[0], d_in), dtype=torch.float32, device=U_.dev())
            G.gptq_dequant_g_idx(q.qweight, q.scales, q.qzeros, q.g_idx, W.shape[0], d_in,
                                 G.make_config(bits, g, False), What)
            out["What"] = What.cpu().numpy().astype(np.float64)
            check_act(W, Uo, perm, out, bits, g, False)
        else:
            U_.check_quant(W, Uo, out, bits, g, False)


def test_shared_input_rejects_mismatched_widths():
    X, Ws = _inputs(3, [64, 64], 256, 256)
    with pytest.raises(ValueError):
        G.quantize_layers_shared_input([U_.t(Ws[0]), U_.t(Ws[1][:, :128].copy())], U_.t(X))
