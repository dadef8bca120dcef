"""GPU checks of the row-sharded layer path on one B200.

Output rows are independent given U (the serverflow page on GPTQ, "Как работает GPTQ —
простыми словами") and H = 2 X^T X is a sum over tokens (tutorial "阶段一").  On one GPU:
  * three shards emulated stage by stage: H summed over three token shards by the Hessian
    kernel (accumulate), then each row shard quantized on its own with the shared U.  The
    rows must come out bit-identical to one call on the whole W with that U, and the
    assembled layer must meet the parity gates against the fp64 oracle;
  * quantize_layer_row_sharded in a one-rank NCCL group must equal quantize_layer bit for
    bit (the all-reduce of one rank leaves H as it is), with and without activation order.
"""

import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from oracle import gptq_oracle as O
from post_weight_quantization_14_b200 import gptq as G
from post_weight_quantization_14_b200 import shard as S

from . import gpu_util as U_

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_dev):
    yield


def _inputs(seed, d_out, d_in, n):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal((n, d_in)) * np.exp(0.7 * rng.standard_normal(d_in))[None, :]).astype(np.float32)
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    return X, W


def test_emulated_three_shards_match_the_whole_layer():
    d_out, d_in, n, bits, g, world = 300, 384, 700, 4, 128, 3
    X, W = _inputs(21, d_out, d_in, n)
    Xd = U_.t(X)
    H = torch.empty((d_in, d_in), dtype=torch.float32, device=U_.dev())
    for r in range(world):
        t0, t1 = S.token_shard(n, world, r)
        G.gptq_hessian_accumulate(Xd[t0:t1], H, accumulate=r > 0)
    U = torch.empty_like(H)
    G.gptq_prepare_hinv(H, U, 0.01)
    cfg = G.make_config(bits, g, False)
    ng = G.n_groups(d_in, g)

    def run(Wpart):
        rows = Wpart.shape[0]
        out = dict(qw=torch.empty(((d_in * bits + 31) // 32, rows), dtype=torch.int32, device=U_.dev()),
                   sc=torch.empty((ng, rows), dtype=torch.float16, device=U_.dev()),
                   qz=torch.empty((ng, (rows * bits + 31) // 32), dtype=torch.int32, device=U_.dev()),
                   es=torch.empty((rows,), dtype=torch.float32, device=U_.dev()))
        G.gptq_quantize_layer(U_.t(Wpart.copy()), U, cfg, out["qw"], out["sc"], out["qz"], out["es"])
        return out

    whole = run(W)
    parts = []
    for r in range(world):
        r0, r1 = S.row_shard(d_out, world, r)
        parts.append(run(W[r0:r1]))
    G.gptq_sync_status()
    cat = {k: torch.cat([p[k] for p in parts], dim=-1) for k in whole}
    for k in whole:
        assert torch.equal(cat[k], whole[k]), k
    out = U_.unpack_outputs(cat["qw"], cat["sc"], cat["qz"], cat["es"], d_out, d_in, bits, g, False)
    Hd, _ = O.damp(O.hessian(X.astype(np.float64)), 0.01)
    U_.check_quant(W, O.hinv_upper_cholesky(Hd), out, bits, g, False)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture
def nccl_one_rank():
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", world_size=1, rank=0,
                            device_id=torch.device("cuda:0"))
    try:
        yield
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("desc_act", [0, 1])
def test_one_rank_nccl_group_equals_quantize_layer(nccl_one_rank, desc_act):
    d_out, d_in, n, bits, g = 200, 256, 512, 4, 64
    X, W = _inputs(5 + desc_act, d_out, d_in, n)
    ref = G.quantize_layer(U_.t(W.copy()), U_.t(X), bits, g, False, 0.01, desc_act)
    ref = {k: getattr(ref, k).clone() if getattr(ref, k) is not None else None
           for k in ("qweight", "scales", "qzeros", "err_sq", "g_idx", "perm")}
    sh = S.quantize_layer_row_sharded(U_.t(W.copy()), U_.t(X), d_out, bits, g, False, 0.01, desc_act)
    assert (sh.row0, sh.row1) == (0, d_out)
    got = S.gather_row_shards(sh, bits)
    for k, v in ref.items():
        if v is None:
            assert getattr(got, k) is None
        else:
            assert torch.equal(getattr(got, k), v), k


def test_row_sharded_rejects_a_wrong_row_count():
    X, W = _inputs(1, 64, 128, 64)
    with pytest.raises(ValueError):
        S.quantize_layer_row_sharded(U_.t(W[:10].copy()), U_.t(X), 64)
