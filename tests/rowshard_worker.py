"""One rank of the CPU check of the row-sharded layer path (gloo ranks on 127.0.0.1).

Run by tests/test_rowshard_cpu.py through torch.distributed.run.  Every rank draws the
same seeded layer; it forms H from its own calibration tokens with the oracle, sums it
over the ranks with the package's all-reduce, rounds its own output rows with the oracle
(eager column order, so a subset of rows takes exactly the arithmetic of the whole), packs
them in the library's layouts and assembles the layer with gather_row_shards.  It writes
one JSON file (rank<r>.json in the directory ROWSHARD_OUT) with what it checked.
"""

import json
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
from oracle import gptq_oracle as O  # noqa: E402
from post_weight_quantization_14_b200 import gptq as G  # noqa: E402
from post_weight_quantization_14_b200 import shard as S  # noqa: E402


def _layer(q_res, bits, sym):
    qweight = torch.from_numpy(O.pack_qweight(q_res.codes, bits).copy())
    scales = torch.from_numpy(q_res.scales.astype(np.float16))
    qzeros = None if sym else torch.from_numpy(O.pack_qzeros(q_res.zeros, bits).copy())
    err_sq = torch.from_numpy(np.sum(q_res.err ** 2, axis=1).astype(np.float32))
    return G.QuantizedLayer(qweight, scales, qzeros, err_sq, 0.0)


def check(d_out, d_in, n, bits, g, sym, seed, world, rank):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d_in)) * np.exp(0.5 * rng.standard_normal(d_in))[None, :]
    W = rng.standard_normal((d_out, d_in)) * 0.02
    t0, t1 = S.token_shard(n, world, rank)
    r0, r1 = S.row_shard(d_out, world, rank)
    H = torch.from_numpy(O.hessian(X[t0:t1]))
    S.allreduce_sum_(H)
    H_full = O.hessian(X)
    h_err = float(np.max(np.abs(H.numpy() - H_full)) / np.max(np.abs(H_full)))
    Hd, _ = O.damp(H_full, 0.01)
    U = O.hinv_upper_cholesky(Hd)
    mine = _layer(O.gptq(W[r0:r1], U, bits, g, sym, block_size=0), bits, sym)
    whole = _layer(O.gptq(W, U, bits, g, sym, block_size=0), bits, sym)
    got = S.gather_row_shards(S.RowShardedLayer(mine, r0, r1, d_out), bits)
    same = {
        "qweight": bool(torch.equal(got.qweight, whole.qweight)),
        "scales": bool(torch.equal(got.scales, whole.scales)),
        "qzeros": True if sym else bool(torch.equal(got.qzeros, whole.qzeros)),
        "err_sq": bool(torch.equal(got.err_sq, whole.err_sq)),
    }
    return {"rows": [r0, r1], "tokens": [t0, t1], "h_rel_err": h_err, "same": same}


def main() -> None:
    dist.init_process_group("gloo")
    try:
        rank, world = dist.get_rank(), dist.get_world_size()
        out = {"rank": rank, "world": world, "cases": []}
        for d_out, d_in, n, bits, g, sym, seed in [(70, 64, 90, 4, 32, False, 1), (40, 32, 17, 3, 16, False, 2),
                                                   (100, 48, 33, 2, -1, True, 3)]:
            out["cases"].append(check(d_out, d_in, n, bits, g, sym, seed, world, rank))
        dist.barrier()
        with open(os.path.join(os.environ["ROWSHARD_OUT"], f"rank{rank}.json"), "w") as f:
            json.dump(out, f)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
