"""The row-sharded layer path's host side on CPU: shard arithmetic, and three gloo ranks that
sum H over their token shards and assemble the layer from their row shards.

Rows are independent given U (the serverflow page on GPTQ, section "Как работает GPTQ —
простыми словами": row-wise quantization) and H = 2 X^T X is a sum over tokens (tutorial
"阶段一"), so the assembled layer must equal the oracle's whole-layer result bit for bit,
and the summed H the whole H up to fp64 rounding.  One case leaves the third rank with no
rows, one leaves the last shard ragged.
"""

import json
import os
import subprocess
import sys

import pytest

from post_weight_quantization_14_b200 import shard as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("total,world,align", [(4096, 8, 32), (4096, 3, 32), (100, 3, 32), (33, 4, 32), (0, 2, 32),
                                               (2048, 7, 1), (5, 8, 1)])
def test_shards_cover_disjoint_aligned_balanced(total, world, align):
    parts = [S.shard_range(total, world, r, align) for r in range(world)]
    assert parts[0][0] == 0 and parts[-1][1] == total
    for (a0, a1), (b0, b1) in zip(parts, parts[1:]):
        assert a1 == b0 and a0 <= a1
    for a, b in parts:
        assert (a % align == 0 or a == total) and (b % align == 0 or b == total)
    units = [(b - a + align - 1) // align for a, b in parts]
    assert max(units) - min(units) <= 1
    assert units == sorted(units, reverse=True)


def test_bad_shard_requests():
    for args in [(10, 0, 0), (10, 2, 2), (-1, 2, 0), (10, 2, -1)]:
        with pytest.raises(ValueError):
            S.shard_range(*args)
    with pytest.raises(ValueError):
        S.shard_range(10, 2, 0, 0)


def test_row_shards_keep_packed_zero_words_whole():
    for bits in (2, 3, 4, 8):
        for d_out in (32, 100, 4096, 11008):
            words = 0
            for r in range(5):
                a, b = S.row_shard(d_out, 5, r)
                if b > a and b < d_out:
                    assert (b - a) * bits % 32 == 0
                words += ((b - a) * bits + 31) // 32
            assert words == (d_out * bits + 31) // 32


def test_three_gloo_ranks_sum_h_and_assemble_the_layer(tmp_path):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=3", "--standalone",
           "--local-addr", "127.0.0.1", os.path.join(ROOT, "tests", "rowshard_worker.py")]
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", OMP_NUM_THREADS="1", ROWSHARD_OUT=str(tmp_path))
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=240, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    res = [json.loads((tmp_path / f"rank{k}.json").read_text()) for k in range(3)]
    assert [d["rank"] for d in res] == [0, 1, 2]
    rows = [[d["cases"][c]["rows"] for d in res] for c in range(3)]
    assert rows[0] == [[0, 32], [32, 64], [64, 70]]     # ragged last shard
    assert rows[1] == [[0, 32], [32, 40], [40, 40]]     # the third rank owns no rows
    for d in res:
        for c in d["cases"]:
            assert c["h_rel_err"] < 1e-13
            assert all(c["same"].values()), c
