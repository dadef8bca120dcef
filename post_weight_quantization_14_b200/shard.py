"""One layer quantized by several ranks: tokens and output rows split across a process group.

Two facts make the layer shard.  H = 2 X^T X is a sum over calibration tokens (tutorial
"阶段一", the Hessian of the layer's squared output error), so each rank forms the part of
H from its own tokens and one sum over ranks (an all-reduce) gives every rank the whole H.
And given U, every output row of W is rounded on its own (the serverflow page "GPTQ:
практическое квантование языковых моделей без потери смысла", section "Как работает GPTQ —
простыми словами": row-wise quantization), so each rank runs the column loop on its own
rows only.  The one exchange is the all-reduce of H (plus the column activity sums with
activation ordering); every rank then factors the identical H itself (the factorization is
deterministic: the same H gives the same U bits on every rank), which costs no more time
than factoring on one rank and broadcasting U, and needs no second exchange.

Shards are contiguous: tokens in near-equal runs, rows in runs whose boundaries are
multiples of ROW_ALIGN, so that no int32 word of the packed zero points straddles two
ranks (32 rows are whole words for 2, 3, 4 and 8 bits).  The collectives are
torch.distributed's (NCCL between GPUs); they run on the current CUDA stream's order.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import gptq as G

ROW_ALIGN = 32


def shard_range(total: int, world: int, rank: int, align: int = 1) -> tuple[int, int]:
    """[start, stop) of rank's part of ``total`` items split over ``world`` ranks in runs whose
    boundaries are multiples of ``align``; earlier ranks get the longer runs, and a rank may
    get an empty run when there are fewer aligned units than ranks."""
    if world < 1 or not 0 <= rank < world or total < 0 or align < 1:
        raise ValueError(f"bad shard request: total={total} world={world} rank={rank} align={align}")
    units = (total + align - 1) // align
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return min(total, u0 * align), min(total, u1 * align)


def row_shard(d_out: int, world: int, rank: int) -> tuple[int, int]:
    """The output rows [r0, r1) quantized by ``rank``."""
    return shard_range(d_out, world, rank, ROW_ALIGN)


def token_shard(n: int, world: int, rank: int) -> tuple[int, int]:
    """The calibration tokens [t0, t1) whose part of H ``rank`` forms."""
    return shard_range(n, world, rank, 1)


def _world(group) -> tuple[int, int]:
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def allreduce_sum_(t: torch.Tensor, group=None) -> torch.Tensor:
    """t <- the sum of every rank's t (in place); a no-op without a process group."""
    world, _ = _world(group)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


@dataclass
class RowShardedLayer:
    """This rank's part of a row-sharded layer: the outputs of rows [row0, row1) of d_out, in
    the layouts of QuantizedLayer for a layer of row1 - row0 rows.  With activation ordering
    layer.perm is set on every rank and layer.g_idx on every rank that owns rows."""
    layer: G.QuantizedLayer
    row0: int
    row1: int
    d_out: int


def quantize_layer_row_sharded(W_rows: torch.Tensor, X_tokens: torch.Tensor, d_out: int, bits=4, group_size=128,
                               sym=False, damp_rel=0.01, desc_act=0, group=None) -> RowShardedLayer:
    """GPTQ of one layer by all ranks of ``group`` (the default group when None).

    W_rows: this rank's rows W[r0:r1] (fp32, [r1 - r0, d_in]) with (r0, r1) = row_shard(d_out,
    world, rank); overwritten with natural order, as in quantize_layer.  X_tokens: this rank's
    calibration tokens (bf16 or fp32, [n_rank, d_in], n_rank >= 1), any split of the layer's
    tokens.  Every rank must call this with the same d_out, d_in and configuration; the ranks
    take the same collective steps in the same order.  The result holds this rank's rows;
    gather_row_shards assembles the whole layer."""
    world, rank = _world(group)
    r0, r1 = row_shard(d_out, world, rank)
    if W_rows.dim() != 2 or X_tokens.dim() != 2 or W_rows.shape[1] != X_tokens.shape[1]:
        raise ValueError("W_rows must be [rows, d_in] and X_tokens [n_rank, d_in]")
    if W_rows.shape[0] != r1 - r0:
        raise ValueError(f"rank {rank} of {world} owns rows [{r0}, {r1}) of {d_out}; W_rows has {W_rows.shape[0]}")
    if X_tokens.shape[0] < 1:
        raise ValueError("every rank needs at least one calibration token")
    d_in = W_rows.shape[1]
    cfg = G.make_config(bits, group_size, sym, 128, damp_rel, desc_act)
    dev = X_tokens.device
    L = G.lib()
    xt = G.GPTQ_BF16 if X_tokens.dtype == torch.bfloat16 else G.GPTQ_F32
    rows = r1 - r0
    ws = max(L.gptq_hessian_workspace_bytes(X_tokens.shape[0], d_in, xt), L.gptq_prepare_hinv_workspace_bytes(d_in),
             L.gptq_quantize_workspace_bytes(max(rows, 1), d_in, ctypes.byref(cfg)))
    ws = G._workspace(ws, dev)
    H = torch.empty((d_in, d_in), dtype=torch.float32, device=dev)
    U = torch.empty((d_in, d_in), dtype=torch.float32, device=dev)
    lam = torch.zeros((1,), dtype=torch.float32, device=dev)

    G.gptq_hessian_accumulate(X_tokens, H, accumulate=False, workspace=ws)
    allreduce_sum_(H, group)
    perm = None
    if desc_act:
        act = torch.empty((d_in,), dtype=torch.float64, device=dev)
        perm = torch.empty((d_in,), dtype=torch.int32, device=dev)
        rk = torch.empty((d_in,), dtype=torch.int32, device=dev)
        G.gptq_act_sum_accumulate(X_tokens, act, accumulate=False)
        allreduce_sum_(act, group)
        G.gptq_act_order(act, desc_act, perm, rk)
    G.gptq_prepare_hinv_async(H, U, damp_rel, workspace=ws, lam=lam, perm=perm)

    ng = G.n_groups(d_in, group_size)
    qweight = torch.empty(((d_in * bits + 31) // 32, rows), dtype=torch.int32, device=dev)
    scales = torch.empty((ng, rows), dtype=torch.float16, device=dev)
    qzeros = None if sym else torch.empty((ng, (rows * bits + 31) // 32), dtype=torch.int32, device=dev)
    err_sq = torch.empty((rows,), dtype=torch.float32, device=dev)
    g_idx = torch.empty((d_in,), dtype=torch.int32, device=dev) if desc_act and rows > 0 else None
    if rows > 0 and desc_act:
        G.gptq_quantize_layer_act_order(W_rows, U, perm, cfg, qweight, scales, qzeros, g_idx, err_sq, workspace=ws)
    elif rows > 0:
        G.gptq_quantize_layer(W_rows, U, cfg, qweight, scales, qzeros, err_sq, workspace=ws)
    G.gptq_sync_status()
    q = G.QuantizedLayer(qweight, scales, qzeros, err_sq, float(lam.item()), g_idx, perm)
    return RowShardedLayer(q, r0, r1, d_out)


def _gather_cols(local: torch.Tensor, counts: list[int], group) -> torch.Tensor:
    """Concatenate every rank's ``local`` along its last dimension (rank order); the ranks'
    widths are ``counts``.  Each part is padded to the widest for the all-gather."""
    width = max(counts)
    pad = torch.zeros(local.shape[:-1] + (width,), dtype=local.dtype, device=local.device)
    pad[..., :local.shape[-1]] = local
    parts = [torch.empty_like(pad) for _ in counts]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([p[..., :c] for p, c in zip(parts, counts)], dim=-1).contiguous()


def gather_row_shards(shard: RowShardedLayer, bits: int, group=None) -> G.QuantizedLayer:
    """The whole layer on every rank from the ranks' RowShardedLayer parts (an all-gather
    per array).  Rows are concatenated in rank order; the packed zero points concatenate
    word for word because shard boundaries are multiples of ROW_ALIGN rows."""
    world, _ = _world(group)
    q = shard.layer
    if world == 1:
        return q
    d_out = shard.d_out
    rows = [row_shard(d_out, world, r) for r in range(world)]
    nrow = [b - a for a, b in rows]
    qweight = _gather_cols(q.qweight, nrow, group)
    scales = _gather_cols(q.scales, nrow, group)
    err_sq = _gather_cols(q.err_sq, nrow, group)
    qzeros = None
    if q.qzeros is not None:
        qzeros = _gather_cols(q.qzeros, [(n * bits + 31) // 32 for n in nrow], group)
    g_idx = q.g_idx
    if q.perm is not None:   # the group index is the same on every rank; rank 0 always owns rows
        buf = q.g_idx if q.g_idx is not None else torch.zeros_like(q.perm)
        parts = [torch.empty_like(buf) for _ in range(world)]
        dist.all_gather(parts, buf, group=group)
        g_idx = parts[0]
    return G.QuantizedLayer(qweight, scales, qzeros, err_sq, q.lam, g_idx, q.perm)
