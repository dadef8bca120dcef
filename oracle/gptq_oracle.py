"""Plain fp64 CPU oracle for GPTQ quantization of one linear layer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's ``smoke()`` check
and the benchmark's CPU-baseline leg may import this module.  The CUDA library
never calls it and shares no code with it.

What it follows (page titles as printed on the pages; section names in quotes):

* "GPTQ：基于近似二阶信息的大模型权重量化" (freeguideonline GPTQ tutorial):
  - "对称与仿射量化": q = round(x/s) + z, symmetric mode has z = 0 around the
    signed grid, group-wise scale/zero.
  - "量化误差与补偿": the error of a quantized weight is pushed into the other
    not-yet-quantized weights of the same row.
  - "阶段一：构建 Hessian 逆近似": E = ||WX - What X||_F^2 per layer, H = 2 X^T X
    plus damping lambda*I, Cholesky factor (upper triangular) instead of a full
    inverse.
  - "阶段二：贪婪顺序量化与懒惰批更新": fixed increasing column order, lazy batch
    updates of the not-yet-quantized columns.
  - "阶段三：量化与反量化": group-wise scale (and zero) found during the pass;
    dequantization multiplies the integer by its scale.
  - "激活排序（desc_act）": the columns may be visited in an order ranked by
    the sum of absolute input activations instead of their natural order.
* "GPTQ-2D: 三次时间复杂度的双侧自适应舍入" (ai-feeds summary), "问题背景" and
  "核心洞察": one-sided GPTQ equals Babai's nearest-plane algorithm; "方法": the
  two-sided problem and its vectorized (Kronecker Gram) form.
* "GPTQ/AWQ量化中Group Size的精确含义与计算" (feinterview group-size article),
  opening paragraphs and "存储代价": 4-bit codes 0..15, one scale and one zero per
  group of consecutive weights along the input (reduction) dimension,
  group_size = -1 means one group per row, (16 + 4)/g metadata bits per weight,
  symmetric mode stores no zero.

Readings of points the pages leave open (each is implemented below):

* Loss orientation: E = ||(W - What) X^T||_F^2 with X of shape n x d_in.
* H = 2 X^T X literally; lambda = damp_rel * mean(diag H).
* The factor used in the column loop is U, the upper Cholesky factor of
  (H + lambda I)^-1 (U^T U = Hd^-1).  Computed here the textbook way: explicit
  inverse, then Cholesky.
* The current column already carries all earlier compensation; its own error
  e_c = (w_c - what_c) / U_cc is pushed forward with row c of U.
* Quantization groups (metadata) and lazy blocks are distinct; a group size
  must divide the block size (or be -1).
* Group parameters are taken at the group's first column from the current
  (already compensated) values of the group's columns; group -1 takes them
  from the whole original row.
* Asymmetric: xmin = min(0, min v), xmax = max(0, max v); the zero point is an
  integer code so 0 lies on the grid.  Symmetric: range [-m, m] with
  m = max|v|, step 2m/maxq, implicit stored zero 2^(b-1).
* Scale rounded to fp16 (round to nearest even) before the zero and the codes
  are computed.  A group whose range is 0 gets scale 1.  A positive scale that
  rounds to 0 in fp16 is raised to the smallest positive fp16 value 2^-24.
* Rounding of codes: round half to even (IEEE rint), then clamp to [0, maxq].
* Zero stored in b bits.
* Activation ordering ("激活排序（desc_act）" on the tutorial page): the page
  ranks columns by the sum of absolute input activations and quantizes the
  least influential first, while the flag's name suggests descending order.
  desc_act = 1 follows the text (ascending), desc_act = 2 the name
  (descending); ties keep column order.  Groups are formed in quantization
  order, and a per-column group index maps each column to its group.
* GPTQ-2D: the objective is ||A (X - Z) B||_F^2 with Gram matrices G_left = A^T A
  and G_right = B B^T given, Z an integer matrix on the unbounded lattice (no scales,
  no clamp); the vectorization is column-major, and the one-dimensional GPTQ over it
  visits coordinates in increasing index, the GPTQ orientation of the rest of this
  module (first coordinate first).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

F16_MIN_POS = 2.0 ** -24


# ----------------------------------------------------------------------------
# Stage 1: Hessian, damping, inverse-Hessian Cholesky factor
# ----------------------------------------------------------------------------

def hessian(X: np.ndarray) -> np.ndarray:
    """H = 2 X^T X in fp64 (tutorial page, "阶段一", H = 2X^T X)."""
    Xd = np.asarray(X, dtype=np.float64)
    return 2.0 * (Xd.T @ Xd)


def damp(H: np.ndarray, damp_rel: float = 0.01) -> tuple[np.ndarray, float]:
    """Hd = H + lambda I with lambda = damp_rel * mean(diag H) (tutorial page, "阶段一")."""
    Hd = np.array(H, dtype=np.float64, copy=True)
    lam = float(damp_rel) * float(np.mean(np.diag(Hd)))
    Hd[np.diag_indices_from(Hd)] += lam
    return Hd, lam


def hinv_upper_cholesky(Hd: np.ndarray) -> np.ndarray:
    """U upper triangular with U^T U = Hd^-1: explicit inverse, then Cholesky.

    Tutorial page, "阶段一" step 2 (Cholesky, upper triangular) read as the upper
    Cholesky factor of the inverse Hessian.
    """
    Hinv = np.linalg.inv(np.asarray(Hd, dtype=np.float64))
    Hinv = 0.5 * (Hinv + Hinv.T)
    Lo = np.linalg.cholesky(Hinv)          # Hinv = Lo Lo^T, Lo lower
    return np.ascontiguousarray(Lo.T)      # U = Lo^T, upper, U^T U = Hinv


# ----------------------------------------------------------------------------
# The quantizer (tutorial "对称与仿射量化", group-size article)
# ----------------------------------------------------------------------------

def fp16_round(x):
    """Round to the nearest fp16 value (ties to even), returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def group_params(v: np.ndarray, bits: int, sym: bool):
    """Scale and zero for each row of ``v`` (shape rows x group_columns).

    Returns (scale, zero, scale_unrounded, lo, hi) with lo/hi the grid range
    that produced the scale; ``scale`` is the fp16-rounded value.
    """
    maxq = (1 << bits) - 1
    v = np.asarray(v, dtype=np.float64)
    if sym:
        m = np.max(np.abs(v), axis=1)
        lo, hi = -m, m
    else:
        lo = np.minimum(np.min(v, axis=1), 0.0)
        hi = np.maximum(np.max(v, axis=1), 0.0)
    raw = (hi - lo) / maxq
    scale = fp16_round(raw)
    scale = np.where(scale == 0.0, F16_MIN_POS, scale)
    degenerate = hi == lo
    scale = np.where(degenerate, 1.0, scale)
    raw = np.where(degenerate, 1.0, raw)
    if sym:
        zero = np.full(v.shape[0], float(1 << (bits - 1)))
    else:
        zero = np.clip(np.rint(-lo / scale), 0, maxq)
    return scale, zero, raw, lo, hi


def quantize(w, scale, zero, maxq):
    """q = clamp(round(w / s) + z, 0, maxq)."""
    return np.clip(np.rint(np.asarray(w, dtype=np.float64) / scale) + zero, 0, maxq)


def dequantize(q, scale, zero):
    """w_hat = s * (q - z) (group-size article, opening paragraph)."""
    return scale * (np.asarray(q, dtype=np.float64) - zero)


def boundary_distance(w, scale, zero, maxq):
    """Distance, in weight units, from w to the nearest rounding boundary of its code.

    Rounding boundaries of the unclamped grid sit at s*(k + 1/2 - z); codes
    clamped at 0 or maxq have only the inner boundary.
    """
    w = np.asarray(w, dtype=np.float64)
    x = w / scale + zero                      # grid coordinate
    k = np.floor(x)
    d_lo = np.abs(x - (k - 0.5))
    d_mid = np.abs(x - (k + 0.5))
    coord = np.minimum(d_lo, d_mid)
    # clamped region: only the boundary at 0.5 (low end) or maxq - 0.5 (high end) matters
    coord = np.where(x < 0.5, np.abs(x - 0.5), coord)
    coord = np.where(x > maxq - 0.5, np.abs(x - (maxq - 0.5)), coord)
    return coord * scale


# ----------------------------------------------------------------------------
# Stage 2: the greedy OBS column loop
# ----------------------------------------------------------------------------

@dataclass
class GPTQResult:
    codes: np.ndarray        # int64 [d_out, d_in], 0..maxq
    scales: np.ndarray       # fp64 [n_groups, d_out] (fp16-representable values)
    zeros: np.ndarray        # int64 [n_groups, d_out]
    err: np.ndarray          # fp64 [d_out, d_in], e_c = (w_c - what_c) / U_cc
    pre: np.ndarray          # fp64 [d_out, d_in], value w_c that was rounded
    what: np.ndarray         # fp64 [d_out, d_in], dequantized weights
    own_scales: np.ndarray | None = None   # replay only: this oracle's own fp16 scales
    forced_codes: int = 0
    forced_params: int = 0
    hard_codes: int = 0
    hard_params: int = 0
    worst_forced_dist: float = 0.0


def _group_len(group_size: int, d_in: int) -> int:
    return d_in if group_size == -1 else group_size


def n_groups(d_in: int, group_size: int) -> int:
    g = _group_len(group_size, d_in)
    return (d_in + g - 1) // g


class _Replay:
    """Teacher-forced replay against another implementation's outputs.

    Where this oracle and the other side disagree on a decision (a code, an
    fp16 scale, a zero point) and the oracle's own unrounded value lies within
    ``tol`` (weight units) of the rounding boundary, the other side's decision
    is adopted and counted as forced; any other disagreement is counted hard.
    """

    def __init__(self, codes, scales, zeros, tol):
        self.codes = np.asarray(codes)
        self.scales = np.asarray(scales, dtype=np.float64)
        self.zeros = None if zeros is None else np.asarray(zeros)
        self.tol = float(tol)
        self.forced_codes = self.forced_params = self.hard_codes = self.hard_params = 0
        self.worst = 0.0
        self.own_scales = np.array(self.scales, copy=True)

    def params(self, gi, scale, zero, raw, lo, hi, bits, sym):
        maxq = (1 << bits) - 1
        self.own_scales[gi] = scale
        other_s = self.scales[gi]
        diff = other_s != scale
        if np.any(diff):
            # distance of the unrounded range (hi - lo) to the fp16 tie point between the two
            mid = 0.5 * (other_s + scale)
            dist = np.abs((hi - lo) - maxq * mid)
            ok = diff & (dist <= self.tol)
            self.forced_params += int(np.count_nonzero(ok))
            self.hard_params += int(np.count_nonzero(diff & ~ok))
            scale = np.where(diff, other_s, scale)
            if not sym:
                zero = np.clip(np.rint(-lo / scale), 0, maxq)
        if not sym and self.zeros is not None:
            other_z = self.zeros[gi].astype(np.float64)
            dz = other_z != zero
            if np.any(dz):
                mid = 0.5 * (other_z + zero)
                dist = np.abs(-lo - scale * mid)
                ok = dz & (dist <= self.tol)
                self.forced_params += int(np.count_nonzero(ok))
                self.hard_params += int(np.count_nonzero(dz & ~ok))
                zero = np.where(dz, other_z, zero)
        return scale, zero

    def code(self, c, q, w, scale, zero, maxq):
        other = self.codes[:, c].astype(np.float64)
        diff = other != q
        if np.any(diff):
            dist = boundary_distance(w, scale, zero, maxq)
            ok = diff & (dist <= self.tol)
            self.forced_codes += int(np.count_nonzero(ok))
            self.hard_codes += int(np.count_nonzero(diff & ~ok))
            if np.any(ok):
                self.worst = max(self.worst, float(np.max(dist[ok])))
            q = np.where(diff, other, q)
        return q


def gptq(W0: np.ndarray, U: np.ndarray, bits: int = 4, group_size: int = 128,
         sym: bool = False, block_size: int = 0, replay: _Replay | None = None,
         fixed_grid: tuple[np.ndarray, np.ndarray] | None = None) -> GPTQResult:
    """GPTQ column loop over all rows at once (rows are independent).

    ``block_size = 0`` is the eager form: after each column the whole
    remainder of the row is updated.  ``block_size = B > 0`` is the lazy-batch
    form of the tutorial's "阶段二": inside a block of B columns each column's
    error is propagated to the rest of the block at once; after the block the
    columns to its right receive one batched update W[:, e:] -= Err_blk U[blk, e:].
    Both forms compute the same values up to rounding order.

    ``fixed_grid = (scale, zero)`` (one value per row) replaces the group
    parameters with a fixed grid and disables clamping; it is used to compare
    with Babai's nearest-plane algorithm on an unbounded lattice.
    """
    W = np.array(W0, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    d_out, d_in = W.shape
    maxq = (1 << bits) - 1
    g = _group_len(group_size, d_in)
    B = block_size if block_size > 0 else d_in
    if group_size != -1 and block_size > 0 and B % g != 0:
        raise ValueError("group size must divide the block size")
    ng = n_groups(d_in, group_size)
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    scales = np.zeros((ng, d_out))
    zeros = np.zeros((ng, d_out), dtype=np.int64)
    err = np.zeros((d_out, d_in))
    pre = np.zeros((d_out, d_in))
    what = np.zeros((d_out, d_in))
    scale = zero = None
    for b0 in range(0, d_in, B):
        b1 = min(b0 + B, d_in)
        for c in range(b0, b1):
            if fixed_grid is not None:
                scale, zero = fixed_grid
            elif c % g == 0:
                gi = c // g
                scale, zero, raw, lo, hi = group_params(W[:, c:min(c + g, d_in)], bits, sym)
                if replay is not None:
                    scale, zero = replay.params(gi, scale, zero, raw, lo, hi, bits, sym)
                scales[gi] = scale
                zeros[gi] = zero
            w = W[:, c].copy()
            if fixed_grid is not None:
                q = np.rint(w / scale) + zero
            else:
                q = quantize(w, scale, zero, maxq)
            if replay is not None:
                q = replay.code(c, q, w, scale, zero, maxq)
            wh = dequantize(q, scale, zero)
            e = (w - wh) / U[c, c]
            pre[:, c] = w
            codes[:, c] = q.astype(np.int64)
            what[:, c] = wh
            err[:, c] = e
            if block_size > 0:
                W[:, c + 1:b1] -= np.outer(e, U[c, c + 1:b1])
            else:
                W[:, c + 1:] -= np.outer(e, U[c, c + 1:])
        if block_size > 0 and b1 < d_in:
            W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]
    res = GPTQResult(codes, scales, zeros, err, pre, what)
    if replay is not None:
        res.forced_codes, res.forced_params = replay.forced_codes, replay.forced_params
        res.hard_codes, res.hard_params = replay.hard_codes, replay.hard_params
        res.worst_forced_dist = replay.worst
        res.own_scales = replay.own_scales
    return res


def gptq_replay(W0, U, other_codes, other_scales, other_zeros, bits=4, group_size=128,
                sym=False, block_size=128, tol=1e-5) -> GPTQResult:
    """Run the column loop, adopting the other side's decisions only near rounding boundaries."""
    rp = _Replay(other_codes, other_scales, other_zeros, tol)
    return gptq(W0, U, bits, group_size, sym, block_size, replay=rp)


def rtn(W0: np.ndarray, bits: int = 4, group_size: int = 128, sym: bool = False) -> GPTQResult:
    """Round-to-nearest baseline: group params from the original weights, no compensation."""
    W = np.asarray(W0, dtype=np.float64)
    d_out, d_in = W.shape
    maxq = (1 << bits) - 1
    g = _group_len(group_size, d_in)
    ng = n_groups(d_in, group_size)
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    scales = np.zeros((ng, d_out))
    zeros = np.zeros((ng, d_out), dtype=np.int64)
    what = np.zeros((d_out, d_in))
    for gi in range(ng):
        c0, c1 = gi * g, min(gi * g + g, d_in)
        s, z, _, _, _ = group_params(W[:, c0:c1], bits, sym)
        q = quantize(W[:, c0:c1], s[:, None], z[:, None], maxq)
        codes[:, c0:c1] = q.astype(np.int64)
        scales[gi], zeros[gi] = s, z
        what[:, c0:c1] = dequantize(q, s[:, None], z[:, None])
    return GPTQResult(codes, scales, zeros, np.zeros_like(what), W.copy(), what)


def gptq_naive_obs(W0: np.ndarray, Hd: np.ndarray, bits=4, group_size=128, sym=False,
                   order: np.ndarray | None = None) -> GPTQResult:
    """Literal OBS form for tiny inputs: after each column, re-invert the remaining Hessian.

    For column c the inverse of Hd restricted to the not-yet-quantized columns
    is formed explicitly; the error of column c, divided by that inverse's
    diagonal entry for c, is pushed along its row (tutorial page, "阶段一" and
    the pseudocode's per-column downdate).  Uses no Cholesky factor, so it
    checks the U form independently.

    ``order`` (a permutation of the columns) visits the columns in that order
    and works in the original coordinates throughout: no permuted copy of W or
    Hd is made, group k takes the columns order[k*g:(k+1)*g], and codes land in
    their own columns.  It checks the permute/unpermute of the act-order form.
    """
    W = np.array(W0, dtype=np.float64, copy=True)
    Hd = np.asarray(Hd, dtype=np.float64)
    d_out, d_in = W.shape
    order = np.arange(d_in) if order is None else np.asarray(order)
    maxq = (1 << bits) - 1
    g = _group_len(group_size, d_in)
    ng = n_groups(d_in, group_size)
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    scales = np.zeros((ng, d_out))
    zeros = np.zeros((ng, d_out), dtype=np.int64)
    what = np.zeros((d_out, d_in))
    for k in range(d_in):
        c = order[k]
        rest = order[k:]                 # c first, then the columns still to come
        if k % g == 0:
            s, z, _, _, _ = group_params(W[:, order[k:min(k + g, d_in)]], bits, sym)
            scales[k // g], zeros[k // g] = s, z
        Hinv_rem = np.linalg.inv(Hd[np.ix_(rest, rest)])
        w = W[:, c].copy()
        q = quantize(w, s, z, maxq)
        wh = dequantize(q, s, z)
        codes[:, c], what[:, c] = q.astype(np.int64), wh
        W[:, rest[1:]] -= np.outer((w - wh) / Hinv_rem[0, 0], Hinv_rem[0, 1:])
    return GPTQResult(codes, scales, zeros, np.zeros_like(what), np.zeros_like(what), what)


def babai_nearest_plane(x: np.ndarray, basis: np.ndarray) -> np.ndarray:
    """Babai's nearest-plane rounding of real coordinates ``x`` on the lattice spanned by basis columns.

    Gram-Schmidt runs from the last basis vector backward, so the GS vector of
    b_0 is orthogonal to all other basis vectors and coordinate 0 is decided
    first; this is the order in which GPTQ quantizes columns (GPTQ-2D summary,
    "问题背景": GPTQ is Babai's nearest-plane algorithm).
    """
    Bm = np.asarray(basis, dtype=np.float64)
    n = Bm.shape[1]
    gs = np.zeros_like(Bm)
    for j in range(n - 1, -1, -1):
        v = Bm[:, j].copy()
        for k in range(j + 1, n):
            v -= (Bm[:, j] @ gs[:, k]) / (gs[:, k] @ gs[:, k]) * gs[:, k]
        gs[:, j] = v
    t = Bm @ np.asarray(x, dtype=np.float64)
    c = np.zeros(n)
    for j in range(n):
        c[j] = np.rint((t @ gs[:, j]) / (gs[:, j] @ gs[:, j]))
        t = t - c[j] * Bm[:, j]
    return c


# ----------------------------------------------------------------------------
# Loss, packing, dequantization, metadata size
# ----------------------------------------------------------------------------

def layer_loss(W0: np.ndarray, What: np.ndarray, X: np.ndarray) -> float:
    """E = ||(W - W_hat) X^T||_F^2 (tutorial page, "阶段一", output squared error)."""
    D = np.asarray(W0, dtype=np.float64) - np.asarray(What, dtype=np.float64)
    Y = D @ np.asarray(X, dtype=np.float64).T
    return float(np.sum(Y * Y))


def row_losses(W0, What, X) -> np.ndarray:
    D = np.asarray(W0, dtype=np.float64) - np.asarray(What, dtype=np.float64)
    Y = D @ np.asarray(X, dtype=np.float64).T
    return np.sum(Y * Y, axis=1)


def pack_bitstream(values: np.ndarray, bits: int) -> np.ndarray:
    """Pack each row of non-negative integers as a little-endian b-bit stream of int32 words.

    values: [rows, cols] -> uint32 words [rows, ceil(cols*bits/32)]; value j of a
    row occupies bits j*b .. j*b+b-1 of the stream (LSB first), and a value may
    straddle two words when 32 is not a multiple of b.
    """
    values = np.asarray(values, dtype=np.int64)
    rows, cols = values.shape
    nwords = (cols * bits + 31) // 32
    out = np.zeros((rows, nwords), dtype=np.uint64)
    for j in range(cols):
        bit = j * bits
        w, sh = divmod(bit, 32)
        v = values[:, j].astype(np.uint64)
        out[:, w] |= (v << np.uint64(sh)) & np.uint64(0xFFFFFFFF)
        if sh + bits > 32:
            out[:, w + 1] |= v >> np.uint64(32 - sh)
    return out.astype(np.uint32)


def unpack_bitstream(words: np.ndarray, bits: int, cols: int) -> np.ndarray:
    words = np.asarray(words).astype(np.uint64) & np.uint64(0xFFFFFFFF)
    rows = words.shape[0]
    out = np.zeros((rows, cols), dtype=np.int64)
    mask = (1 << bits) - 1
    for j in range(cols):
        bit = j * bits
        w, sh = divmod(bit, 32)
        v = words[:, w] >> np.uint64(sh)
        if sh + bits > 32:
            v = v | (words[:, w + 1] << np.uint64(32 - sh))
        out[:, j] = (v & np.uint64(mask)).astype(np.int64)
    return out


def pack_qweight(codes: np.ndarray, bits: int) -> np.ndarray:
    """qweight int32 [ceil(d_in*b/32), d_out]: column o is row o's code stream along d_in."""
    return np.ascontiguousarray(pack_bitstream(codes, bits).T).view(np.int32)


def pack_qzeros(zeros: np.ndarray, bits: int) -> np.ndarray:
    """qzeros int32 [n_groups, ceil(d_out*b/32)]: each group's zeros packed along d_out."""
    return np.ascontiguousarray(pack_bitstream(zeros, bits)).view(np.int32)


def dequant_packed(qweight, scales, qzeros, d_out, d_in, bits, group_size, sym, g_idx=None) -> np.ndarray:
    """W_hat[o, c] = scale[g(c), o] * (q[o, c] - zero[g(c), o]) from the packed arrays.

    g(c) = c // group_size, or g_idx[c] when a per-column group index is given
    (activation ordering)."""
    codes = unpack_bitstream(np.asarray(qweight).view(np.uint32).T, bits, d_in)
    g = _group_len(group_size, d_in)
    gi = np.arange(d_in) // g if g_idx is None else np.asarray(g_idx, dtype=np.int64)
    s = np.asarray(scales, dtype=np.float64)[gi, :].T
    if sym:
        z = float(1 << (bits - 1))
    else:
        zall = unpack_bitstream(np.asarray(qzeros).view(np.uint32), bits, d_out)
        z = zall[gi, :].T.astype(np.float64)
    return s * (codes - z)


def dequant_gemm(X, qweight, scales, qzeros, d_out, d_in, bits, group_size, sym, g_idx=None) -> np.ndarray:
    """Y = X W_hat^T in fp64, W_hat dequantized from the packed arrays (tutorial page,
    "阶段三": the weights a layer computes with are the integers times their scales)."""
    What = dequant_packed(qweight, scales, qzeros, d_out, d_in, bits, group_size, sym, g_idx)
    return np.asarray(X, dtype=np.float64) @ What.T


def metadata_bits_per_weight(d_out, d_in, bits, group_size, sym, scale_bits=16) -> float:
    """Bits of stored scale + zero per weight (group-size article, "存储代价")."""
    ng = n_groups(d_in, group_size)
    meta = ng * d_out * scale_bits + (0 if sym else ng * d_out * bits)
    return meta / (d_out * d_in)


def babai_bound(U: np.ndarray, scale: float) -> float:
    """Nearest-plane residual bound in GPTQ coordinates: 1/4 * sum_j s^2 / U_jj^2."""
    d = np.diag(np.asarray(U, dtype=np.float64))
    return 0.25 * float(np.sum(scale * scale / (d * d)))


def quantize_layer(W0, X, bits=4, group_size=128, sym=False, block_size=128, damp_rel=0.01):
    """Whole layer: H, damping, U, blocked column loop.  Returns (result, H, U, lam)."""
    H = hessian(X)
    Hd, lam = damp(H, damp_rel)
    U = hinv_upper_cholesky(Hd)
    res = gptq(W0, U, bits, group_size, sym, block_size)
    return res, H, U, lam


# ----------------------------------------------------------------------------
# Activation ordering (desc_act)
# ----------------------------------------------------------------------------

ACT_ASCENDING = 1    # the tutorial's procedure: least output impact first
ACT_DESCENDING = 2   # the order the flag's name suggests


def act_abs_sum(X: np.ndarray) -> np.ndarray:
    """a_c = sum_t |X[t, c]| in fp64 (tutorial page, "激活排序（desc_act）": columns
    are ranked by the sum of the absolute values of their input activations)."""
    return np.sum(np.abs(np.asarray(X, dtype=np.float64)), axis=0)


def act_order(a: np.ndarray, desc_act: int) -> np.ndarray:
    """Quantization order perm: perm[k] is the column quantized at position k.

    desc_act = 1 sorts a ascending: the columns whose activations move the output
    least are quantized first and the sensitive ones, quantized last, absorb the
    compensation (the tutorial's "激活排序（desc_act）" text).  desc_act = 2 sorts
    descending.  Equal values keep increasing column index in both directions.
    """
    a = np.asarray(a, dtype=np.float64)
    if desc_act == ACT_ASCENDING:
        return np.argsort(a, kind="stable")
    if desc_act == ACT_DESCENDING:
        return np.argsort(-a, kind="stable")
    raise ValueError("desc_act must be 1 (ascending) or 2 (descending)")


def g_idx_of(perm: np.ndarray, group_size: int) -> np.ndarray:
    """Per-column group index: column perm[k] belongs to group k // g."""
    perm = np.asarray(perm)
    g = _group_len(group_size, perm.size)
    gi = np.empty(perm.size, dtype=np.int64)
    gi[perm] = np.arange(perm.size) // g
    return gi


@dataclass
class ActOrderResult:
    codes: np.ndarray        # int64 [d_out, d_in], original column order
    scales: np.ndarray       # fp64 [n_groups, d_out], groups in quantization order
    zeros: np.ndarray        # int64 [n_groups, d_out]
    g_idx: np.ndarray        # int64 [d_in]
    what: np.ndarray         # fp64 [d_out, d_in], original column order
    perm: np.ndarray         # quantization order
    U: np.ndarray            # upper Cholesky factor of the permuted (P^T Hd P)^-1
    lam: float
    inner: GPTQResult        # the column loop's own result, in quantization order


def gptq_act_order(W0: np.ndarray, H: np.ndarray, perm: np.ndarray, bits=4, group_size=128, sym=False,
                   block_size=128, damp_rel=0.01) -> ActOrderResult:
    """GPTQ with the columns visited in the order perm.

    The column loop is the unchanged fixed-order one applied to the permuted
    problem: Hp[i, j] = H[perm[i], perm[j]], Wp = W0[:, perm]; damping and U are
    taken from Hp (lambda is unchanged: the diagonal is only reordered).  Codes
    and dequantized weights are put back in the original columns; groups stay in
    quantization order and g_idx maps each column to its group.
    """
    perm = np.asarray(perm)
    Hp = np.asarray(H, dtype=np.float64)[np.ix_(perm, perm)]
    Hd, lam = damp(Hp, damp_rel)
    U = hinv_upper_cholesky(Hd)
    res = gptq(np.asarray(W0, dtype=np.float64)[:, perm], U, bits, group_size, sym, block_size)
    codes = np.empty_like(res.codes)
    codes[:, perm] = res.codes
    what = np.empty_like(res.what)
    what[:, perm] = res.what
    return ActOrderResult(codes, res.scales, res.zeros, g_idx_of(perm, group_size), what, perm, U, lam, res)


# ----------------------------------------------------------------------------
# GPTQ-2D: two-sided adaptive rounding
# ----------------------------------------------------------------------------

def gptq2d_loss(X: np.ndarray, Z: np.ndarray, G_left: np.ndarray, G_right: np.ndarray) -> float:
    """tr((X - Z)^T G_left (X - Z) G_right) = ||A (X - Z) B||_F^2 for G_left = A^T A and
    G_right = B B^T (GPTQ-2D summary, "方法": a real matrix rounded to an integer one under a
    quadratic metric with fixed nonsingular bases on both sides)."""
    D = np.asarray(X, dtype=np.float64) - np.asarray(Z, dtype=np.float64)
    return float(np.trace(D.T @ np.asarray(G_left, dtype=np.float64) @ D @ np.asarray(G_right, dtype=np.float64)))


def gptq2d_vectorized(X: np.ndarray, G_left: np.ndarray, G_right: np.ndarray) -> np.ndarray:
    """Two-sided adaptive rounding by the vectorized route (GPTQ-2D summary, "问题背景",
    "方法"): the one-dimensional GPTQ run over vec(X).  Tiny sizes only.

    Column-major vectorization (p = i + m j) turns the objective into the quadratic form of
    the Kronecker Gram G = G_right (x) G_left.  GPTQ visits p = 0, 1, ... with U the upper
    Cholesky factor of G^-1, formed explicitly as an mn x mn matrix; each coordinate is
    rounded to the nearest integer (ties to even, no clamp: the unbounded lattice) and
    its error e_p = (x_p - z_p) / U_pp is pushed forward along row p of U.  This is
    Babai's nearest plane on that lattice; O((mn)^2) work in the loop, quartic in n.
    """
    X = np.asarray(X, dtype=np.float64)
    m, n = X.shape
    U = hinv_upper_cholesky(np.kron(np.asarray(G_right, dtype=np.float64), np.asarray(G_left, dtype=np.float64)))
    x = X.reshape(-1, order="F").copy()
    z = np.zeros(m * n)
    for p in range(m * n):
        z[p] = np.rint(x[p])
        e = (x[p] - z[p]) / U[p, p]
        x[p + 1:] -= e * U[p, p + 1:]
    return z.reshape((m, n), order="F")


def gptq2d_antidiagonal(X: np.ndarray, U_left: np.ndarray, U_right: np.ndarray) -> np.ndarray:
    """Two-sided adaptive rounding by the anti-diagonal route (GPTQ-2D summary, "方法",
    steps 1-3): the entries of X are taken anti-diagonal by anti-diagonal, i + j = k for
    k = 0, 1, ..., m + n - 2; every entry of one anti-diagonal is rounded from the errors of
    the entries before that anti-diagonal (they do not depend on one another), and its error
    is then pushed forward through the Cholesky factors of both sides.

    U_left (m x m) and U_right (n x n) are the upper Cholesky factors of G_left^-1 and
    G_right^-1.  Kept for row i: T[i, :] = sum of e_ij U_right[j, :] over the entries (i, j)
    rounded so far, so the correction of entry (i, j) is the dot product of column i of
    U_left with column j of T.  Rounding is to the nearest integer, ties to even, no clamp.
    O(m n (m + n)) work; equal in exact arithmetic to gptq2d_vectorized (the errors of
    entry (i', j') reach (i, j) only when i' <= i and j' <= j, and both routes visit such
    entries first).
    """
    X = np.asarray(X, dtype=np.float64)
    UL = np.asarray(U_left, dtype=np.float64)
    UR = np.asarray(U_right, dtype=np.float64)
    m, n = X.shape
    Z = np.zeros((m, n))
    T = np.zeros((m, n))
    for k in range(m + n - 1):
        cells = [(i, k - i) for i in range(max(0, k - n + 1), min(m, k + 1))]
        vals = [X[i, j] - UL[:i + 1, i] @ T[:i + 1, j] for i, j in cells]   # all before any update
        for (i, j), v in zip(cells, vals):
            Z[i, j] = np.rint(v)
            e = (v - Z[i, j]) / (UL[i, i] * UR[j, j])
            T[i, j:] += e * UR[j, j:]
    return Z

