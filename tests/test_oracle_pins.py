"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: numbers the
pages print (tests/golden), closed forms, brute force on tiny inputs, an
independent algorithm (Babai nearest plane, literal OBS re-inversion), or an
invariant.  A plausible slip in the oracle (dropped compensation term, wrong
sign, transposed factor, wrong group boundary, wrong rounding) fails at least
one of them.
"""

import itertools
import json
import os

import numpy as np
import pytest

from oracle import gptq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def round_half_up(x, nd):
    """Decimal rounding as printed on the pages (0.3125 -> 0.313)."""
    f = 10 ** nd
    return np.floor(x * f + 0.5) / f


def _rand_problem(seed, d_out, d_in, n, hot=2):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d_in))
    if hot:
        X[:, rng.choice(d_in, hot, replace=False)] *= 8.0
    W = rng.standard_normal((d_out, d_in)) * 0.02
    H = O.hessian(X)
    Hd, lam = O.damp(H, 0.01)
    U = O.hinv_upper_cholesky(Hd)
    return X, W, H, Hd, U


# ---------------------------------------------------------------- stage 1

def test_hessian_is_sum_of_token_outer_products():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((7, 5))
    brute = np.zeros((5, 5))
    for t in range(7):
        for i in range(5):
            for j in range(5):
                brute[i, j] += 2.0 * X[t, i] * X[t, j]
    np.testing.assert_allclose(O.hessian(X), brute, rtol=1e-13, atol=1e-13)


def test_damping_closed_form():
    H = np.diag([1.0, 2.0, 3.0, 4.0])
    Hd, lam = O.damp(H, 0.01)
    assert lam == pytest.approx(0.025, rel=1e-15)
    np.testing.assert_allclose(np.diag(Hd), [1.025, 2.025, 3.025, 4.025], rtol=1e-15)
    assert Hd[0, 1] == 0.0


def test_U_is_the_upper_cholesky_factor_of_the_inverse():
    _, _, _, Hd, U = _rand_problem(2, 3, 24, 40)
    assert np.all(np.tril(U, -1) == 0.0)
    assert np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U @ Hd, np.eye(24), atol=1e-10)


def test_U_rows_are_normalised_rows_of_trailing_inverses():
    # OBS downdate form: row c of U is row 0 of inv(Hd[c:, c:]) / sqrt of its (0,0) entry
    _, _, _, Hd, U = _rand_problem(3, 3, 12, 30)
    for c in range(12):
        Ri = np.linalg.inv(Hd[c:, c:])
        np.testing.assert_allclose(U[c, c:], Ri[0, :] / np.sqrt(Ri[0, 0]), rtol=1e-9, atol=1e-12)


def test_U_of_reversed_cholesky_route_agrees():
    # Hd = R R^T with R upper (Cholesky of the index-reversed matrix) gives U = R^-1.
    _, _, _, Hd, U = _rand_problem(4, 3, 16, 40)
    J = np.arange(16)[::-1]
    L = np.linalg.cholesky(Hd[np.ix_(J, J)])
    R = L[np.ix_(J, J)]
    assert np.allclose(np.tril(R, -1), 0.0)
    np.testing.assert_allclose(np.linalg.inv(R), U, rtol=1e-8, atol=1e-12)


# ---------------------------------------------------------------- quantizer

def test_group_params_hand_values_asym():
    v = np.array([[-0.02, 0.0, 0.01, 0.02]])
    s, z, raw, lo, hi = O.group_params(v, 4, sym=False)
    assert raw[0] == pytest.approx(0.04 / 15, rel=1e-15)
    assert s[0] == float(np.float16(0.04 / 15))
    # zero = rint(0.02 / s) with s slightly below 0.0026667 -> 7.5002 -> 8
    assert z[0] == 8.0
    q = O.quantize(v, s[:, None], z[:, None], 15)
    assert list(q[0]) == [0.0, 8.0, 12.0, 15.0]


def test_group_params_range_contains_zero():
    v = np.array([[0.1, 0.2, 0.3]])
    s, z, _, lo, hi = O.group_params(v, 4, sym=False)
    assert lo[0] == 0.0 and z[0] == 0.0
    assert s[0] == float(np.float16(0.3 / 15))


def test_group_params_sym_and_degenerate():
    v = np.array([[-0.5, 0.1, 0.25], [0.0, 0.0, 0.0]])
    s, z, _, _, _ = O.group_params(v, 3, sym=True)
    assert s[0] == float(np.float16(1.0 / 7)) and z[0] == 4.0
    assert s[1] == 1.0 and z[1] == 4.0
    q = O.quantize(np.zeros(3), 1.0, 4.0, 7)
    assert np.all(O.dequantize(q, 1.0, 4.0) == 0.0)


def test_tiny_range_scale_clamped_to_smallest_fp16():
    v = np.array([[1e-12, -1e-12]])
    s, z, _, _, _ = O.group_params(v, 4, sym=False)
    assert s[0] == 2.0 ** -24


def test_round_half_to_even_and_clamp():
    s, z = 1.0, 0.0
    assert list(O.quantize(np.array([0.5, 1.5, 2.5, -3.0, 99.0]), s, z, 15)) == [0.0, 2.0, 2.0, 0.0, 15.0]


def test_grid_step_example_from_group_size_page():
    g = json.load(open(os.path.join(GOLDEN, "grid_step_example.json")))
    bits = g["bits"]
    lo, hi = g["tight_group_range"]
    tight = np.array([[lo, hi, 0.001]])
    s1, _, raw1, _, _ = O.group_params(tight, bits, sym=True)
    outl = np.array([[lo, hi, g["outlier_magnitude"]]])
    s2, _, raw2, _, _ = O.group_params(outl, bits, sym=True)
    assert raw1[0] == pytest.approx(g["tight_step_printed"], abs=0.5e-4)
    assert raw2[0] == pytest.approx(g["outlier_step_printed"], abs=0.5e-3)
    assert raw2[0] / raw1[0] == pytest.approx(g["coarser_factor_printed"], rel=1e-12)
    assert (1 << bits) - 1 == g["levels_divisor"]
    # the asymmetric grid on the tight range gives the same step
    sa, _, rawa, _, _ = O.group_params(tight, bits, sym=False)
    assert rawa[0] == pytest.approx(g["tight_step_printed"], abs=0.5e-4)


# ---------------------------------------------------------------- metadata size

def test_metadata_overhead_matches_group_size_page():
    gd = json.load(open(os.path.join(GOLDEN, "group_size_overhead.json")))
    d_out, d_in = 64, 1024
    rng = np.random.default_rng(5)
    for row in gd["overhead_bits_per_weight"]:
        g = row["group_size"]
        # measure from the arrays the packer actually writes
        ng = O.n_groups(d_in, g)
        zeros = rng.integers(0, 16, size=(ng, d_out))
        scales = np.zeros((ng, d_out), dtype=np.float16)
        qz = O.pack_qzeros(zeros, 4)
        measured = (scales.nbytes + qz.nbytes) * 8 / (d_out * d_in)
        assert measured == pytest.approx(O.metadata_bits_per_weight(d_out, d_in, 4, g, False), rel=1e-15)
        if g == -1:
            assert measured == pytest.approx(20.0 / d_in, rel=1e-15)
            # "~0": one scale+zero per row of a real layer (d_in = 4096..11008) rounds to 0.00
            for d_row in (4096, 11008):
                big = O.metadata_bits_per_weight(8, d_row, 4, -1, False)
                assert round_half_up(big, 2) == row["overhead"]
                assert round_half_up(4 + big, 2) == row["total"]
        else:
            assert measured == 20.0 / g
            assert round_half_up(measured, gd["printed_decimals"]) == pytest.approx(row["overhead"], abs=1e-12)
            assert round_half_up(4 + measured, gd["printed_decimals"]) == pytest.approx(row["total"], abs=1e-12)
    # symmetric drops the zero: numerator 16
    assert O.metadata_bits_per_weight(d_out, d_in, 4, 128, True) * 128 == gd["symmetric_numerator_bits"]


def test_model_size_lines_of_group_size_page():
    gd = json.load(open(os.path.join(GOLDEN, "group_size_overhead.json")))
    sizes = {}
    for row in gd["model_7b_gb"]:
        g = row["group_size"]
        bpw = 4 + round_half_up(20.0 / g, 3)     # the page rounds the overhead before multiplying
        gb = 7.0e9 * bpw / 8 / 1e9
        sizes[g] = gb
        assert round_half_up(gb, gd["gb_decimals"]) == pytest.approx(row["gb"], abs=1e-9)
    span = sizes[32] - sizes[128]
    assert round(span, 2) == pytest.approx(gd["span_128_to_32_gb"], abs=1e-9)
    assert round(span / sizes[128], 2) == pytest.approx(gd["span_fraction_approx"], abs=1e-9)
    extra = 20.0 / 32 - 20.0 / 128
    assert round(extra, 3) == pytest.approx(gd["model_70b_extra_bits"], abs=1e-9)
    assert round(70e9 * extra / 8 / 1e9, 1) == pytest.approx(gd["model_70b_extra_gb"], abs=1e-9)


# ---------------------------------------------------------------- packing

def test_pack_hand_example_4bit():
    codes = np.array([[1, 2, 3, 4, 5, 6, 7, 8, 15, 0, 0, 0, 0, 0, 0, 9]])
    w = O.pack_bitstream(codes, 4)
    assert w.shape == (1, 2)
    assert int(w[0, 0]) == 0x87654321
    assert int(w[0, 1]) == 0x9000000F


def test_pack_hand_example_3bit_straddle():
    # 11 values of 3 bits: value 10 occupies bits 30..32, straddling words 0 and 1
    codes = np.zeros((1, 11), dtype=np.int64)
    codes[0, 0] = 5          # bits 0..2  -> 0b101
    codes[0, 10] = 7         # bits 30..32 -> word0 bits 30,31 and word1 bit 0
    w = O.pack_bitstream(codes, 3)
    assert w.shape == (1, 2)
    assert int(w[0, 0]) == (5 | (3 << 30))
    assert int(w[0, 1]) == 1


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=(5, 77))
    w = O.pack_bitstream(codes, bits)
    assert w.shape[1] == (77 * bits + 31) // 32
    np.testing.assert_array_equal(O.unpack_bitstream(w, bits, 77), codes)


def test_qweight_layout_and_dequant_hand_example():
    # 2 output rows, 8 input columns, one group: W_hat = s * (q - z)
    codes = np.array([[0, 1, 2, 3, 4, 5, 6, 7], [15, 14, 13, 12, 11, 10, 9, 8]])
    qw = O.pack_qweight(codes, 4)
    assert qw.shape == (1, 2)
    assert int(qw.view(np.uint32)[0, 0]) == 0x76543210
    assert int(qw.view(np.uint32)[0, 1]) == 0x89ABCDEF
    scales = np.array([[0.5, 0.25]], dtype=np.float16)
    qz = O.pack_qzeros(np.array([[3, 8]]), 4)
    assert int(qz.view(np.uint32)[0, 0]) == 0x83
    What = O.dequant_packed(qw, scales, qz, 2, 8, 4, -1, False)
    np.testing.assert_array_equal(What[0], 0.5 * (np.arange(8) - 3))
    np.testing.assert_array_equal(What[1], 0.25 * (np.arange(15, 7, -1) - 8))


# ---------------------------------------------------------------- column loop

@pytest.mark.parametrize("bits,g,sym", [(4, 128, False), (3, 64, True), (2, 32, False), (4, -1, False)])
def test_identity_hessian_reduces_to_rtn(bits, g, sym):
    rng = np.random.default_rng(7)
    W = rng.standard_normal((9, 256)) * 0.02
    U = O.hinv_upper_cholesky(np.eye(256))
    r = O.gptq(W, U, bits, g, sym, block_size=128)
    ref = O.rtn(W, bits, g, sym)
    np.testing.assert_array_equal(r.codes, ref.codes)
    np.testing.assert_array_equal(r.scales, ref.scales)
    np.testing.assert_array_equal(r.zeros, ref.zeros)


def test_diagonal_hessian_reduces_to_rtn():
    rng = np.random.default_rng(8)
    W = rng.standard_normal((6, 128)) * 0.02
    Hd = np.diag(rng.uniform(0.5, 5.0, 128))
    r = O.gptq(W, O.hinv_upper_cholesky(Hd), 4, 32, False, block_size=0)
    np.testing.assert_array_equal(r.codes, O.rtn(W, 4, 32, False).codes)


@pytest.mark.parametrize("bits,g,sym", [(4, 128, False), (3, 64, True), (2, 32, False), (4, -1, False), (8, 16, False)])
def test_lazy_blocks_equal_eager(bits, g, sym):
    _, W, _, _, U = _rand_problem(9, 17, 384, 300)
    eager = O.gptq(W, U, bits, g, sym, block_size=0)
    lazy = O.gptq(W, U, bits, g, sym, block_size=128)
    np.testing.assert_array_equal(eager.codes, lazy.codes)
    np.testing.assert_array_equal(eager.scales, lazy.scales)
    np.testing.assert_allclose(eager.err, lazy.err, rtol=1e-9, atol=1e-12)


def test_lazy_blocks_equal_eager_ragged():
    _, W, _, _, U = _rand_problem(10, 5, 200, 150)
    eager = O.gptq(W, U, 4, 32, False, block_size=0)
    lazy = O.gptq(W, U, 4, 32, False, block_size=128)
    np.testing.assert_array_equal(eager.codes, lazy.codes)
    assert eager.scales.shape == (7, 5)      # 6 full groups + one of 8 columns


@pytest.mark.parametrize("seed", [11, 12, 13])
def test_U_form_equals_literal_obs_reinversion(seed):
    _, W, _, Hd, U = _rand_problem(seed, 6, 8, 20, hot=1)
    a = O.gptq(W, U, 3, 4, False, block_size=0)
    b = O.gptq_naive_obs(W, Hd, 3, 4, False)
    np.testing.assert_array_equal(a.codes, b.codes)
    np.testing.assert_allclose(a.what, b.what, rtol=0, atol=1e-15)


@pytest.mark.parametrize("seed", range(20, 30))
def test_gptq_equals_babai_nearest_plane(seed):
    X, W, H, Hd, U = _rand_problem(seed, 4, 7, 12, hot=1)
    rng = np.random.default_rng(seed + 100)
    s = np.full(4, 0.004)
    z = rng.integers(0, 8, 4).astype(np.float64)
    r = O.gptq(W, U, 4, -1, False, block_size=0, fixed_grid=(s, z))
    # an independent basis with B^T B = Hd: symmetric square root
    ev, V = np.linalg.eigh(Hd)
    Bm = V @ np.diag(np.sqrt(ev)) @ V.T
    for o in range(4):
        c = O.babai_nearest_plane(W[o] / s[o] + z[o], Bm)
        np.testing.assert_array_equal(r.codes[o], c.astype(np.int64))


@pytest.mark.parametrize("seed", range(40, 46))
def test_bruteforce_bracket_and_babai_bound(seed):
    X, W, H, Hd, U = _rand_problem(seed, 1, 5, 9, hot=1)
    s, z = np.array([0.01]), np.array([0.0])
    r = O.gptq(W, U, 4, -1, False, block_size=0, fixed_grid=(s, z))
    x = W[0] / s[0]
    def loss(q):
        d = s[0] * (x - q)
        return d @ Hd @ d
    l_gptq = loss(r.codes[0].astype(np.float64))
    base = np.floor(x)
    rad = int(np.max(np.abs(r.codes[0] - base))) + 2
    offs = np.array(list(itertools.product(range(-rad, rad + 2), repeat=5)), dtype=np.float64)
    D = s[0] * (x[None, :] - (base[None, :] + offs))
    all_losses = np.einsum("ij,jk,ik->i", D, Hd, D)
    best = all_losses.min()
    assert best <= l_gptq * (1 + 1e-12)
    assert l_gptq <= O.babai_bound(U, s[0]) * (1 + 1e-12)


@pytest.mark.parametrize("bits", [2, 4])
def test_loss_identity_sum_of_squared_errors(bits):
    # per row: (W0 - W_hat) Hd (W0 - W_hat)^T == sum_c e_c^2, for any codes (clamped ones too)
    _, W, _, Hd, U = _rand_problem(50, 8, 96, 120)
    r = O.gptq(W * 3.0, U, bits, 32, False, block_size=64)
    D = W * 3.0 - r.what
    lhs = np.einsum("ij,jk,ik->i", D, Hd, D)
    np.testing.assert_allclose(lhs, np.sum(r.err ** 2, axis=1), rtol=1e-9)


def test_layer_loss_is_half_the_quadratic_form_of_H():
    X, W, H, Hd, U = _rand_problem(51, 5, 40, 60)
    r = O.gptq(W, U, 4, 8, False, block_size=0)
    D = W - r.what
    np.testing.assert_allclose(O.layer_loss(W, r.what, X), 0.5 * np.einsum("ij,jk,ik->", D, H, D), rtol=1e-10)
    np.testing.assert_allclose(O.row_losses(W, r.what, X).sum(), O.layer_loss(W, r.what, X), rtol=1e-12)


def test_codes_invariant_under_hessian_scaling():
    X, W, H, Hd, U = _rand_problem(52, 7, 128, 90)
    U2 = O.hinv_upper_cholesky(7.3 * Hd)
    a = O.gptq(W, U, 4, 32, False, 64)
    b = O.gptq(W, U2, 4, 32, False, 64)
    np.testing.assert_array_equal(a.codes, b.codes)


def test_compensation_lowers_layer_loss_vs_rtn():
    X, W, H, Hd, U = _rand_problem(53, 32, 128, 400, hot=4)
    g = O.gptq(W, U, 3, 32, False, 64)
    r = O.rtn(W, 3, 32, False)
    assert O.layer_loss(W, g.what, X) < O.layer_loss(W, r.what, X)


# ---------------------------------------------------------------- replay protocol

def test_replay_accepts_own_outputs():
    _, W, _, _, U = _rand_problem(60, 6, 128, 150)
    a = O.gptq(W, U, 4, 32, False, 128)
    rr = O.gptq_replay(W, U, a.codes, a.scales, a.zeros, 4, 32, False, 128)
    assert rr.forced_codes == rr.hard_codes == rr.hard_params == rr.forced_params == 0


def test_replay_flags_planted_far_mistake_and_forces_near_one():
    _, W, _, _, U = _rand_problem(61, 6, 128, 150)
    a = O.gptq(W, U, 4, 32, False, 128)
    dist = O.boundary_distance(a.pre, np.repeat(a.scales.T, 32, axis=1), np.repeat(a.zeros.T, 32, axis=1), 15)
    # planted far mistake: the entry farthest from any boundary gets a different code
    far = np.unravel_index(np.argmax(dist), dist.shape)
    bad = a.codes.copy()
    bad[far] = bad[far] + 1 if bad[far] < 15 else bad[far] - 1
    rr = O.gptq_replay(W, U, bad, a.scales, a.zeros, 4, 32, False, 128)
    assert rr.hard_codes >= 1
    # near-boundary disagreement: move one weight onto a boundary, flip it, replay with a loose tolerance
    near = np.unravel_index(np.argmin(dist), dist.shape)
    bad2 = a.codes.copy()
    x = a.pre[near] / a.scales[near[1] // 32, near[0]] + a.zeros[near[1] // 32, near[0]]
    bad2[near] = int(np.floor(x)) if a.codes[near] == int(np.floor(x)) + 1 else int(np.floor(x)) + 1
    bad2[near] = min(max(bad2[near], 0), 15)
    if bad2[near] != a.codes[near]:
        tol = float(dist[near]) * 1.0001 + 1e-300
        rr2 = O.gptq_replay(W, U, bad2, a.scales, a.zeros, 4, 32, False, 128, tol=tol)
        assert rr2.forced_codes >= 1


def test_boundary_distance_closed_form():
    s, z = 0.1, 3.0
    # w = 0.1*(1.5-3) + 0.004 -> grid coordinate 1.54, nearest boundary 1.5 -> distance 0.004
    assert O.boundary_distance(np.array([0.1 * (1.5 - 3) + 0.004]), s, z, 15)[0] == pytest.approx(0.004, rel=1e-9)
    # clamped low: x = -2 -> only boundary 0.5 matters -> 2.5 grid units
    assert O.boundary_distance(np.array([0.1 * (-2 - 3)]), s, z, 15)[0] == pytest.approx(0.25, rel=1e-9)


# ---------------------------------------------------------------- activation ordering

def test_act_abs_sum_closed_form():
    # X[t, c] = (-1)^t (t + 1) (c + 1): sum_t |X[t, c]| = (c + 1) n (n + 1) / 2, exactly
    n, d = 37, 9
    t = np.arange(n)[:, None]
    c = np.arange(d)[None, :]
    X = np.where(t % 2 == 0, 1.0, -1.0) * (t + 1) * (c + 1)
    np.testing.assert_array_equal(O.act_abs_sum(X), (np.arange(d) + 1) * n * (n + 1) / 2)


def test_act_order_directions_and_ties():
    a = np.array([3.0, 1.0, 2.0, 1.0, 5.0, 0.0])
    np.testing.assert_array_equal(O.act_order(a, O.ACT_ASCENDING), [5, 1, 3, 2, 0, 4])
    np.testing.assert_array_equal(O.act_order(a, O.ACT_DESCENDING), [4, 0, 2, 1, 3, 5])
    # group index of column perm[k] is k // g
    np.testing.assert_array_equal(O.g_idx_of(np.array([5, 1, 3, 2, 0, 4]), 2), [2, 0, 1, 1, 2, 0])
    np.testing.assert_array_equal(O.g_idx_of(np.array([2, 0, 1]), -1), [0, 0, 0])


@pytest.mark.parametrize("seed,desc", [(60, 1), (61, 2), (62, 1), (63, 2)])
@pytest.mark.parametrize("g", [4, -1])
def test_act_order_equals_literal_obs_in_that_order(seed, desc, g):
    # an independent algorithm: OBS on the original coordinates, visiting columns in
    # the order, re-inverting the remaining Hessian each step (no permuted copies)
    X, W, H, Hd, U = _rand_problem(seed, 5, 12, 30, hot=2)
    perm = O.act_order(O.act_abs_sum(X), desc)
    a = O.gptq_act_order(W, H, perm, 3, g, False, block_size=0)
    b = O.gptq_naive_obs(W, Hd, 3, g, False, order=perm)
    np.testing.assert_array_equal(a.codes, b.codes)
    np.testing.assert_allclose(a.scales, b.scales, rtol=0, atol=0)
    np.testing.assert_array_equal(a.zeros, b.zeros)
    np.testing.assert_allclose(a.what, b.what, rtol=0, atol=1e-15)


def test_act_order_identity_order_is_plain_gptq():
    # columns whose activation sums already increase: the ascending order is the identity
    rng = np.random.default_rng(70)
    d_in, n = 64, 96
    X = rng.standard_normal((n, d_in))
    X *= (1.0 + 0.1 * np.arange(d_in))[None, :] / np.sum(np.abs(X), axis=0)[None, :]
    a = O.act_abs_sum(X)
    assert np.all(np.diff(a) > 0)
    perm = O.act_order(a, O.ACT_ASCENDING)
    np.testing.assert_array_equal(perm, np.arange(d_in))
    W = rng.standard_normal((8, d_in)) * 0.02
    ao = O.gptq_act_order(W, O.hessian(X), perm, 4, 16, False)
    plain, _, _, lam = O.quantize_layer(W, X, 4, 16, False)
    np.testing.assert_array_equal(ao.codes, plain.codes)
    np.testing.assert_array_equal(ao.g_idx, np.arange(d_in) // 16)
    assert ao.lam == lam


@pytest.mark.parametrize("seed", [71, 72])
def test_act_order_equivariant_under_column_relabelling(seed):
    # relabelling the input channels of W and X relabels the codes and g_idx the same way
    rng = np.random.default_rng(seed)
    X, W, H, _, _ = _rand_problem(seed, 6, 32, 64, hot=3)
    Q = rng.permutation(32)
    r1 = O.gptq_act_order(W, H, O.act_order(O.act_abs_sum(X), 1), 4, 8, False)
    XQ, WQ = X[:, Q], W[:, Q]
    r2 = O.gptq_act_order(WQ, O.hessian(XQ), O.act_order(O.act_abs_sum(XQ), 1), 4, 8, False)
    np.testing.assert_array_equal(r2.codes, r1.codes[:, Q])
    np.testing.assert_array_equal(r2.g_idx, r1.g_idx[Q])
    np.testing.assert_array_equal(r2.scales, r1.scales)


def test_act_order_error_identity_and_packed_roundtrip():
    # sum_c e_c^2 of the permuted loop equals (W0 - W_hat) Hd (W0 - W_hat)^T in the
    # original coordinates; packing + g_idx dequantization reproduces W_hat
    X, W, H, Hd, _ = _rand_problem(73, 7, 48, 80, hot=2)
    perm = O.act_order(O.act_abs_sum(X), 1)
    r = O.gptq_act_order(W, H, perm, 4, 16, False, block_size=16)
    D = W - r.what
    np.testing.assert_allclose(np.sum(r.inner.err ** 2, axis=1), np.einsum("oi,ij,oj->o", D, Hd, D), rtol=1e-9)
    qw = O.pack_qweight(r.codes, 4)
    qz = O.pack_qzeros(r.zeros, 4)
    Wh = O.dequant_packed(qw, r.scales, qz, 7, 48, 4, 16, False, g_idx=r.g_idx)
    np.testing.assert_array_equal(Wh, r.what)


# ---------------------------------------------------------------- dequantizing GEMM

def test_dequant_gemm_hand_example():
    # 2 x 4 weights, 4-bit, groups of 2 along d_in; W_hat by hand:
    #   row 0: 0.5 (1-1), 0.5 (2-1), 2 (3-0), 2 (4-0)   = [0, 0.5, 6, 8]
    #   row 1: 0.25 (15-8), 0.25 (0-8), 1 (7-7), 1 (8-7) = [1.75, -2, 0, 1]
    codes = np.array([[1, 2, 3, 4], [15, 0, 7, 8]])
    scales = np.array([[0.5, 0.25], [2.0, 1.0]])
    zeros = np.array([[1, 8], [0, 7]])
    X = np.array([[1.0, 1.0, 1.0, 1.0], [1.0, -1.0, 0.0, 2.0]])
    Y = O.dequant_gemm(X, O.pack_qweight(codes, 4), scales, O.pack_qzeros(zeros, 4), 2, 4, 4, 2, False)
    np.testing.assert_array_equal(Y, [[14.5, 0.75], [15.5, 5.75]])


def test_dequant_gemm_matches_the_column_loops_own_weights():
    # packed arrays -> Y equals X times the dequantized weights the column loop produced
    X, W, H, Hd, U = _rand_problem(80, 12, 64, 40, hot=2)
    r = O.gptq(W, U, 4, 16, False, 16)
    Y = O.dequant_gemm(X, O.pack_qweight(r.codes, 4), r.scales, O.pack_qzeros(r.zeros, 4), 12, 64, 4, 16, False)
    np.testing.assert_allclose(Y, X @ r.what.T, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- GPTQ-2D (two-sided rounding)

def _spd(rng, k, spread=1.0):
    A = rng.standard_normal((k, k)) * np.exp(spread * rng.standard_normal(k))[None, :]
    return A.T @ A + 0.1 * np.eye(k), A


def _problem2d(seed, m, n):
    rng = np.random.default_rng(seed)
    G_left, A = _spd(rng, m)
    G_right, B = _spd(rng, n)
    X = rng.standard_normal((m, n)) * 3.0
    return X, G_left, G_right, A, B


@pytest.mark.parametrize("seed", range(90, 94))
def test_gptq2d_one_sided_case_is_columnwise_gptq(seed):
    # G_right = I: every column is an independent one-sided GPTQ problem with metric G_left
    X, G_left, _, _, _ = _problem2d(seed, 6, 5)
    Z = O.gptq2d_vectorized(X, G_left, np.eye(5))
    U_left = O.hinv_upper_cholesky(G_left)
    r = O.gptq(X.T, U_left, 4, -1, False, block_size=0, fixed_grid=(np.ones(5), np.zeros(5)))
    np.testing.assert_array_equal(Z, r.codes.T)


@pytest.mark.parametrize("seed", range(94, 98))
def test_gptq2d_is_babai_on_the_kronecker_lattice(seed):
    X, G_left, G_right, _, _ = _problem2d(seed, 4, 3)
    Z = O.gptq2d_vectorized(X, G_left, G_right)
    G = np.kron(G_right, G_left)
    ev, V = np.linalg.eigh(G)
    basis = V @ np.diag(np.sqrt(ev)) @ V.T          # independent basis with basis^T basis = G
    z = O.babai_nearest_plane(X.reshape(-1, order="F"), basis)
    np.testing.assert_array_equal(Z.reshape(-1, order="F"), z)


def test_gptq2d_kronecker_factor_structure():
    # the upper Cholesky factor of (G_right (x) G_left)^-1 is U_right (x) U_left
    X, G_left, G_right, _, _ = _problem2d(98, 5, 4)
    U = O.hinv_upper_cholesky(np.kron(G_right, G_left))
    K = np.kron(O.hinv_upper_cholesky(G_right), O.hinv_upper_cholesky(G_left))
    np.testing.assert_allclose(U, K, rtol=0, atol=1e-10 * np.abs(K).max())


@pytest.mark.parametrize("seed", range(100, 106))
def test_gptq2d_bruteforce_bracket(seed):
    # best integer matrix <= two-sided GPTQ <= Babai's bound on the Kronecker lattice
    X, G_left, G_right, _, _ = _problem2d(seed, 2, 2)
    Z = O.gptq2d_vectorized(X, G_left, G_right)
    best = min(O.gptq2d_loss(X, np.array(c, dtype=float).reshape(2, 2), G_left, G_right)
               for c in itertools.product(*[range(int(np.floor(v)) - 2, int(np.floor(v)) + 4) for v in X.reshape(-1)]))
    got = O.gptq2d_loss(X, Z, G_left, G_right)
    bound = O.babai_bound(O.hinv_upper_cholesky(np.kron(G_right, G_left)), 1.0)
    assert best <= got + 1e-12
    assert got <= bound + 1e-12


@pytest.mark.parametrize("seed,m,n", [(110, 5, 7), (111, 8, 3), (112, 6, 6), (113, 1, 9), (114, 9, 1),
                                      (115, 12, 10), (116, 16, 3)])
def test_gptq2d_antidiagonal_route_gives_the_same_integers(seed, m, n):
    # the summary's claim ("方法", "核心洞察"): the anti-diagonal route gives exactly the
    # integers of the quartic vectorized route
    X, G_left, G_right, _, _ = _problem2d(seed, m, n)
    Z = O.gptq2d_vectorized(X, G_left, G_right)
    Zad = O.gptq2d_antidiagonal(X, O.hinv_upper_cholesky(G_left), O.hinv_upper_cholesky(G_right))
    np.testing.assert_array_equal(Z, Zad)


# ---------------------------------------------------------------- replay protocol: scale and zero decisions
#
# The group-size article fixes the metadata of a group: a 16-bit scale and a b-bit zero
# point ("存储代价").  The replay adopts the other side's scale or zero only when the
# oracle's own unrounded quantity lies within tol (weight units) of that decision's
# rounding tie.  These pins build groups whose distance to the tie is known exactly, so a
# distance measured in the wrong units (grid units, raw-scale units) or against the wrong
# point (the other value instead of the tie) fails one of them.

def _f16_neighbours(s0: float) -> tuple[float, float]:
    a = np.float16(s0)
    return float(a), float(np.nextafter(a, np.float16(np.inf)))


def _one_group_replay(v, other_scale, other_zero, bits, tol):
    """Replay a single row holding one group (no compensation: U = I)."""
    W = np.asarray(v, dtype=np.float64)[None, :]
    g = W.shape[1]
    maxq = (1 << bits) - 1
    codes = np.clip(np.rint(W / other_scale) + other_zero, 0, maxq).astype(np.int64)
    scales = np.array([[other_scale]])
    zeros = np.array([[other_zero]], dtype=np.int64)
    return O.gptq_replay(W, np.eye(g), codes, scales, zeros, bits, g, False, g, tol=tol)


@pytest.mark.parametrize("delta", [1e-6, -1e-6, 3e-7])
def test_replay_scale_tie_distance_is_the_range_distance_in_weight_units(delta):
    bits, maxq = 4, 15
    s0, s1 = _f16_neighbours(0.0068359375)          # two adjacent fp16 scales
    mid = 0.5 * (s0 + s1)                            # the fp16 rounding tie of raw = range / maxq
    hi = maxq * mid + delta                          # asymmetric, all values >= 0: lo = 0, range = hi
    rng = np.random.default_rng(7)
    v = np.concatenate([[hi], rng.uniform(0.0, hi, 31)])
    own = s1 if delta > 0 else s0                    # what the oracle rounds to
    other = s0 if delta > 0 else s1                  # the other side's neighbouring fp16 scale
    assert float(O.fp16_round(hi / maxq)) == own
    loose = _one_group_replay(v, other, 0, bits, tol=2.0 * abs(delta))
    assert loose.forced_params == 1 and loose.hard_params == 0
    strict = _one_group_replay(v, other, 0, bits, tol=0.5 * abs(delta))
    assert strict.hard_params == 1 and strict.forced_params == 0


@pytest.mark.parametrize("k,eps", [(7, 1e-6), (3, -1e-6), (12, 4e-7)])
def test_replay_zero_tie_distance_is_in_weight_units(k, eps):
    bits, maxq = 4, 15
    s = float(np.float16(0.0068359375))
    lo = -(k + 0.5) * s - eps                        # -lo / s = k + 1/2 + eps / s
    hi = lo + maxq * s                               # range = maxq * s exactly: raw rounds to s
    rng = np.random.default_rng(k)
    v = np.concatenate([[lo, hi], rng.uniform(lo, hi, 30)])
    _, z, _, _, _ = O.group_params(v[None, :], bits, False)
    own = k + 1 if eps > 0 else k
    assert int(z[0]) == own
    other = k if eps > 0 else k + 1
    loose = _one_group_replay(v, s, other, bits, tol=2.0 * abs(eps))
    assert loose.forced_params == 1 and loose.hard_params == 0
    strict = _one_group_replay(v, s, other, bits, tol=0.5 * abs(eps))
    assert strict.hard_params == 1 and strict.forced_params == 0


def _far_from_tie_problem():
    _, W, _, _, U = _rand_problem(62, 8, 128, 150)
    a = O.gptq(W, U, 4, 32, False, 128)
    return W, U, a


def test_replay_flags_a_scale_one_fp16_ulp_off_far_from_its_tie():
    W, U, a = _far_from_tie_problem()
    # the group (of row 0) whose range lies farthest from both neighbouring fp16 ties
    best, best_d = None, -1.0
    for gi in range(a.scales.shape[0]):
        v = a.pre[0:1, 32 * gi:32 * gi + 32]
        s, _, raw, lo, hi = O.group_params(v, 4, False)
        lo_n = float(np.nextafter(np.float16(s[0]), np.float16(0)))
        hi_n = float(np.nextafter(np.float16(s[0]), np.float16(np.inf)))
        d = min(abs(raw[0] - 0.5 * (s[0] + lo_n)), abs(raw[0] - 0.5 * (s[0] + hi_n))) * 15
        if d > best_d:
            best, best_d = gi, d
    assert best_d > 1e-5
    sc = a.scales.copy()
    sc[best, 0] = float(np.nextafter(np.float16(sc[best, 0]), np.float16(np.inf)))
    rr = O.gptq_replay(W, U, a.codes, sc, a.zeros, 4, 32, False, 128)
    assert rr.hard_params >= 1


def test_replay_flags_a_zero_point_off_by_one_far_from_its_tie():
    W, U, a = _far_from_tie_problem()
    best, best_d = None, -1.0
    for gi in range(a.scales.shape[0]):
        v = a.pre[0:1, 32 * gi:32 * gi + 32]
        s, z, _, lo, _ = O.group_params(v, 4, False)
        x = -lo[0] / s[0]
        d = abs(x - (np.floor(x) + 0.5)) * s[0]      # weight-unit distance to the nearest tie
        if 0 < z[0] < 15 and d > best_d:
            best, best_d = gi, d
    assert best is not None and best_d > 1e-5
    zz = a.zeros.copy()
    zz[best, 0] += 1
    rr = O.gptq_replay(W, U, a.codes, a.scales, zz, 4, 32, False, 128)
    assert rr.hard_params >= 1
