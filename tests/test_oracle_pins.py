"""Pins of the float64 oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: each check is a hand-worked
fixture (tests/golden), a closed form, brute force, an independent linear-algebra
solve, or an invariant of the method, chosen so that a dropped term, a wrong
sign or index, or a transposed operand in the oracle fails at least one test.
"""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import gptq_ref as o
from post_weight_quantization_20_b200.synthetic import gen_spd

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


def _layer(seed, R, C, tokens=None, mix=0):
    g = _rng(seed)
    n = tokens or 4 * C
    X = g.standard_normal((n, C))
    if mix:
        X += g.standard_normal((n, mix)) @ g.standard_normal((mix, C))
    X *= g.uniform(0.3, 3.0, size=C)
    W = 0.02 * g.standard_normal((R, C))
    return W, X


# --------------------------------------------------------------------------- Hessian
def test_hessian_hand_fixture():
    f = _load("hessian_small.json")
    X = np.array(f["X"])
    H, n = o.hessian(X)
    assert n == f["n"]
    np.testing.assert_allclose(H, f["H"], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(o.damp(H, f["damp"]), f["H_damped"], rtol=1e-14)
    assert list(o.act_order_perm(H)) == f["act_order_perm"]


@pytest.mark.parametrize("chunk", [1, 3, 7, None])
def test_hessian_chunks_equal_sum_of_outer_products(chunk):
    g = _rng(1)
    X = g.standard_normal((23, 5))
    H, n = o.hessian(X, chunk=chunk)
    brute = np.zeros((5, 5))
    for t in range(X.shape[0]):
        brute += np.outer(X[t], X[t])
    brute *= 2.0 / X.shape[0]
    assert n == 23
    np.testing.assert_allclose(H, brute, rtol=1e-13, atol=1e-14)


def test_hessian_empty_chunk_is_noop():
    H = np.eye(3)
    H2, n = o.hessian_accumulate(H, 5, np.zeros((0, 3)))
    assert n == 5 and np.array_equal(H2, H)


# --------------------------------------------------------------------------- act-order, damping
def test_act_order_descending_with_stable_ties():
    H = np.diag([2.0, 5.0, 5.0, 1.0, 5.0])
    assert list(o.act_order_perm(H)) == [1, 2, 4, 0, 3]


def test_damp_is_relative_to_mean_diagonal():
    H = np.diag([1.0, 3.0]) + np.array([[0, 0.5], [0.5, 0]])
    Hd = o.damp(H, 0.1)
    np.testing.assert_allclose(Hd - H, 0.2 * np.eye(2), rtol=1e-15)


# --------------------------------------------------------------------------- inverse Cholesky factor
def test_inverse_cholesky_closed_form_2x2():
    a, b, c = 4.0, 1.5, 2.0
    det = a * c - b * b
    U = o.inverse_cholesky_upper(np.array([[a, b], [b, c]]))
    expect = np.array([[np.sqrt(c / det), -b / np.sqrt(c * det)], [0.0, 1.0 / np.sqrt(c)]])
    np.testing.assert_allclose(U, expect, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("cond", [1.0, 1e3, 1e6])
def test_inverse_cholesky_factor_properties(cond):
    Hp = gen_spd(37, seed=3, cond=cond)
    U = o.inverse_cholesky_upper(Hp)
    assert np.all(np.tril(U, -1) == 0)
    assert np.all(np.diag(U) > 0)
    err = np.abs(U.T @ U @ Hp - np.eye(37)).max()
    assert err < 1e-13 * max(cond, 1.0) * 10


def test_not_positive_definite_raises():
    with pytest.raises(o.NotPositiveDefinite):
        o.inverse_cholesky_upper(np.zeros((3, 3)))
    x = np.array([[1.0, 2.0, 3.0]])
    with pytest.raises(o.NotPositiveDefinite):
        o.prepare(2 * x.T @ x, 0.0, False)


# --------------------------------------------------------------------------- grid / quantizer
@pytest.mark.parametrize("case", _load("grid_rows.json")["cases"], ids=lambda c: c["name"])
def test_grid_hand_fixtures(case):
    row = np.array([case["row"]])
    s, z, _ = o.grid(row, case["bits"], case["sym"])
    if "scale" in case:
        assert float(s[0]) == case["scale"]
    assert float(z[0]) == case["zero"]
    c, Q, _ = o.quantize(row[0][:, None].T.T.reshape(1, -1)[0], np.repeat(s, row.shape[1]),
                         np.repeat(z, row.shape[1]), case["bits"])
    assert list(c) == case["codes"]
    np.testing.assert_array_equal(Q, np.array(case["Q"]))


def test_grid_clamp_fixture():
    f = _load("grid_rows.json")["clamp"]
    x = np.array(f["x"])
    s = np.full(len(x), np.float32(f["scale"]))
    z = np.full(len(x), np.float32(f["zero"]))
    c, Q, _ = o.quantize(x, s, z, f["bits"])
    assert list(c) == f["codes"]
    np.testing.assert_array_equal(Q, f["Q"])


@pytest.mark.parametrize("bits,sym", [(2, False), (3, False), (4, False), (4, True), (3, True)])
def test_grid_properties(bits, sym):
    g = _rng(bits + 10 * sym)
    v = g.standard_normal((200, 17)) * g.uniform(0.001, 3.0, size=(200, 1)) + g.uniform(-1, 1, (200, 1))
    maxq = 2 ** bits - 1
    s, z, _ = o.grid(v, bits, sym)
    assert np.all(z == np.rint(z)) and np.all((z >= 0) & (z <= maxq))
    c, Q, _ = o.quantize(v, s[:, None], z[:, None], bits)
    assert np.all((c >= 0) & (c <= maxq))
    # Q lies on the grid s*(k - z)
    k = Q / s[:, None].astype(np.float64) + z[:, None]
    np.testing.assert_allclose(k, np.rint(k), atol=1e-9)
    # values inside the covered range are within half a step (float32 division slack)
    lo = s[:, None] * (0 - z[:, None]).astype(np.float64)
    hi = s[:, None] * (maxq - z[:, None]).astype(np.float64)
    inside = (v >= lo) & (v <= hi)
    err = np.abs(v - Q) / s[:, None]
    assert np.all(err[inside] <= 0.5 + 1e-5)
    # zero is exactly representable
    c0, Q0, _ = o.quantize(np.zeros(200), s, z, bits)
    assert np.all(Q0 == 0.0)


# --------------------------------------------------------------------------- the sweep
def _prep(seed, R, C, act=False, mix=3, rel=0.01):
    W, X = _layer(seed, R, C, mix=mix)
    H, n = o.hessian(X)
    perm, Hp, U = o.prepare(H, rel, act)
    return W, X, H, n, perm, Hp, U


@pytest.mark.parametrize("k", [1, 2, 5, 11, 19])
@pytest.mark.parametrize("group", [0, 4])
def test_sweep_state_equals_constrained_least_squares(k, group):
    """After k columns, the remaining weights minimise (v-w)Hp(v-w)^T with v_K = Q_K
    ([Deep-dive §2.2] OBS; solved here directly with np.linalg.solve)."""
    W, X, H, n, perm, Hp, U = _prep(5, 6, 24)
    Wp = W[:, perm]
    res = o.sweep(Wp, U, 3, group, False, block_size=8, stop_after=k)
    K, F = slice(0, k), slice(k, 24)
    dK = Wp[:, K] - res["Q"][:, K]
    expect = Wp[:, F] + np.linalg.solve(Hp[F, F], Hp[F, K] @ dK.T).T
    np.testing.assert_allclose(res["W"][:, F], expect, rtol=1e-9, atol=1e-12)


def _naive_fixed_order_obq(Wp, Hp, bits, group, sym):
    """Fixed-order OBQ with an explicit inverse and Gaussian-elimination downdates."""
    W = Wp.copy()
    R, C = W.shape
    Hinv = np.linalg.inv(Hp)
    codes = np.zeros((R, C), dtype=np.int64)
    Q = np.zeros((R, C))
    losses = np.zeros(C)
    if group == 0:
        s, z, _ = o.grid(Wp, bits, sym)
    for q in range(C):
        if group and q % group == 0:
            s, z, _ = o.grid(W[:, q:q + group], bits, sym)
        c, Qq, _ = o.quantize(W[:, q], s, z, bits)
        codes[:, q], Q[:, q] = c, Qq
        d = Hinv[q, q]
        losses[q] = np.sum((W[:, q] - Qq) ** 2) / (2 * d)
        W -= np.outer((W[:, q] - Qq) / d, Hinv[q, :])
        W[:, q] = Qq
        Hinv = Hinv - np.outer(Hinv[:, q], Hinv[q, :]) / d
    return codes, Q, losses


@pytest.mark.parametrize("bits,group,sym", [(4, 0, False), (3, 4, False), (2, 8, False), (4, 8, True)])
def test_sweep_matches_explicit_inverse_obq(bits, group, sym):
    W, X, H, n, perm, Hp, U = _prep(7, 9, 32, act=True)
    res = o.sweep(W[:, perm], U, bits, group, sym, block_size=8)
    c2, Q2, l2 = _naive_fixed_order_obq(W[:, perm], Hp, bits, group, sym)
    np.testing.assert_array_equal(res["codes"], c2)
    np.testing.assert_allclose(res["Q"], Q2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(res["losses"], l2, rtol=1e-9, atol=1e-18)


@pytest.mark.parametrize("group", [0, 8])
def test_lazy_batching_is_exact(group):
    W, X, H, n, perm, Hp, U = _prep(9, 12, 48)
    ref = o.sweep(W[:, perm], U, 4, group, False, block_size=1)
    for B in (2, 4, 8, 16, 48):
        if not o.supported(group, B):
            continue
        r = o.sweep(W[:, perm], U, 4, group, False, block_size=B)
        np.testing.assert_array_equal(r["codes"], ref["codes"])
        np.testing.assert_allclose(r["Q"], ref["Q"], atol=1e-14)
        np.testing.assert_allclose(r["losses"], ref["losses"], rtol=1e-10)


def test_unsupported_group_block_pair():
    assert not o.supported(96, 128)
    assert o.supported(64, 128) and o.supported(256, 128) and o.supported(0, 7)
    with pytest.raises(ValueError):
        o.sweep(np.zeros((1, 4)), np.eye(4), 4, 3, False, block_size=2)


@pytest.mark.parametrize("group", [0, 4])
def test_diagonal_hessian_reduces_to_round_to_nearest(group):
    """No cross-column curvature -> no compensation ([Deep-dive §1.2] RTN)."""
    g = _rng(11)
    W = 0.02 * g.standard_normal((10, 16))
    H = np.diag(g.uniform(0.5, 4.0, 16))
    out = o.gptq_quantize(W, H, bits=3, group_size=group, damp_rel=0.01, block_size=8)
    for j0 in range(0, 16, group or 16):
        j1 = j0 + (group or 16)
        s, z, _ = o.grid(W[:, j0:j1], 3, False)
        c, Q, _ = o.quantize(W[:, j0:j1], s[:, None], z[:, None], 3)
        np.testing.assert_array_equal(out["codes"][:, j0:j1], c)


@pytest.mark.parametrize("bits,group,sym,act", [(4, 0, False, False), (4, 8, False, True),
                                                  (3, 0, True, False), (2, 4, False, True)])
def test_loss_identity(bits, group, sym, act):
    """sum of per-column losses = 1/2 tr((Wp-Qp) Hp (Wp-Qp)^T) ([Deep-dive §2.1] quadratic term)."""
    W, X, H, n, perm, Hp, U = _prep(13, 15, 40, act=act)
    out = o.gptq_quantize(W, H, bits, group, sym, act, 0.01, 8)
    lhs = float(np.sum(out["losses"]))
    rhs = o.half_trace_loss(out["Wp"], out["Qp"], out["Hp"])
    assert abs(lhs - rhs) <= 1e-9 * abs(rhs)


@pytest.mark.parametrize("bits", [2, 4])
def test_exhaustive_tiny_layer(bits):
    """2 x 4 layer: codes on the grid; the brute-force optimum over all code vectors
    (same per-row grid) is no worse than the greedy GPTQ sequence."""
    g = _rng(17 + bits)
    W = 0.05 * g.standard_normal((2, 4))
    Hp = gen_spd(4, seed=bits, cond=50.0)
    U = o.inverse_cholesky_upper(Hp)
    res = o.sweep(W, U, bits, 0, False, block_size=4)
    maxq = 2 ** bits - 1
    s, z, _ = o.grid(W, bits, False)
    assert np.all((res["codes"] >= 0) & (res["codes"] <= maxq))
    for r in range(2):
        np.testing.assert_allclose(res["Q"][r], float(s[r]) * (res["codes"][r] - float(z[r])), atol=0)
        combos = np.array(list(itertools.product(range(maxq + 1), repeat=4)), dtype=np.float64)
        Qall = float(s[r]) * (combos - float(z[r]))
        D = W[r][None, :] - Qall
        losses = 0.5 * np.sum((D @ Hp) * D, axis=1)
        greedy = 0.5 * float((W[r] - res["Q"][r]) @ Hp @ (W[r] - res["Q"][r]))
        assert losses.min() <= greedy + 1e-15
        assert abs(np.sum(res["losses"]) - 0) >= 0  # losses are finite
    assert np.all(np.isfinite(res["losses"]))


def test_codes_invariant_under_hessian_scaling():
    W, X, H, n, *_ = _prep(19, 8, 32, mix=2)
    a = o.gptq_quantize(W, H, 4, 8, False, True, 0.01, 8)
    b = o.gptq_quantize(W, 4.0 * H, 4, 8, False, True, 0.01, 8)
    c = o.gptq_quantize(W, 3.0 * H, 4, 8, False, True, 0.01, 8)
    np.testing.assert_array_equal(a["codes"], b["codes"])
    np.testing.assert_array_equal(a["Q"], b["Q"])
    np.testing.assert_array_equal(a["codes"], c["codes"])


def test_act_order_with_constant_diagonal_is_natural_order():
    g = _rng(23)
    A = g.standard_normal((16, 16)) * 0.1
    H = A + A.T
    np.fill_diagonal(H, 5.0)
    W = 0.02 * g.standard_normal((5, 16))
    a = o.gptq_quantize(W, H, 4, 4, False, True, 0.01, 8)
    b = o.gptq_quantize(W, H, 4, 4, False, False, 0.01, 8)
    assert list(a["perm"]) == list(range(16))
    np.testing.assert_array_equal(a["codes"], b["codes"])


def test_act_order_equivariant_under_column_permutation():
    W, X, H, n, *_ = _prep(29, 7, 24, mix=2)
    pi = _rng(30).permutation(24)
    a = o.gptq_quantize(W, H, 4, 8, False, True, 0.01, 8)
    b = o.gptq_quantize(W[:, pi], H[np.ix_(pi, pi)], 4, 8, False, True, 0.01, 8)
    np.testing.assert_array_equal(b["codes"], a["codes"][:, pi])
    np.testing.assert_allclose(b["losses"], a["losses"][pi], rtol=1e-12)


def test_dequantization_consistency_of_outputs():
    """Q[:, c] = scales[:, g_idx[c]] * (codes[:, c] - zeros[:, g_idx[c]]) in the original order."""
    W, X, H, n, *_ = _prep(31, 6, 32)
    out = o.gptq_quantize(W, H, 4, 8, False, True, 0.01, 8)
    s = out["scales"][:, out["g_idx"]].astype(np.float64)
    z = out["zeros"][:, out["g_idx"]].astype(np.float64)
    np.testing.assert_array_equal(out["Q"], s * (out["codes"] - z))
    assert sorted(np.bincount(out["g_idx"])) == [8, 8, 8, 8]


def test_reconstruction_error_matches_direct_product():
    W, X, H, n, *_ = _prep(37, 5, 12)
    out = o.gptq_quantize(W, H, 4, 0, False, False, 0.01, 4)
    direct = float(np.sum(((W - out["Q"]) @ X.T) ** 2))
    assert abs(o.reconstruction_error(W, out["Q"], H, n) - direct) <= 1e-10 * direct


def test_gptq_beats_round_to_nearest_on_correlated_layer():
    """Compensation lowers the layer objective relative to RTN ([Deep-dive §1.2, §2.2])."""
    W, X, H, n, *_ = _prep(41, 64, 64, mix=8)
    out = o.gptq_quantize(W, H, 3, 0, False, False, 0.01, 16)
    s, z, _ = o.grid(W, 3, False)
    _, Qr, _ = o.quantize(W, s[:, None], z[:, None], 3)
    assert o.reconstruction_error(W, out["Q"], H, n) < 0.8 * o.reconstruction_error(W, Qr, H, n)


def test_hints_only_move_near_ties_to_a_neighbour():
    W, X, H, n, perm, Hp, U = _prep(43, 20, 32)
    base = o.sweep(W[:, perm], U, 4, 8, False, block_size=8)
    hint = base["codes"].copy()
    hint[0, 0] = (hint[0, 0] + 5) % 16                 # not a neighbour: rejected when near a tie
    r = o.sweep(W[:, perm], U, 4, 8, False, block_size=8, hints={"codes": hint}, tau=0.5)
    assert not r["forced"]["codes"]
    np.testing.assert_array_equal(r["codes"], base["codes"])
    assert ("code", 0, 0) in r["forced"]["bad_hint"]


# --------------------------------------------------------------------------- packing
@pytest.mark.parametrize("case", _load("pack_words.json")["cases"], ids=lambda c: f"{c['bits']}b-{len(c['codes'])}")
def test_pack_hand_fixtures(case):
    codes = np.array([case["codes"]])
    words = o.pack(codes, case["bits"])
    assert [int(w) for w in words[0]] == case["words"]
    np.testing.assert_array_equal(o.unpack(words, case["bits"], codes.shape[1]), codes)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("cols", [1, 7, 32, 33, 100])
def test_pack_matches_numpy_packbits(bits, cols):
    g = _rng(bits * 1000 + cols)
    codes = g.integers(0, 2 ** bits, size=(5, cols))
    # independent route: explode to bits, LSB first, then numpy's little-endian packbits
    bitmat = ((codes[:, :, None] >> np.arange(bits)) & 1).reshape(5, cols * bits).astype(np.uint8)
    nw = (cols * bits + 31) // 32
    padded = np.zeros((5, nw * 32), dtype=np.uint8)
    padded[:, :cols * bits] = bitmat
    expect = np.packbits(padded, axis=1, bitorder="little").view("<u4")
    np.testing.assert_array_equal(o.pack(codes, bits), expect)
    np.testing.assert_array_equal(o.unpack(o.pack(codes, bits), bits, cols), codes)


# --------------------------------------------------------------------------- degenerate inputs
def test_dead_input_channel_is_rounded_to_nearest_and_feeds_nothing():
    """X[:, j] = 0 makes column j of H zero; after damping, Hp couples nothing to j, so
    U has no off-diagonal entry in row or column j: column j is round-to-nearest of the
    original weights on the row's grid, and the other columns do not see it."""
    rng = np.random.default_rng(31)
    R, C, j = 12, 40, 17
    X = rng.standard_normal((500, C)) + 0.5 * rng.standard_normal((500, 1))
    X[:, j] = 0.0
    H, _ = o.hessian(X)
    W = 0.02 * rng.standard_normal((R, C))
    W[:, j] *= 0.1              # never a row's extreme, so the row grids ignore its sign
    out = o.gptq_quantize(W, H, bits=4, group_size=0, block_size=16)
    U = out["U"]
    assert np.all(U[j, j + 1:] == 0.0) and np.all(U[:j, j] == 0.0)
    s, z, _ = o.grid(W, 4, False)
    codes_j, Q_j, _ = o.quantize(W[:, j:j + 1], s[:, None], z[:, None], 4)
    np.testing.assert_array_equal(out["codes"][:, j], codes_j[:, 0])
    # the other columns do not see column j: flipping its sign (same row grids)
    # leaves every other code unchanged
    W2 = W.copy()
    W2[:, j] = -W[:, j]
    s2, z2, _ = o.grid(W2, 4, False)
    assert np.array_equal(s2, s) and np.array_equal(z2, z)
    out2 = o.gptq_quantize(W2, H, bits=4, group_size=0, block_size=16)
    others = np.arange(C) != j
    np.testing.assert_array_equal(out2["codes"][:, others], out["codes"][:, others])


def test_all_zero_weight_row_quantizes_to_zero():
    """A row of zeros has the degenerate range [0, 0], widened to [-1, 1]: every code is
    the zero-point, Q = 0, and the row adds nothing to the losses."""
    rng = np.random.default_rng(32)
    R, C = 6, 32
    X = rng.standard_normal((300, C))
    H, _ = o.hessian(X)
    W = 0.02 * rng.standard_normal((R, C))
    W[2] = 0.0
    for bits, sym in ((4, False), (3, True)):
        out = o.gptq_quantize(W, H, bits=bits, group_size=0, sym=sym, block_size=8)
        zr = np.ravel(out["zeros"][2])[0]
        assert np.all(out["codes"][2] == int(zr))
        assert np.all(out["Q"][2] == 0.0)
        Wz = np.delete(W, 2, axis=0)
        ref = o.gptq_quantize(Wz, H, bits=bits, group_size=0, sym=sym, block_size=8)
        np.testing.assert_allclose(out["losses"], ref["losses"], rtol=1e-12, atol=0)


def test_all_zero_hessian_is_not_positive_definite():
    """H = 0 gives lambda = damp * mean(diag H) = 0 and a zero pivot."""
    with pytest.raises(o.NotPositiveDefinite):
        o.gptq_quantize(np.ones((2, 8)), np.zeros((8, 8)), bits=4, group_size=0)


# --------------------------------------------------------------------------- stored form
def test_dequant_matmul_hand_fixture():
    """One row of 4-bit codes 0..7 (packed word 0x76543210), scale 0.5, zero 3:
    Q = 0.5 (c - 3) = -1.5, -1, ..., 2; all-ones input gives 0.5 (28 - 24) = 2, and
    the input (1, -1, 0, ...) gives -1.5 - (-1) = -0.5."""
    packed = np.array([[0x76543210]], dtype=np.uint32)
    g_idx = np.zeros(8, dtype=np.int64)
    s, z = np.array([[0.5]], np.float32), np.array([[3.0]], np.float32)
    np.testing.assert_array_equal(o.dequantize(packed, s, z, g_idx, 4, 8)[0],
                                  [-1.5, -1.0, -0.5, 0.0, 0.5, 1.0, 1.5, 2.0])
    X = np.array([[1.0] * 8, [1.0, -1.0] + [0.0] * 6])
    np.testing.assert_array_equal(o.dequant_matmul(X, packed, s, z, g_idx, 4), [[2.0], [-0.5]])


@pytest.mark.parametrize("bits,group,sym,act", [(4, 8, False, True), (3, 0, False, False),
                                                (2, 4, True, True), (3, 16, False, True)])
def test_stored_form_reproduces_the_sweeps_weights(bits, group, sym, act):
    """Unpacking the stored codes and gathering each column's grid through g_idx gives
    exactly the Q the sweep formed column by column in sweep order (a transposed or
    un-gathered g_idx, or a wrong field offset, breaks the equality under act-order)."""
    W, X, H, n, *_ = _prep(41 + bits, 7, 32, act=act)
    out = o.gptq_quantize(W, H, bits, group, sym, act, 0.01, 8)
    if act:
        assert not np.all(np.diff(out["g_idx"]) >= 0)       # the gather is not the identity
    Q = o.dequantize(o.pack(out["codes"], bits), out["scales"], out["zeros"], out["g_idx"],
                     bits, 32)
    np.testing.assert_array_equal(Q, out["Q"])


def test_dequant_matmul_output_error_is_the_reconstruction_error():
    """||X W^T - Y||^2 with Y from the stored form equals (n/2) tr((W - Q) H (W - Q)^T)
    for the undamped H = 2 X^T X / n: the product's orientation pinned through the
    Hessian route ([Deep-dive §2.1])."""
    W, X, H, n, *_ = _prep(47, 9, 24, act=True)
    out = o.gptq_quantize(W, H, 4, 8, False, True, 0.01, 8)
    Y = o.dequant_matmul(X, o.pack(out["codes"], 4), out["scales"], out["zeros"], out["g_idx"], 4)
    assert Y.shape == (X.shape[0], W.shape[0])
    err = float(np.sum((X @ W.T - Y) ** 2))
    ref = o.reconstruction_error(W, out["Q"], H, n)
    assert abs(err - ref) <= 1e-9 * ref


def test_dequant_matmul_one_hot_inputs_pick_weight_columns():
    """Token e_c reads column c of Q for every output row."""
    W, X, H, n, *_ = _prep(53, 5, 16)
    out = o.gptq_quantize(W, H, 3, 4, False, False, 0.01, 4)
    Y = o.dequant_matmul(np.eye(16), o.pack(out["codes"], 3), out["scales"], out["zeros"],
                         out["g_idx"], 3)
    np.testing.assert_array_equal(Y, out["Q"].T)


@pytest.mark.parametrize("bits", [3, 4])
def test_packing_density_matches_the_quoted_model_sizes(bits):
    """A 175B-parameter model takes ~87.5 GB at 4 bits and ~65.6 GB at 3 bits
    ([Deep-dive §4.3]), i.e. exactly bits/8 bytes per weight: at the OPT-175B layer
    widths (12288, 49152 columns) the packed rows carry no padding."""
    for cols in (12288, 49152):
        codes = np.zeros((2, cols), dtype=np.int64)
        assert o.pack(codes, bits).nbytes == 2 * cols * bits // 8
    assert 175e9 * bits / 8 / 1e9 == pytest.approx({4: 87.5, 3: 65.6}[bits], abs=0.05)



def test_block_cholesky_matches_lapack():
    """The block Cholesky used above 46340 columns against LAPACK's unblocked one, with
    blocks of 64 on an order of 300 (a ragged last block)."""
    A = gen_spd(300, seed=12, cond=1e5)
    L = o._cholesky_lower_blocked(A, nb=64)
    assert np.allclose(np.triu(L, 1), 0.0)
    assert np.linalg.norm(L - np.linalg.cholesky(A)) <= 1e-12 * np.linalg.norm(L)
    # a block that is not positive definite is reported
    B = A.copy()
    B[200, 200] = -1.0
    with pytest.raises(o.NotPositiveDefinite):
        o._cholesky_lower_blocked(B, nb=64)


def test_block_triangular_inverse_matches_a_general_inverse():
    L = np.linalg.cholesky(gen_spd(300, seed=13, cond=1e4))
    X = o._tri_inverse_lower_blocked(L, nb=64)
    assert np.allclose(np.triu(X, 1), 0.0)
    assert np.abs(X @ L - np.eye(300)).max() < 1e-10
    assert np.linalg.norm(X - np.linalg.inv(L)) <= 1e-10 * np.linalg.norm(X)


def test_lower_gram_of_a_lower_triangular_matrix():
    X = np.tril(np.random.default_rng(14).standard_normal((300, 300)))
    G = o._lower_gram_of_lower(X, nb=64)
    full = X.T @ X
    for j0 in range(0, 300, 64):       # block columns: rows from the block's first column
        np.testing.assert_allclose(G[j0:, j0:j0 + 64], full[j0:, j0:j0 + 64], rtol=1e-12, atol=1e-12)
    assert np.all(G[np.triu_indices(300, 64)] == 0.0)


def test_wide_inverse_factor_route_matches_the_potri_route():
    """Above 46340 columns the oracle forms U on the block algorithms instead of
    SciPy's potri; both routes give the same U, checked here at a small order with
    blocks of 64, and it satisfies U^T U Hp = I."""
    Hp = gen_spd(200, seed=11, cond=1e4)
    U1 = o.inverse_cholesky_upper(Hp)
    U2 = o._inverse_cholesky_upper_wide(Hp, nb=64)
    assert np.allclose(np.tril(U2, -1), 0.0) and np.all(np.diag(U2) > 0)
    assert np.linalg.norm(U1 - U2) <= 1e-10 * np.linalg.norm(U1)
    assert np.abs(U2.T @ U2 @ Hp - np.eye(200)).max() < 1e-8
