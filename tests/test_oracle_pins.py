"""Pins for the oracle: each check is fixed by the GPTQ pages or by mathematics, not by the oracle.

A plausible mistake anywhere in the oracle (a dropped term, a wrong sign or index, a transposed
operand, quantizing the original instead of the compensated value) fails at least one of these;
``test_planted_mistakes_are_caught`` plants such mistakes on the CPU and checks that.
"""
import os

import numpy as np
import pytest

import oracle as O
from conftest import read_golden


def _spd(d, rng, cond=50.0):
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    ev = np.geomspace(1.0, cond, d)
    return (Q * ev) @ Q.T


def _correlated_x(n, d, rng):
    return rng.standard_normal((n, d)) @ (rng.standard_normal((d, d)) / np.sqrt(d))


# ------------------------------------------------------------------------------------ A1 / A2
def test_hessian_worked_example(golden_dir):
    g = read_golden(os.path.join(golden_dir, "hessian_example.txt"))
    X = np.array(g["x"], dtype=float).reshape(3, 2)
    np.testing.assert_array_equal(O.hessian(X), np.array(g["h"], dtype=float).reshape(2, 2))
    np.testing.assert_allclose(O.dampen(O.hessian(X), 0.01),
                               np.array(g["hd"], dtype=float).reshape(2, 2), rtol=0, atol=1e-12)


def test_hessian_is_sum_of_token_outer_products():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((37, 9))
    H = np.zeros((9, 9))
    for t in range(37):  # brute force, one token at a time
        for i in range(9):
            for j in range(9):
                H[i, j] += 2.0 * X[t, i] * X[t, j]
    np.testing.assert_allclose(O.hessian(X), H, rtol=1e-13, atol=1e-12)
    Hc = np.zeros((9, 9))
    for c0 in range(0, 37, 8):  # accumulation over token chunks is additive
        O.hessian_accumulate(Hc, X[c0:c0 + 8])
    np.testing.assert_allclose(Hc, H, rtol=1e-13, atol=1e-12)


def test_dampen_adds_fraction_of_mean_diagonal():
    H = np.diag([1.0, 2.0, 3.0, 6.0]) + 0.5
    Hd = O.dampen(H, 0.01)
    lam = 0.01 * np.mean([1.5, 2.5, 3.5, 6.5])
    np.testing.assert_allclose(np.diag(Hd) - np.diag(H), lam)
    off = ~np.eye(4, dtype=bool)
    np.testing.assert_array_equal(Hd[off], H[off])


# ------------------------------------------------------------------------------------ A3
@pytest.mark.parametrize("d", [1, 2, 7, 40, 130])
def test_upper_factor_of_inverse(d):
    rng = np.random.default_rng(d)
    Hd = _spd(d, rng, cond=1e3)
    U = O.inverse_upper_cholesky(Hd)
    assert np.allclose(np.tril(U, -1), 0.0)
    assert np.all(np.diag(U) > 0)
    # U^T U = Hd^-1  <=>  U Hd U^T = I (U invertible); no inverse needed on this side
    res = np.linalg.norm(U @ Hd @ U.T - np.eye(d)) / np.sqrt(d)
    assert res < 1e-10
    np.testing.assert_allclose(O.inverse_upper_cholesky_reversed(Hd), U, rtol=1e-8, atol=1e-10)


def test_upper_factor_worked_example(golden_dir):
    g = read_golden(os.path.join(golden_dir, "worked_example_d3.txt"))
    Hd = np.array(g["hd"], dtype=float).reshape(3, 3)
    U = O.inverse_upper_cholesky(Hd)
    np.testing.assert_allclose(np.diag(U), np.array(g["u_diag"], dtype=float), rtol=1e-14)
    np.testing.assert_allclose(U[0, 1] / U[0, 0], -2.0 / 3.0, rtol=1e-14)
    np.testing.assert_allclose(U[0, 2] / U[0, 0], 1.0 / 3.0, rtol=1e-14)
    np.testing.assert_allclose(U[1, 2] / U[1, 1], -0.5, rtol=1e-14)


# ------------------------------------------------------------------------------------ A4 grid
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_grid_is_a_uniform_asymmetric_quantizer(bits):
    rng = np.random.default_rng(bits)
    maxq = 2 ** bits - 1
    for _ in range(200):
        x = rng.standard_normal(64) * rng.uniform(0.01, 3.0) + rng.uniform(-1, 1)
        s, z = O.grid_params(x.min(), x.max(), bits)
        lo, hi = min(0.0, x.min()), max(0.0, x.max())
        assert 0 <= z <= maxq
        q = O.quantize_codes(x, s, z, bits)
        assert q.min() >= 0 and q.max() <= maxq
        assert O.dequantize(z, s, z) == 0.0          # zero is exactly representable
        np.testing.assert_allclose(s, (hi - lo) / maxq, rtol=1e-6)
        # every value of the range lies within half a step (plus the zero-point shift) of its level
        err = np.abs(O.dequantize(q, s, z) - x)
        assert err.max() <= s * 1.0 + 1e-6
        # an all-zero range falls back to [-1, 1]
    s, z = O.grid_params(0.0, 0.0, bits)
    np.testing.assert_allclose(s, 2.0 / maxq, rtol=1e-7)


def test_grid_in_range_error_is_half_step_for_symmetric_endpoints():
    # when -xmin/scale is an integer the grid contains both endpoints and rounding error <= scale/2
    s, z = O.grid_params(-0.3, 0.6, 2)  # scale 0.3, zero 1 -> levels -0.3, 0, 0.3, 0.6
    assert z == 1
    x = np.linspace(-0.3, 0.6, 1001)
    err = np.abs(O.dequantize(O.quantize_codes(x, s, z, 2), s, z) - x)
    assert err.max() <= 0.15 + 1e-6


# ------------------------------------------------------------------------------------ A5 / A6
def test_worked_example_d3(golden_dir):
    g = read_golden(os.path.join(golden_dir, "worked_example_d3.txt"))
    Hd = np.array(g["hd"], dtype=float).reshape(3, 3)
    w = np.array(g["w"], dtype=float)[None, :]
    bits = int(g["bits"][0])
    U = O.inverse_upper_cholesky(Hd)
    r = O.gptq_quantize(w, U, bits)
    np.testing.assert_array_equal(r["codes"][0], np.array(g["codes"], dtype=int))
    np.testing.assert_allclose(r["Err"][0], np.array(g["err"], dtype=float), rtol=1e-6)
    comp = r["Wq"][0] + r["Err"][0] * np.diag(U)  # compensated value = deq + delta
    np.testing.assert_allclose(comp, np.array(g["compensated"], dtype=float), rtol=1e-6)
    np.testing.assert_array_equal(O.rtn_quantize(w, bits)["codes"][0],
                                  np.array(g["rtn_codes"], dtype=int))


def _group_golden(golden_dir):
    g = read_golden(os.path.join(golden_dir, "worked_example_group.txt"))
    Hd = np.array(g["hd"], dtype=float).reshape(4, 4)
    w = np.array(g["w"], dtype=float)[None, :]
    return g, Hd, w, int(g["bits"][0]), int(g["group_size"][0])


def _check_group_golden(g, Hd, w, bits, gs, block_size):
    """True when the oracle reproduces every hand-worked value of the group example."""
    U = O.inverse_upper_cholesky(Hd)
    r = O.gptq_quantize(w, U, bits, gs, block_size)
    comp = r["Wq"][0] + r["Err"][0] * np.diag(U)
    return (np.array_equal(r["codes"][0], np.array(g["codes"], dtype=int))
            and np.allclose(r["scales"][0], np.array(g["scales"], dtype=float), rtol=1e-6, atol=0)
            and np.array_equal(r["zeros"][0], np.array(g["zeros"], dtype=int))
            and np.allclose(comp, np.array(g["compensated"], dtype=float), rtol=0, atol=1e-7)
            and np.allclose(r["Err"][0], np.array(g["err"], dtype=float), rtol=0, atol=1e-7))


@pytest.mark.parametrize("block_size", [0, 1, 2, 4])
def test_worked_example_group_grid_from_current_values(golden_dir, block_size):
    """Per-group grids are taken from the compensated values when the loop reaches the group: the
    hand-worked d = 4, g = 2 example, where compensation moves group 1's maximum and the grid from
    the original W would give a different code."""
    g, Hd, w, bits, gs = _group_golden(golden_dir)
    U = O.inverse_upper_cholesky(Hd)
    np.testing.assert_allclose(np.diag(U), np.array(g["u_diag"], dtype=float), rtol=1e-14)
    assert _check_group_golden(g, Hd, w, bits, gs, block_size)
    np.testing.assert_array_equal(O.rtn_quantize(w, bits, gs)["codes"][0], np.array(g["rtn_codes"], dtype=int))


@pytest.mark.parametrize("group_size", [0, 8])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_diagonal_hessian_reduces_to_rtn(bits, group_size):
    """H proportional to I (or any diagonal H): U is diagonal, no error is propagated, and GPTQ's
    codes are round-to-nearest's on the same grid."""
    rng = np.random.default_rng(10 * bits + group_size)
    W = rng.standard_normal((16, 32)) * 0.02
    for Hd in (3.7 * np.eye(32), np.diag(rng.uniform(0.5, 5.0, 32))):
        U = O.inverse_upper_cholesky(Hd)
        assert np.allclose(U, np.diag(np.diag(U)))
        g = O.gptq_quantize(W, U, bits, group_size, block_size=8)
        r = O.rtn_quantize(W, bits, group_size)
        np.testing.assert_array_equal(g["codes"], r["codes"])
        np.testing.assert_array_equal(g["scales"], r["scales"])
        np.testing.assert_array_equal(g["zeros"], r["zeros"])


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("group_size", [0, 4])
def test_cholesky_form_equals_explicit_obs(seed, group_size):
    rng = np.random.default_rng(seed)
    d = 16
    X = _correlated_x(64, d, rng)
    Hd = O.dampen(O.hessian(X), 0.01)
    W = rng.standard_normal((12, d)) * 0.02
    g = O.gptq_quantize(W, O.inverse_upper_cholesky(Hd), 3, group_size)
    o = O.obs_quantize(W, Hd, 3, group_size)
    np.testing.assert_array_equal(g["codes"], o["codes"])
    np.testing.assert_allclose(g["scales"], o["scales"], rtol=1e-6)
    np.testing.assert_array_equal(g["zeros"], o["zeros"])


@pytest.mark.parametrize("d,bits", [(3, 4), (4, 3), (5, 2), (6, 2), (6, 3)])
def test_greedy_matches_conditional_least_squares_and_bruteforce(d, bits):
    """(i) After any prefix of columns is fixed, the compensated remaining values are the
    least-squares optimum of the layer objective given that prefix; (ii) the exhaustive optimum over
    all code vectors is no worse than the greedy result or round-to-nearest."""
    rng = np.random.default_rng(100 * d + bits)
    for trial in range(4):
        X = _correlated_x(32, d, rng)
        Hd = O.dampen(O.hessian(X), 0.01)
        U = O.inverse_upper_cholesky(Hd)
        w = rng.standard_normal((1, d)) * 0.02
        r = O.gptq_quantize(w, U, bits)
        comp = r["Wq"][0] + r["Err"][0] * np.diag(U)
        for k in range(1, d):
            v = O.conditional_ls_values(w[0], Hd, r["Wq"][0, :k])
            np.testing.assert_allclose(comp[k], v[0], rtol=1e-9, atol=1e-12)
        s, z = r["scales"][0, 0], r["zeros"][0, 0]
        qbest, obest = O.bruteforce_best_codes(w[0], Hd, bits, s, z)
        dg = w[0] - r["Wq"][0]
        ogreedy = dg @ Hd @ dg
        dr = w[0] - O.rtn_quantize(w, bits)["Wq"][0]
        assert obest <= ogreedy * (1 + 1e-12) + 1e-18
        assert obest <= dr @ Hd @ dr * (1 + 1e-12) + 1e-18


def test_gptq_beats_rtn_statistic():
    """Expected statistic (the pages: GPTQ beats round-to-nearest at 3-4 bits because correlated
    inputs let other weights absorb the error): on the tiny correlated layer shape, the layer
    reconstruction error is at most RTN's in at least 95 of 100 seeded trials."""
    wins = 0
    for seed in range(100):
        rng = np.random.default_rng(seed)
        W = rng.standard_normal((64, 128)) * 0.02
        Z = rng.standard_normal((256, 128))
        A = rng.standard_normal((128, 128)) / np.sqrt(128)
        X = Z @ A
        res = O.gptq_layer(W, X, bits=4, group_size=0, block_size=32)
        e_rtn = O.reconstruction_error(W, O.rtn_quantize(W, 4)["Wq"], res["H"])
        wins += res["E"] <= e_rtn
    assert wins >= 95


@pytest.mark.parametrize("group_size", [0, 8, 32])
def test_blocking_and_scaling_do_not_change_codes(group_size):
    rng = np.random.default_rng(7 + group_size)
    d = 64
    X = _correlated_x(128, d, rng)
    H = O.hessian(X)
    W = rng.standard_normal((20, d)) * 0.02
    U = O.inverse_upper_cholesky(O.dampen(H, 0.01))
    ref = O.gptq_quantize(W, U, 3, group_size, block_size=0)
    for B in (1, 4, 32):
        if group_size and group_size % B and B % group_size:
            continue
        r = O.gptq_quantize(W, U, 3, group_size, block_size=B)
        np.testing.assert_array_equal(r["codes"], ref["codes"])
        np.testing.assert_allclose(r["Wq"], ref["Wq"], rtol=0, atol=1e-12)
    # H -> c H (the pages' H = 2XX^T versus X^T X / N): damping scales along, codes are unchanged
    Us = O.inverse_upper_cholesky(O.dampen(H * 1e-3 / len(X), 0.01))
    r = O.gptq_quantize(W, Us, 3, group_size, block_size=16 if group_size != 8 else 8)
    np.testing.assert_array_equal(r["codes"], ref["codes"])


def test_reconstruction_error_two_forms():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((50, 12))
    W = rng.standard_normal((5, 12))
    Wq = W + 0.01 * rng.standard_normal((5, 12))
    direct = np.sum(((W - Wq) @ X.T) ** 2)
    np.testing.assert_allclose(O.reconstruction_error(W, Wq, O.hessian(X)), direct, rtol=1e-12)


# ------------------------------------------------------------------------------------ A7 pack
def test_pack_hand_worked_examples(golden_dir):
    g = read_golden(os.path.join(golden_dir, "pack_examples.txt"))
    for row in g["rows"]:
        bits, n, period = int(row[0]), int(row[1]), int(row[2])
        words = np.array([int(h, 16) for h in row[3:]], dtype=np.uint64).astype(np.uint32)
        codes = (np.arange(n) % period)[None, :]
        packed = O.pack_codes(codes, bits)
        np.testing.assert_array_equal(packed.view(np.uint32)[0], words)
        np.testing.assert_array_equal(O.unpack_codes(packed, bits, n), codes)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 2 ** bits, size=(7, 96))
    p = O.pack_codes(codes, bits)
    assert p.shape == (7, 96 * bits // 32) and p.dtype == np.int32
    np.testing.assert_array_equal(O.unpack_codes(p, bits, 96), codes)


# ------------------------------------------------------------------------------------ act-order
def _act_golden(golden_dir):
    g = read_golden(os.path.join(golden_dir, "worked_example_act_order.txt"))
    return g, np.array(g["hd"], dtype=float).reshape(3, 3), np.array(g["w"], dtype=float)[None, :], int(g["bits"][0])


def _act_golden_holds(golden_dir, fn=None):
    g, Hd, w, bits = _act_golden(golden_dir)
    fn = fn or (lambda w, Hd, bits: O.gptq_quantize_act_order(w, Hd, bits, damp=0.0))
    r = fn(w, Hd, bits)
    return (np.array_equal(r["perm"], np.array(g["perm"], dtype=int))
            and np.array_equal(r["codes"][0], np.array(g["codes"], dtype=int)))


def test_act_order_worked_example(golden_dir):
    g, Hd, w, bits = _act_golden(golden_dir)
    r = O.gptq_quantize_act_order(w, Hd, bits, damp=0.0)  # Hd is used as the damped matrix directly
    np.testing.assert_array_equal(r["perm"], np.array(g["perm"], dtype=int))
    np.testing.assert_array_equal(r["codes"][0], np.array(g["codes"], dtype=int))
    U = r["U"]
    rin = O.gptq_quantize(w[:, r["perm"]], U, bits)
    comp = rin["Wq"][0] + rin["Err"][0] * np.diag(U)
    np.testing.assert_allclose(comp, np.array(g["compensated_in_order"], dtype=float), rtol=0, atol=1e-12)
    nat = O.gptq_quantize(w, O.inverse_upper_cholesky(Hd), bits)
    np.testing.assert_array_equal(nat["codes"][0], np.array(g["codes_natural"], dtype=int))
    assert _act_golden_holds(golden_dir)


@pytest.mark.parametrize("group_size", [0, 4])
def test_act_order_with_sorted_diagonal_is_the_plain_method(group_size):
    rng = np.random.default_rng(21)
    d = 16
    X = _correlated_x(64, d, rng)
    H = O.hessian(X)
    order = np.argsort(-np.diag(H), kind="stable")
    H = H[np.ix_(order, order)]                     # diag(H) now descending
    W = rng.standard_normal((10, d)) * 0.02
    a = O.gptq_quantize_act_order(W, H, 3, group_size)
    np.testing.assert_array_equal(a["perm"], np.arange(d))
    p = O.gptq_quantize(W, O.inverse_upper_cholesky(O.dampen(H, 0.01)), 3, group_size)
    np.testing.assert_array_equal(a["codes"], p["codes"])
    np.testing.assert_array_equal(a["scales"], p["scales"])


@pytest.mark.parametrize("group_size", [0, 8])
def test_act_order_with_diagonal_hessian_is_rtn_in_that_order(group_size):
    rng = np.random.default_rng(22)
    d = 32
    H = np.diag(rng.uniform(0.5, 5.0, d))
    W = rng.standard_normal((12, d)) * 0.02
    a = O.gptq_quantize_act_order(W, H, 4, group_size, block_size=8)
    perm = np.argsort(-np.diag(H))
    r = O.rtn_quantize(W[:, perm], 4, group_size)
    inv = np.argsort(perm)
    np.testing.assert_array_equal(a["codes"], r["codes"][:, inv])
    np.testing.assert_array_equal(a["scales"], r["scales"])
    np.testing.assert_array_equal(a["g_idx"], (inv // group_size) if group_size else np.zeros(d, dtype=int))


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("group_size", [0, 4])
def test_act_order_equals_obs_recursion_in_that_order(seed, group_size):
    """The explicit OBS recursion, taking the columns in act-order on the unpermuted inverse Hessian,
    gives the same codes as the Cholesky form on the permuted problem."""
    rng = np.random.default_rng(30 + seed)
    d = 16
    X = _correlated_x(64, d, rng) * rng.uniform(0.2, 3.0, d)   # distinct column scales
    H = O.hessian(X)
    W = rng.standard_normal((12, d)) * 0.02
    a = O.gptq_quantize_act_order(W, H, 3, group_size)
    o = O.obs_quantize(W, O.dampen(H, 0.01), 3, group_size, order=a["perm"])
    np.testing.assert_array_equal(a["codes"], o["codes"])
    np.testing.assert_allclose(a["scales"], o["scales"], rtol=1e-6)


# ------------------------------------------------------------------------------------ inference product
def test_dequant_matmul_closed_forms():
    """Codes all at the zero point give Y = 0; codes one level above it give Y = scale * sum(x) per
    group; a single code at level k gives scale * (k - zero) * x_j (hand-checkable)."""
    rng = np.random.default_rng(50)
    m, d, bits, gs = 3, 64, 3, 32
    scales = np.array([[0.5, 0.25], [1.0, 2.0], [0.125, 4.0]], dtype=np.float32)
    zeros = np.array([[3, 4], [0, 7], [5, 1]])
    x = rng.standard_normal((2, d))
    codes = np.repeat(zeros, gs, axis=1)
    Y = O.dequant_matmul(O.pack_codes(codes, bits), scales, zeros, bits, gs, d, x)
    np.testing.assert_array_equal(Y, 0.0)
    Y = O.dequant_matmul(O.pack_codes(np.minimum(codes + 1, 7), bits), scales, zeros, bits, gs, d, x)
    for r in range(m):
        want = sum(float(scales[r, k]) * (min(zeros[r, k] + 1, 7) - zeros[r, k]) * x[:, k * gs:(k + 1) * gs].sum(1)
                   for k in range(2))
        np.testing.assert_allclose(Y[:, r], want, rtol=1e-12, atol=1e-12)
    one = codes.copy()
    one[1, 40] = 2                               # row 1, group 1 (scale 2, zero 7): level 2 -> 2 * (2 - 7)
    Y1 = O.dequant_matmul(O.pack_codes(one, bits), scales, zeros, bits, gs, d, x)
    np.testing.assert_allclose(Y1[:, 1], 2.0 * (2 - 7) * x[:, 40], rtol=1e-12)


@pytest.mark.parametrize("group_size", [0, 32])
def test_dequant_matmul_is_the_layer_product_with_quantized_weights(group_size):
    rng = np.random.default_rng(51)
    d, m = 96, 20
    X = _correlated_x(200, d, rng)
    W = rng.standard_normal((m, d)) * 0.02
    res = O.gptq_layer(W, X, bits=4, group_size=group_size, block_size=32)
    x_in = rng.standard_normal((5, d))
    Y = O.dequant_matmul(res["packed"], res["scales"], res["zeros"], 4, group_size, d, x_in)
    np.testing.assert_allclose(Y, x_in @ res["Wq"].T, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------------------------ mutation check
def test_planted_mistakes_are_caught():
    """Plant plausible mistakes in what the column loop is given and check a pin fails for each."""
    rng = np.random.default_rng(11)
    d = 12
    X = _correlated_x(48, d, rng)
    Hd = O.dampen(O.hessian(X), 0.01)
    W = rng.standard_normal((16, d)) * 0.05
    U = O.inverse_upper_cholesky(Hd)
    obs = O.obs_quantize(W, Hd, 3)["codes"]
    assert np.array_equal(O.gptq_quantize(W, U, 3)["codes"], obs)
    Uo = U - np.diag(np.diag(U))
    mistakes = {
        "transposed U": U.T,
        "wrong sign of the update": np.diag(np.diag(U)) - Uo,
        "dropped division by U_ii": Uo + np.eye(d),
        "Cholesky of H instead of its inverse": np.linalg.cholesky(Hd).T,
        "no compensation": np.diag(np.diag(U)),
    }
    for name, Ubad in mistakes.items():
        caught = False
        try:
            caught = not np.array_equal(O.gptq_quantize(W, Ubad, 3)["codes"], obs)
        except Exception:
            caught = True
        assert caught, name


def test_planted_group_grid_from_original_w_is_caught(golden_dir, monkeypatch):
    """Plant the mistake of taking each group's grid from the original W (rather than from the
    compensated values at the group start) in the oracle, and check the hand-worked group pin fails.
    The OBS recursion shares the grid routine, so it cannot see this mistake; the golden file can."""
    import oracle.gptq_oracle as OM
    g, Hd, w, bits, gs = _group_golden(golden_dir)
    assert _check_group_golden(g, Hd, w, bits, gs, 2)
    original = OM.grid_params
    groups = [w[:, k:k + gs] for k in range(0, w.shape[1], gs)]
    calls = {"n": 0}

    def grid_from_original(xmin, xmax, b):
        k = calls["n"] % len(groups)
        calls["n"] += 1
        return original(groups[k].min(axis=1), groups[k].max(axis=1), b)

    monkeypatch.setattr(OM, "grid_params", grid_from_original)
    assert not _check_group_golden(g, Hd, w, bits, gs, 2), "group grid from the original W"


def test_planted_act_order_mistakes_are_caught(golden_dir):
    """Plausible mistakes in the act-order bookkeeping each fail the hand-worked act-order pin."""
    def not_unpermuted(w, Hd, bits):
        r = O.gptq_quantize_act_order(w, Hd, bits, damp=0.0)
        return {**r, "codes": r["codes_in_order"]}

    def ascending(w, Hd, bits):
        return O.gptq_quantize_act_order(w, Hd, bits, damp=0.0, perm=np.argsort(np.diag(Hd), kind="stable"))

    def h_not_permuted(w, Hd, bits):
        perm = O.act_order_permutation(Hd)
        r = O.gptq_quantize(w[:, perm], O.inverse_upper_cholesky(Hd), bits)
        inv = np.argsort(perm)
        return {"perm": perm, "codes": r["codes"][:, inv]}

    # the OBS recursion in act-order on a layer whose permutation is not its own inverse (the golden
    # example's [2, 1, 0] is)
    rng = np.random.default_rng(40)
    d = 16
    X = _correlated_x(64, d, rng) * rng.uniform(0.2, 3.0, d)
    H = O.hessian(X)
    W = rng.standard_normal((12, d)) * 0.02
    perm = O.act_order_permutation(H)
    assert not np.array_equal(perm[perm], np.arange(d))
    obs = O.obs_quantize(W, O.dampen(H, 0.01), 3, order=perm)["codes"]

    def obs_pin_holds(fn):
        return np.array_equal(fn(W, H, 3)["codes"], obs)

    def inverse_used_as_perm_obs(W, H, bits):
        r = O.gptq_quantize_act_order(W, H, bits)
        return {"codes": r["codes_in_order"][:, r["perm"]]}

    assert _act_golden_holds(golden_dir)
    assert obs_pin_holds(lambda W, H, b: O.gptq_quantize_act_order(W, H, b))
    for name, fn in {"codes left in quantization order": not_unpermuted, "ascending diag(H)": ascending,
                     "H not permuted": h_not_permuted}.items():
        assert not _act_golden_holds(golden_dir, fn), name
    assert not obs_pin_holds(inverse_used_as_perm_obs), "un-permuted with perm instead of its inverse"
