"""Pins for the float64 oracle: each checks it against something other than
itself (hand-worked fixtures, closed forms, brute force, invariants, library
routines on special cases), so that a dropped term, a wrong sign or index or a
transposed operand in the oracle fails at least one of them."""
import itertools
import json
import os

import numpy as np
import pytest
import scipy.linalg as sla

import oracle
from synthetic import CONFIGS, make_layer_host, random_layer_host

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _spd(n, seed, cond_boost=1.0):
    r = _rng(seed)
    A = r.standard_normal((n, 3 * n))
    return A @ A.T + cond_boost * np.eye(n)


# ----------------------------------------------------------------------------- Hessian

def test_hessian_brute_triple_loop():
    r = _rng(0)
    x = r.standard_normal((7, 5))
    H = oracle.hessian(x, chunk=3)
    for i in range(5):
        for j in range(5):
            s = 0.0
            for t in range(7):
                s += x[t, i] * x[t, j]
            assert H[i, j] == pytest.approx(2.0 * s, rel=1e-13, abs=1e-13)


def test_hessian_symmetric_psd_and_additive():
    r = _rng(1)
    x = r.standard_normal((300, 40))
    x[:, 3] *= 20
    H = oracle.hessian(x, chunk=64)
    assert np.array_equal(H, H.T) or np.abs(H - H.T).max() <= 1e-12 * np.abs(H).max()
    assert np.linalg.eigvalsh(H).min() >= -1e-12 * np.abs(H).max()
    H2 = oracle.hessian(x[150:], H0=oracle.hessian(x[:150]))
    assert np.abs(H2 - H).max() <= 1e-12 * np.abs(H).max()


# ----------------------------------------------------------------------------- QEP

def _small_qep_case(seed=3, m=24, n=16, N=200):
    r = _rng(seed)
    W = r.standard_normal((m, n)) * 0.1
    x = r.standard_normal((N, n))
    xh = x + 0.05 * r.standard_normal((N, n))
    return W, x, xh


def test_qep_alpha_zero_returns_w_exactly():
    W, x, xh = _small_qep_case()
    assert np.array_equal(oracle.qep_correct(W, x, xh, alpha=0.0, damp=0.01), W)


def test_qep_identical_inputs_return_w():
    W, x, _ = _small_qep_case()
    out = oracle.qep_correct(W, x, x, alpha=0.5, damp=0.01)
    assert np.abs(out - W).max() <= 1e-10 * np.abs(W).max()


def test_qep_linear_in_alpha():
    W, x, xh = _small_qep_case()
    d1 = oracle.qep_correct(W, x, xh, 1.0, 0.01) - W
    d07 = oracle.qep_correct(W, x, xh, 0.7, 0.01) - W
    assert np.abs(d07 - 0.7 * d1).max() <= 1e-12 * np.abs(d1).max()


def test_qep_normal_equation_identity():
    # At alpha = 1 the corrected weight satisfies the stationarity condition of
    # ||W X^T - W' Xh^T||^2 + lam ||W' - W||^2:  (W X^T - W' Xh^T) Xh = lam (W' - W).
    W, x, xh = _small_qep_case()
    damp = 0.05
    Wp = oracle.qep_correct(W, x, xh, 1.0, damp)
    lam = damp * np.mean(np.sum(xh * xh, axis=0))
    lhs = (W @ x.T - Wp @ xh.T) @ xh
    rhs = lam * (Wp - W)
    assert np.abs(lhs - rhs).max() <= 1e-10 * np.abs(rhs).max()


def test_qep_no_damping_is_least_squares():
    # lam -> 0 with more tokens than channels: W' minimises ||W X^T - W' Xh^T||,
    # which numpy's least-squares solver gives independently.
    W, x, xh = _small_qep_case(seed=5, N=400)
    Wp = oracle.qep_correct(W, x, xh, 1.0, 0.0)
    ls = np.linalg.lstsq(xh, x @ W.T, rcond=None)[0].T
    assert np.abs(Wp - ls).max() <= 1e-9 * np.abs(ls).max()


def test_qep_given_h_equals_recomputed():
    W, x, xh = _small_qep_case()
    H = oracle.hessian(xh)
    a = oracle.qep_correct(W, x, xh, 0.5, 0.01, H=H)
    b = oracle.qep_correct(W, x, xh, 0.5, 0.01)
    assert np.abs(a - b).max() <= 1e-12 * np.abs(W).max()


def test_qep_scale_invariance_power_of_two():
    W, x, xh = _small_qep_case()
    a = oracle.qep_correct(W, x, xh, 0.5, 0.01)
    b = oracle.qep_correct(W, 2.0 * x, 2.0 * xh, 0.5, 0.01)
    assert np.abs(a - b).max() <= 1e-13 * np.abs(W).max()


# ----------------------------------------------------------------------------- factor

def test_inv_chol_upper_properties_and_routes():
    Hd = _spd(40, 7)
    U = oracle.inv_chol_upper(Hd)
    assert np.allclose(np.tril(U, -1), 0.0)
    assert (np.diag(U) > 0).all()
    inv = np.linalg.inv(Hd)
    assert np.abs(U.T @ U - inv).max() <= 1e-10 * np.abs(inv).max()
    Ub = oracle.inv_chol_upper_reversed(Hd)
    assert np.abs(U - Ub).max() <= 1e-10 * np.abs(U).max()


def test_inv_chol_upper_2x2_closed_form():
    a, b, c = 3.0, 1.2, 2.0
    U = oracle.inv_chol_upper(np.array([[a, b], [b, c]]))
    # Hd = R R^T with R upper: r22 = sqrt(c), r12 = b/sqrt(c), r11 = sqrt(a - b^2/c); U = R^-1.
    r22, r12 = np.sqrt(c), b / np.sqrt(c)
    r11 = np.sqrt(a - b * b / c)
    expect = np.array([[1 / r11, -r12 / (r11 * r22)], [0.0, 1 / r22]])
    assert np.abs(U - expect).max() <= 1e-14


# ----------------------------------------------------------------------------- grid / rounding

def test_grid_and_codes_hand_worked():
    with open(os.path.join(GOLDEN, "grid_rounding.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        maxq = (1 << c["wbits"]) - 1
        w = np.array([c["w"]])
        s, z = oracle.group_params(w, maxq)
        assert s[0] == pytest.approx(c["scale"], rel=1e-15)
        assert z[0] == c["zero"]
        q, dq = oracle.quantize_values(w[0], s[0], z[0], maxq)
        assert q.astype(int).tolist() == c["codes"], c["why"]
        assert np.allclose(dq, s[0] * (q - z[0]))


def test_pack_hand_worked_patterns_and_roundtrip():
    with open(os.path.join(GOLDEN, "pack_patterns.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        codes = np.array([c["codes"]])
        words = oracle.pack_codes(codes, c["wbits"])
        assert words[0].tolist() == c["words"], c["why"]
        back = oracle.unpack_codes(words, c["wbits"], codes.shape[1])
        assert np.array_equal(back, codes)
    r = _rng(11)
    for b in (2, 3, 4):
        codes = r.integers(0, 1 << b, size=(5, 96))
        assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(codes, b), b, 96), codes)


# ----------------------------------------------------------------------------- GPTQ

def _rtn(W, wbits, G):
    # Round-to-nearest on the group grid without any error feedback, computed
    # group by group from the unmodified weights.
    maxq = (1 << wbits) - 1
    m, n = W.shape
    codes = np.zeros((m, n), dtype=np.int64)
    for g in range(n // G):
        s, z = oracle.group_params(W[:, g * G:(g + 1) * G], maxq)
        q, _ = oracle.quantize_values(W[:, g * G:(g + 1) * G], s[:, None], z[:, None], maxq)
        codes[:, g * G:(g + 1) * G] = q
    return codes


@pytest.mark.parametrize("act_order", [False, True])
@pytest.mark.parametrize("wbits,G", [(4, 32), (3, 64), (2, 16)])
def test_gptq_identity_or_diagonal_h_is_rtn(act_order, wbits, G):
    r = _rng(21)
    W = r.standard_normal((12, 64)) * 0.02
    for H in (np.eye(64), np.diag(r.uniform(0.5, 4.0, 64))):
        res = oracle.gptq_quantize(W, H, wbits, G, damp=0.01, act_order=act_order)
        assert np.array_equal(res["codes"], _rtn(W, wbits, G))


def test_gptq_two_column_closed_form():
    # Quantising column 1 with error d1 = w1 - q1 moves column 2 to the
    # continuous optimum w2 + d1 * H12 / H22 before it is rounded.
    r = _rng(5)
    for trial in range(50):
        H = _spd(2, 100 + trial, cond_boost=0.1)
        W = r.standard_normal((1, 2))
        res = oracle.gptq_quantize(W, H, 4, -1, damp=0.0, act_order=False, unblocked=True)
        s, z = res["scales"][0, 0], res["zeros"][0, 0]
        d1 = W[0, 0] - res["deq"][0, 0]
        w2 = W[0, 1] + d1 * H[0, 1] / H[1, 1]
        q2, _ = oracle.quantize_values(np.array([w2]), s, z, 15)
        assert res["codes"][0, 1] == q2[0]


def _reduced_objective(Hd, w, deq_prefix, j):
    # min over continuous later columns of e^T Hd e with e_<=j fixed = e_<=j^T S e_<=j,
    # S the Schur complement of the trailing block.
    k = j + 1
    e = w[:k] - deq_prefix
    A = Hd[:k, :k]
    if k < Hd.shape[0]:
        B = Hd[:k, k:]
        C = Hd[k:, k:]
        A = A - B @ np.linalg.solve(C, B.T)
    return float(e @ A @ e)


@pytest.mark.parametrize("act_order", [False, True])
def test_gptq_each_code_is_greedy_optimal_brute_force(act_order):
    # At every column the GPTQ code minimises, over every code of that column's
    # grid, the loss with earlier columns fixed at their codes and later columns
    # left at their continuous optimum.  Checked by enumerating all codes.
    r = _rng(8)
    n, wbits, G = 8, 2, 4
    maxq = 3
    for trial in range(20):
        H = _spd(n, 300 + trial, cond_boost=0.2)
        W = r.standard_normal((3, n))
        res = oracle.gptq_quantize(W, H, wbits, G, damp=0.01, act_order=act_order,
                                   unblocked=True)
        perm = res["perm"]
        Hd = res["Hd"]
        for row in range(3):
            w = W[row, perm]
            deq = res["deq"][row, perm]
            codes = res["codes"][row, perm]
            for j in range(n):
                g = perm[j] // G
                s, z = res["scales"][row, g], res["zeros"][row, g]
                vals = [_reduced_objective(Hd, w, np.append(deq[:j], s * (c - z)), j)
                        for c in range(maxq + 1)]
                best = min(vals)
                assert vals[codes[j]] <= best + 1e-12 * max(1.0, abs(best))


def test_gptq_4x4_2bit_brute_force_bound():
    # Enumerating all 4^4 codes of a row on GPTQ's grid can only do as well or
    # better than GPTQ's greedy choice (a consistency check of the objective and
    # the grid; the greedy-optimality test above pins the update itself).
    r = _rng(12)
    for trial in range(30):
        H = _spd(4, 500 + trial, cond_boost=0.05)
        W = r.standard_normal((2, 4))
        res = oracle.gptq_quantize(W, H, 2, 4, damp=0.0, act_order=False, unblocked=True)
        for row in range(2):
            s, z = res["scales"][row, 0], res["zeros"][row, 0]
            best = min(oracle.gptq_objective(W[row:row + 1],
                                             (s * (np.array(c) - z))[None, :], H)
                       for c in itertools.product(range(4), repeat=4))
            got = oracle.gptq_objective(W[row:row + 1], res["deq"][row:row + 1], H)
            assert best <= got + 1e-12


@pytest.mark.parametrize("act_order,G", [(False, 64), (False, 128), (True, 64), (False, 512)])
def test_gptq_blocked_equals_unblocked(act_order, G):
    L = random_layer_host(48, 512, 1024, seed=9)
    H = oracle.hessian(L["Xhat"])
    a = oracle.gptq_quantize(L["W"], H, 3, G, 0.01, act_order, block=128)
    b = oracle.gptq_quantize(L["W"], H, 3, G, 0.01, act_order, unblocked=True)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.abs(a["scales"] - b["scales"]).max() <= 1e-12 * np.abs(b["scales"]).max()
    assert np.abs(a["deq"] - b["deq"]).max() <= 1e-12 * np.abs(b["deq"]).max()


def test_gptq_group_not_tiling_the_block():
    # a 384-wide group starts inside a 256-column block: the blocked forms take
    # 128-column blocks, agree with the unblocked definition, and refuse 256
    L = random_layer_host(24, 768, 1536, seed=19)
    H = oracle.hessian(L["Xhat"])
    a = oracle.gptq_quantize(L["W"], H, 4, 384, 0.01, False, block=128)
    b = oracle.gptq_quantize(L["W"], H, 4, 384, 0.01, False, unblocked=True)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.abs(a["scales"] - b["scales"]).max() <= 1e-12 * np.abs(b["scales"]).max()
    st = oracle.teacher_forced_check(L["W"], H, 4, 384, 0.01, False, a["codes"], a["scales"], a["zeros"],
                                     block=128)
    assert st["n_mismatch"] == 0 and st["n_bad"] == 0 and st["scale_max_rel"] <= 1e-12
    with pytest.raises(ValueError):
        oracle.gptq_quantize(L["W"], H, 4, 384, 0.01, False, block=256)
    with pytest.raises(ValueError):
        oracle.teacher_forced_check(L["W"], H, 4, 384, 0.01, False, a["codes"], a["scales"], a["zeros"],
                                    block=256)


def test_gptq_hessian_scale_invariance():
    L = random_layer_host(16, 256, 512, seed=10)
    H = oracle.hessian(L["Xhat"])
    a = oracle.gptq_quantize(L["W"], H, 4, 128, 0.01, True)
    b = oracle.gptq_quantize(L["W"], 4.0 * H, 4, 128, 0.01, True)
    assert np.array_equal(a["codes"], b["codes"])


def test_gptq_single_column_is_rtn():
    r = _rng(13)
    W = r.standard_normal((10, 1))
    res = oracle.gptq_quantize(W, np.array([[2.5]]), 3, 1, 0.01, False, unblocked=True)
    assert np.array_equal(res["codes"], _rtn(W, 3, 1))


def test_gptq_dead_columns():
    L = random_layer_host(8, 64, 256, seed=14)
    x = L["Xhat"].copy()
    x[:, [5, 40]] = 0.0
    H = oracle.hessian(x)
    res = oracle.gptq_quantize(L["W"], H, 4, 32, 0.01, True)
    # a dead column's weight is zeroed before quantisation: it dequantises to
    # the grid point nearest zero
    for j in (5, 40):
        g = j // 32
        s, z = res["scales"][:, g], res["zeros"][:, g]
        assert np.all(np.abs(res["deq"][:, j]) <= s / 2 + 1e-12)


def test_dynamic_group_first_column_reconstructs_within_half_step():
    L = random_layer_host(32, 256, 512, seed=15)
    H = oracle.hessian(L["Xhat"])
    res = oracle.gptq_quantize(L["W"], H, 4, 64, 0.01, False)
    # the first column of the first group has received no feedback yet
    err = np.abs(L["W"][:, 0] - res["deq"][:, 0])
    assert np.all(err <= res["scales"][:, 0] / 2 * (1 + 1e-12))


def test_gptq_lowers_layer_error_vs_rtn():
    L = random_layer_host(64, 256, 2048, seed=16)
    H = oracle.hessian(L["Xhat"])
    res = oracle.gptq_quantize(L["W"], H, 3, 64, 0.01, False)
    rtn = _rtn(L["W"], 3, 64)
    s = np.repeat(res["scales"], 64, axis=1)
    z = np.repeat(res["zeros"], 64, axis=1)
    e_gptq = oracle.gptq_objective(L["W"], res["deq"], H)
    # RTN on the same (dynamic) grids is not well defined after feedback; use its own grid
    maxq = 7
    sr = np.zeros_like(s)
    zr = np.zeros_like(z)
    for g in range(256 // 64):
        a, b = oracle.group_params(L["W"][:, g * 64:(g + 1) * 64], maxq)
        sr[:, g * 64:(g + 1) * 64] = a[:, None]
        zr[:, g * 64:(g + 1) * 64] = b[:, None]
    e_rtn = oracle.gptq_objective(L["W"], sr * (rtn - zr), H)
    assert e_gptq < e_rtn


# ----------------------------------------------------------------------------- teacher forcing

def test_teacher_forcing_accepts_own_output_and_flags_planted_error():
    L = random_layer_host(24, 256, 1024, seed=17)
    H = oracle.hessian(L["Xhat"])
    for act_order in (False, True):
        res = oracle.gptq_quantize(L["W"], H, 4, 128, 0.01, act_order)
        st = oracle.teacher_forced_check(L["W"], H, 4, 128, 0.01, act_order,
                                         res["codes"], res["scales"], res["zeros"])
        assert st["n_mismatch"] == 0 and st["n_bad"] == 0
        assert st["scale_max_rel"] <= 1e-12 and st["zero_bad"] == 0
        # plant a mistake in a copy of the oracle's own codes: move one code by
        # two steps, which no rounding-boundary ambiguity can explain
        bad = res["codes"].copy()
        bad[3, 77] = (bad[3, 77] + 2) % 16
        st = oracle.teacher_forced_check(L["W"], H, 4, 128, 0.01, act_order,
                                         bad, res["scales"], res["zeros"])
        assert st["n_bad"] >= 1


def test_workload_recipes_shapes():
    L = make_layer_host(CONFIGS["layer_512"])
    assert L["W"].shape == (512, 512) and L["X"].shape == (2048, 512)
    assert len(L["outliers"]) == 4
    assert CONFIGS["q_proj_4096"].outlier_count() == 40
    assert CONFIGS["down_proj_11008"].outlier_count() == 55
    assert CONFIGS["down_proj_28672"].outlier_count() == 286


def test_qep_precomputed_terms_over_chunks():
    # H and d are sums over tokens: accumulating them over token chunks and
    # passing them in must give the same W' as the one-shot computation.
    rng = np.random.default_rng(71)
    x = rng.standard_normal((300, 16))
    xh = x + 0.1 * rng.standard_normal(x.shape)
    W = rng.standard_normal((5, 16))
    H = sum(oracle.hessian(xh[t:t + 64]) for t in range(0, 300, 64))
    d = sum(oracle.qep_cross(x[t:t + 64], xh[t:t + 64]) for t in range(0, 300, 64))
    a = oracle.qep_correct(W, x, xh, 0.5, 0.01)
    b = oracle.qep_correct(W, None, None, 0.5, 0.01, H=H, d=d)
    assert np.allclose(a, b, rtol=0, atol=1e-12)


def test_gptq_given_factor_equals_recomputed():
    # Passing the factor of the same preparation (here by the reversed route,
    # which is pinned equal to route A) must not change any output.
    rng = np.random.default_rng(72)
    X = rng.standard_normal((200, 64))
    H = oracle.hessian(X)
    W = rng.standard_normal((6, 64))
    a = oracle.gptq_quantize(W, H, 3, 16, 0.01, True)
    prep = oracle.gptq_prepare(W, H, 0.01, True)
    U = oracle.inv_chol_upper_reversed(prep["Hd"])
    b = oracle.gptq_quantize(W, H, 3, 16, 0.01, True, U=U)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.allclose(a["scales"], b["scales"], rtol=1e-12, atol=0)
    st = oracle.teacher_forced_check(W, H, 3, 16, 0.01, True, a["codes"], a["scales"], a["zeros"], U=U)
    assert st["n_mismatch"] == 0 and st["scale_max_rel"] <= 1e-12


def test_dequantize_inverts_pack():
    rng = np.random.default_rng(73)
    for wbits in (2, 3, 4):
        codes = rng.integers(0, 1 << wbits, size=(5, 64))
        packed = oracle.pack_codes(codes, wbits)
        scales = rng.uniform(0.1, 1.0, size=(5, 2))
        zeros = rng.integers(0, 1 << wbits, size=(5, 2)).astype(np.float64)
        deq = oracle.dequantize(packed, scales, zeros, wbits, 32, 64)
        want = np.repeat(scales, 32, axis=1) * (codes - np.repeat(zeros, 32, axis=1))
        assert np.array_equal(deq, want)


def test_chain_first_layer_is_plain_gptq_and_later_inputs_propagate():
    # Xh_0 = X_0: the first layer's QEP correction vanishes (W' = W to 1e-10);
    # the second layer's inputs are the two streams' forward products.
    rng = np.random.default_rng(74)
    x0 = rng.standard_normal((512, 32))
    Ws = [0.2 * rng.standard_normal((32, 32)), 0.2 * rng.standard_normal((16, 32))]
    layers, (x2, xh2) = oracle.quantize_chain(Ws, x0, 0.5, 0.01, 4, 16, False)
    assert np.abs(layers[0]["W_prime"] - Ws[0]).max() <= 1e-10
    ref = oracle.gptq_quantize(Ws[0], oracle.hessian(oracle._bf16(x0)), 4, 16, 0.01, False)
    assert np.array_equal(layers[0]["codes"], ref["codes"])
    x1 = layers[1]["X"]
    want = oracle._bf16(oracle._act(oracle._bf16(oracle._bf16(x0) @ oracle._bf16(Ws[0]).T), "silu"))
    assert np.array_equal(x1, want)
    assert x2.shape == (512, 16) and xh2.shape == (512, 16)
    assert not np.array_equal(layers[1]["X"], layers[1]["Xhat"])


def test_chain_qep_reduces_propagated_error():
    # QEP's purpose: with quantisation error arriving from earlier layers,
    # correcting for it lowers the chain's final output error ||X_L - Xh_L||.
    rng = np.random.default_rng(75)
    x0 = rng.standard_normal((2048, 64))
    x0[:, :2] *= 8.0
    Ws = [rng.standard_normal((64, 64)) / 8.0 for _ in range(4)]
    errs = {}
    for alpha in (0.0, 0.5, 1.0):
        _, (x, xh) = oracle.quantize_chain(Ws, x0, alpha, 0.01, 3, 16, False)
        errs[alpha] = np.linalg.norm(x - xh) / np.linalg.norm(x)
    assert errs[0.5] < errs[0.0] and errs[1.0] < errs[0.0], errs


def test_hadamard_is_sylvester_and_orthogonal():
    import scipy.linalg as sla
    for b in (1, 2, 8, 64):
        H = oracle.hadamard(b)
        assert np.array_equal(H, sla.hadamard(b))
        assert np.array_equal(H @ H.T, b * np.eye(b))


def test_hadamard_rotation_preserves_layer_output_and_is_an_involution():
    rng = np.random.default_rng(76)
    W = rng.standard_normal((5, 96))
    X = rng.standard_normal((40, 96))
    for b in (2, 32):
        Wr, Xr = oracle.hadamard_rotate(W, b), oracle.hadamard_rotate(X, b)
        assert np.allclose(Wr @ Xr.T, W @ X.T, rtol=0, atol=1e-12)
        assert np.allclose(oracle.hadamard_rotate(Xr, b), X, rtol=0, atol=1e-12)
        # blocks act independently: the first block of a row only mixes its own b features
        assert np.allclose(Xr[:, :b], X[:, :b] @ (oracle.hadamard(b) / np.sqrt(b)), rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- dequantising GEMV

def test_dequant_gemv_by_explicit_sums():
    # y[b][i] = sum_j x[b][j] * scale[i][j // G] * (q[i][j] - zero[i][j // G]), summed by loops
    rng = np.random.default_rng(77)
    for wbits, G, m, n in [(4, 8, 3, 32), (3, 32, 2, 64), (2, 16, 4, 64)]:
        codes = rng.integers(0, 2 ** wbits, size=(m, n))
        scales = rng.uniform(0.5, 2.0, size=(m, n // G))
        zeros = rng.integers(0, 2 ** wbits, size=(m, n // G)).astype(np.float64)
        x = rng.standard_normal((3, n))
        packed = oracle.pack_codes(codes, wbits)
        y = oracle.dequant_gemv(packed, scales, zeros, wbits, G, n, x)
        ref = np.zeros((3, m))
        for b in range(3):
            for i in range(m):
                for j in range(n):
                    ref[b, i] += x[b, j] * scales[i, j // G] * (codes[i, j] - zeros[i, j // G])
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def _bf16_bits(y):
    b = np.asarray(y, dtype=np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "result is not a bf16 number"
    return b >> 16


def test_bf16_rounding_hand_worked_bit_patterns():
    # tests/golden/bf16_rounding.json: ties to even, a tie that a detour
    # through float32 would break the wrong way, carries into the exponent,
    # the largest finite value and overflow, subnormals and signed zeros
    with open(os.path.join(GOLDEN, "bf16_rounding.json")) as f:
        cases = json.load(f)["cases"]
    xs = np.array([float(c["x"]) if c["x"].endswith("inf") else float.fromhex(c["x"]) for c in cases])
    want = np.array([int(c["bits"], 16) for c in cases], dtype=np.uint32)
    got = _bf16_bits(oracle._bf16(xs))
    bad = [(c["x"], hex(int(g)), c["bits"]) for c, g, w in zip(cases, got, want) if g != w]
    assert not bad, bad
    assert np.isnan(oracle._bf16(np.array([np.nan]))[0])


def test_bf16_rounding_fixture_catches_planted_mistakes():
    # Each plausible slip in a rounding routine fails at least one fixture case.
    with open(os.path.join(GOLDEN, "bf16_rounding.json")) as f:
        cases = json.load(f)["cases"]
    fin = [c for c in cases if not c["x"].endswith("inf")]
    xs = np.array([float.fromhex(c["x"]) for c in fin])
    want = np.array([int(c["bits"], 16) for c in fin], dtype=np.uint32)

    def via_float32(a):      # two roundings: float64 -> float32 -> bf16
        u = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
        return ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32).view(np.float32)

    def ties_away(a):        # ties away from zero instead of to even
        u = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
        return ((u + 0x8000) & 0xFFFF0000).astype(np.uint32).view(np.float32)

    def truncate(a):         # chopping the low bits
        u = np.asarray(a, np.float32).view(np.uint32)
        return (u & np.uint32(0xFFFF0000)).view(np.float32)

    for wrong in (via_float32, ties_away, truncate):
        got = np.asarray(wrong(xs), np.float32).view(np.uint32) >> 16
        assert np.any(got != want), wrong.__name__


def test_layer_errors_hand_worked():
    # tests/golden/layer_errors_tiny.json: a 2 x 3 layer on 4 tokens with every
    # product written out by hand
    with open(os.path.join(GOLDEN, "layer_errors_tiny.json")) as f:
        g = json.load(f)
    W, Q, Wp = (np.array(g[k], dtype=np.float64) for k in ("W", "Q", "W_prime"))
    X, Xh = np.array(g["X"], dtype=np.float64), np.array(g["Xhat"], dtype=np.float64)
    e = oracle.layer_errors(W, Q, X, Xh, W_prime=Wp)
    assert abs(e["e_lit"] ** 2 - g["e_lit_sq"]) <= 1e-12 * g["e_lit_sq"]
    assert abs(e["e_qep"] ** 2 - g["e_qep_sq"]) <= 1e-12 * g["e_qep_sq"]
    assert abs(e["e_gptq"] ** 2 - g["e_gptq_sq"]) <= 1e-12 * g["e_gptq_sq"]
    # the fixture tells the inputs apart: exchanging X and Xhat gives the
    # hand-worked 'swapped' values, none equal to the right ones
    s = oracle.layer_errors(W, Q, Xh, X, W_prime=Wp)
    sw = g["swapped"]
    assert abs(s["e_lit"] ** 2 - sw["e_lit_sq_with_Xhat"]) <= 1e-12 * 64
    assert abs(s["e_qep"] ** 2 - sw["e_qep_sq_with_X_and_Xhat_exchanged"]) <= 1e-12 * 64
    assert abs(s["e_gptq"] ** 2 - sw["e_gptq_sq_with_X"]) <= 1e-12 * 64
    assert len({g["e_lit_sq"], sw["e_lit_sq_with_Xhat"]}) == 2
    # a transposed operand cannot be evaluated on these shapes
    with pytest.raises(ValueError):
        oracle.layer_errors(W.T, Q.T, X, Xh)
