"""Pins of the FP64 oracle against what the pages and the mathematics fix.

Each test names the statement it checks.  Pages: pith.science review of
"BaKron: Efficient Quantization with Kronecker-Factored Hessians" (sections
"What carries the argument" = Proposition 3.1, "Core claim" = Theorem 3.2,
"If this is right" = Corollary 3.4's bound, "Load-bearing premise" = GPTQ's
one-sided Hessian) and the arXiv abstract.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import workloads

SHAPES = [(2, 3), (3, 2), (4, 4), (5, 7), (8, 5), (9, 16), (16, 24), (24, 16), (13, 13)]


def _prep(oracle, W, A, B, bits=4):
    qmin, qmax = oracle.grid(bits)
    s = oracle.scales(W, qmax)
    LA, LB = oracle.factor(A), oracle.factor(B)
    return qmin, qmax, s, LA, LB, oracle.normalize(LA), oracle.normalize(LB)


# ---------------------------------------------------------------- Theorem 3.2
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_theorem_3_2_all_variants_agree(oracle_mod, shape, seed):
    """Theorem 3.2: BaKron-naive, -antidiagonal, -recursive and BaKron give the
    same codes.  Checked in FP64 on inputs with no near-tie (min distance of
    any Wt to a decision midpoint reported and required > 1e-9)."""
    o = oracle_mod
    m, n = shape
    W, A, B = workloads.random_problem(m, n, seed=seed + 100 * m + n)
    qmin, qmax, s, LA, LB, LtA, LtB = _prep(o, W, A, B)
    ref, Wt = o.solve(W, LtA, LtB, s, qmin, qmax, mode="pull")
    assert o.midpoint_distance(Wt, s, qmin, qmax).min() > 1e-9
    naive, Wt_naive = o.naive(W, A, B, s, qmin, qmax)
    assert np.array_equal(naive, ref)
    np.testing.assert_allclose(Wt_naive, Wt, rtol=0, atol=1e-12)
    assert np.array_equal(o.solve(W, LtA, LtB, s, qmin, qmax, mode="push")[0], ref)
    for leaf in (1, 2, 3, 16):
        assert np.array_equal(o.solve(W, LtA, LtB, s, qmin, qmax, mode="recursive", T=1, leaf=leaf)[0], ref)
    for T in (2, 4, 8):
        assert np.array_equal(o.solve(W, LtA, LtB, s, qmin, qmax, mode="recursive", T=T, leaf=1)[0], ref)
    assert np.array_equal(o.solve(W, LtA, LtB, s, qmin, qmax, mode="rowcol")[0], ref)


def test_theorem_3_2_any_linear_extension(oracle_mod):
    """Order independence: the pull recurrences visited in a random linear
    extension of the product order (random topological order of the grid)
    give the anti-diagonal result."""
    o = oracle_mod
    m, n = 11, 14
    W, A, B = workloads.random_problem(m, n, seed=5)
    qmin, qmax, s, LA, LB, LtA, LtB = _prep(o, W, A, B)
    ref, _ = o.solve(W, LtA, LtB, s, qmin, qmax)
    g = np.random.default_rng(3)
    for _ in range(5):
        # random topological order: repeatedly pick a random "ready" entry
        done = np.zeros((m, n), bool)
        frontier = {(0, 0)}
        order = []
        while frontier:
            i, j = sorted(frontier)[g.integers(len(frontier))]
            frontier.remove((i, j))
            order.append((i, j))
            done[i, j] = True
            for (a, b) in ((i + 1, j), (i, j + 1)):
                if a < m and b < n and (a == 0 or done[a - 1, b]) and (b == 0 or done[a, b - 1]):
                    frontier.add((a, b))
        assert len(order) == m * n
        codes, _ = o.solve(W, LtA, LtB, s, qmin, qmax, mode="order", order=np.array(order))
        assert np.array_equal(codes, ref)


def test_theorem_3_2_tiny_workload_naive(oracle_mod):
    """Theorem 3.2 on the 64x128 workload, including the literal mn x mn GPTQ."""
    o = oracle_mod
    W, A, B = workloads.generate("tiny")
    qmin, qmax, s, LA, LB, LtA, LtB = _prep(o, W, A, B)
    ref, Wt = o.solve(W, LtA, LtB, s, qmin, qmax)
    print("tiny: min midpoint distance", o.midpoint_distance(Wt, s, qmin, qmax).min())
    assert np.array_equal(o.naive(W, A, B, s, qmin, qmax)[0], ref)
    for T, leaf in ((1, 1), (1, 5), (16, 1), (32, 1), (64, 1)):
        assert np.array_equal(o.solve(W, LtA, LtB, s, qmin, qmax, mode="recursive", T=T, leaf=leaf)[0], ref)
    assert np.array_equal(o.solve(W, LtA, LtB, s, qmin, qmax, mode="rowcol")[0], ref)


# ------------------------------------------------ Proposition 3.1, worked 2x2
def test_prop_3_1_hand_worked_2x2(oracle_mod):
    """Closed form of a 2x2 solve derived by hand from Proposition 3.1.

    A = [[2,1],[1,2]] gives LtA[1,0] = -A01/A11 = -1/2; B = [[4,2],[2,3]] gives
    LtB[1,0] = -B01/B11 = -2/3.  With D = residuals:
      Wt00 = W00
      Wt01 = W01 - LtA[1,0] D00            = W01 + D00/2
      Wt10 = W10 - LtB[1,0] D00            = W10 + 2 D00/3
      Wt11 = W11 - (LtB10 LtA10 D00 + LtB10 D01 + LtA10 D10)
           = W11 - D00/3 + 2 D01/3 + D10/2
    (D01 sits in row 0, so it reaches row 1 through LtB[1,0]; D10 sits in
    column 0, so it reaches column 1 through LtA[1,0].)
    Exchanging A and B (a transposed operand) changes the coefficients, so
    this pins which factor acts on which side."""
    o = oracle_mod
    A = np.array([[2.0, 1.0], [1.0, 2.0]])
    B = np.array([[4.0, 2.0], [2.0, 3.0]])
    W = np.array([[0.30, 0.41], [-0.22, 0.17]])
    s = np.array([0.125, 0.0625], np.float32)  # exact binary steps
    qmin, qmax = -7, 7
    LtA, LtB = o.normalize(o.factor(A)), o.normalize(o.factor(B))
    assert abs(LtA[1, 0] + 0.5) < 1e-15 and abs(LtB[1, 0] + 2.0 / 3.0) < 1e-15

    F = Fraction
    Wf = [[F(str(x)) for x in row] for row in W]
    sf = [F(float(x)) for x in s]

    def rnd(x, i):
        q = x / sf[i]
        # round half to even, exact
        fl = q.numerator // q.denominator
        r = q - fl
        c = fl + 1 if r > F(1, 2) else fl if r < F(1, 2) else (fl if fl % 2 == 0 else fl + 1)
        return max(qmin, min(qmax, c))

    c00 = rnd(Wf[0][0], 0); d00 = Wf[0][0] - sf[0] * c00
    wt01 = Wf[0][1] + d00 / 2
    c01 = rnd(wt01, 0); d01 = wt01 - sf[0] * c01
    wt10 = Wf[1][0] + F(2, 3) * d00
    c10 = rnd(wt10, 1); d10 = wt10 - sf[1] * c10
    wt11 = Wf[1][1] - d00 / 3 + F(2, 3) * d01 + d10 / 2
    c11 = rnd(wt11, 1)
    expect = np.array([[c00, c01], [c10, c11]])
    expect_wt = np.array([[float(Wf[0][0]), float(wt01)], [float(wt10), float(wt11)]])

    codes, Wt = o.solve(W, LtA, LtB, s, qmin, qmax)
    np.testing.assert_allclose(Wt, expect_wt, rtol=0, atol=1e-15)
    assert np.array_equal(codes, expect)
    # the same example stored as a fixture (tests/golden/prop31_2x2.txt)
    g = {}
    for line in open(os.path.join(os.path.dirname(__file__), "golden", "prop31_2x2.txt")):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            g[k] = v
    assert [float(x) for x in g["W"]] == W.ravel().tolist() and [float(x) for x in g["s"]] == s.tolist()
    assert [F(x) for x in g["Wt"]] == [Wf[0][0], wt01, wt10, wt11]  # exact
    assert [int(x) for x in g["codes"]] == codes.ravel().tolist()
    np.testing.assert_allclose(Wt.ravel(), [float(F(x)) for x in g["Wt"]], rtol=0, atol=1e-15)
    assert F(g["LtA10"][0]) == F(-1, 2) and F(g["LtB10"][0]) == F(-2, 3)
    assert np.array_equal(o.naive(W, A, B, s, qmin, qmax)[0], expect)
    # the swapped-roles solve gives different pre-rounding values here
    _, Wt_sw = o.solve(W, LtB, LtA, s, qmin, qmax)
    assert np.abs(Wt_sw - expect_wt).max() > 1e-3


# ------------------------------------------------------- special cases (I5/I6)
@pytest.mark.parametrize("seed", [0, 1])
def test_B_identity_reduces_to_gptq(oracle_mod, seed):
    """B = I: the two-sided solve is one-sided GPTQ with Hessian A on every row
    (GPTQ's Hessian is E[xx^T] (x) I)."""
    o = oracle_mod
    m, n = 12, 20
    W, A, _ = workloads.random_problem(m, n, seed=seed)
    qmin, qmax = o.grid(4)
    s = o.scales(W, qmax)
    LtA = o.normalize(o.factor(A))
    codes, _ = o.solve(W, LtA, np.eye(m), s, qmin, qmax)
    assert np.array_equal(codes, o.gptq(W, A, s, qmin, qmax))


def test_tiny_B_identity_workload_gptq(oracle_mod):
    o = oracle_mod
    W, A, B = workloads.generate("tiny_bI")
    assert np.array_equal(B, np.eye(B.shape[0], dtype=np.float32))
    qmin, qmax = o.grid(4)
    s = o.scales(W, qmax)
    LtA, LtB = o.normalize(o.factor(A)), o.normalize(o.factor(B))
    codes, _ = o.solve(W, LtA, LtB, s, qmin, qmax)
    assert np.array_equal(codes, o.gptq(W, A, s, qmin, qmax))


def test_A_identity_is_gptq_on_columns(oracle_mod):
    """A = I: every column is quantised by GPTQ over the rows with Hessian B
    (the transposed problem), with the per-row steps kept."""
    o = oracle_mod
    m, n = 15, 9
    W, _, B = workloads.random_problem(m, n, seed=4)
    qmin, qmax = o.grid(4)
    s = o.scales(W, qmax)
    LtB = o.normalize(o.factor(B))
    codes, _ = o.solve(W, np.eye(n), LtB, s, qmin, qmax)
    # GPTQ over rows of W^T, but each entry keeps its own row step s_i: run it
    # on W / s (unit step) with the unit-step residual rescaled accordingly.
    Ws = W.astype(np.float64) / s.astype(np.float64)[:, None]
    Binv = np.linalg.inv(B.astype(np.float64))
    Lb = np.linalg.cholesky(0.5 * (Binv + Binv.T))
    # column recurrence: wt_i = w_i - sum_{i'<i} LtB[i,i'] d_i' with d in weight units
    exp = np.zeros((m, n), np.int32)
    for j in range(n):
        d = np.zeros(m)
        for i in range(m):
            wt = W[i, j] - np.dot(LtB[i, :i], d[:i])
            c = o.decide(np.array([[wt]]), s[i:i + 1], qmin, qmax)[0, 0]
            exp[i, j] = c
            d[i] = wt - float(s[i]) * c
    assert np.array_equal(codes, exp)
    del Ws, Lb


def test_diagonal_factors_give_round_to_nearest(oracle_mod):
    """Diagonal A and B: normalised factors are I, the result is RTN."""
    o = oracle_mod
    g = np.random.default_rng(0)
    m, n = 10, 13
    W = (g.standard_normal((m, n)) * 0.02).astype(np.float32)
    A = np.diag(g.uniform(0.5, 2, n)).astype(np.float32)
    B = np.diag(g.uniform(0.5, 2, m)).astype(np.float32)
    qmin, qmax, s, LA, LB, LtA, LtB = _prep(o, W, A, B)
    codes, _ = o.solve(W, LtA, LtB, s, qmin, qmax)
    assert np.array_equal(codes, o.decide(W, s, qmin, qmax))


def test_scale_invariance(oracle_mod):
    """Scaling A or B by a positive constant leaves the normalised factors,
    hence every code, unchanged."""
    o = oracle_mod
    W, A, B = workloads.random_problem(14, 18, seed=9)
    qmin, qmax, s, LA, LB, LtA, LtB = _prep(o, W, A, B)
    ref, Wt = o.solve(W, LtA, LtB, s, qmin, qmax)
    LtA2 = o.normalize(o.factor(A.astype(np.float64) * 3.7))
    LtB2 = o.normalize(o.factor(B.astype(np.float64) * 0.21))
    np.testing.assert_allclose(LtA2, LtA, atol=1e-12)
    codes, _ = o.solve(W, LtA2, LtB2, s, qmin, qmax)
    assert np.array_equal(codes, ref)


# ----------------------------------------------------- identities I1, I2
@pytest.mark.parametrize("shape", [(7, 11), (20, 12), (32, 32)])
def test_error_factorisation_and_loss_identity(oracle_mod, shape):
    """W - V = LtB D LtA^T (all updates of Prop. 3.1 summed) and the proxy loss
    tr(E^T B E A) equals sum_ij D_ij^2 / (dB_i^2 dA_j^2), dA = diag(LA)."""
    o = oracle_mod
    m, n = shape
    W, A, B = workloads.random_problem(m, n, seed=m * n)
    qmin, qmax, s, LA, LB, LtA, LtB = _prep(o, W, A, B)
    codes, Wt = o.solve(W, LtA, LtB, s, qmin, qmax)
    V = s.astype(np.float64)[:, None] * codes
    D = Wt - V
    E = W.astype(np.float64) - V
    np.testing.assert_allclose(LtB @ D @ LtA.T, E, rtol=0, atol=1e-12 * np.abs(E).max())
    loss = o.proxy_loss(W, V, A, B)
    dA, dB = np.diag(LA), np.diag(LB)
    ident = float(np.sum(D ** 2 / (dB[:, None] ** 2 * dA[None, :] ** 2)))
    assert abs(loss - ident) <= 1e-10 * abs(loss)


def test_proxy_loss_closed_form_single_entry(oracle_mod):
    """E = eps * e_i e_j^T gives tr(E^T B E A) = eps^2 * B_ii * A_jj."""
    o = oracle_mod
    _, A, B = workloads.random_problem(5, 6, seed=1)
    W = np.zeros((5, 6))
    V = np.zeros((5, 6))
    V[3, 2] = -0.125
    assert abs(o.proxy_loss(W, V, A, B) - 0.125 ** 2 * float(B[3, 3]) * float(A[2, 2])) < 1e-12


# ----------------------------------------------------------- Corollary 3.4
@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_corollary_3_4_bound_unit_grid(oracle_mod, seed):
    """On a unit-step grid without clamping: |D| <= 1/2 and
    ||B^{1/2}(V-W)A^{1/2}||_F^2 <= 1/4 sum dB^-2 sum dA^-2 <= 1/4 tr(A) tr(B)."""
    o = oracle_mod
    m, n = 16, 20
    W, A, B = workloads.random_problem(m, n, seed=seed)
    W = (W * 100.0 / 0.02).astype(np.float32)  # many steps wide
    s = np.ones(m, np.float32)
    qmin, qmax = -(1 << 20), 1 << 20
    LA, LB = o.factor(A), o.factor(B)
    codes, Wt = o.solve(W, o.normalize(LA), o.normalize(LB), s, qmin, qmax)
    D = Wt - codes
    assert np.abs(D).max() <= 0.5 + 1e-12
    loss = o.proxy_loss(W, codes.astype(np.float64), A, B)
    mid = 0.25 * np.sum(np.diag(LB) ** -2.0) * np.sum(np.diag(LA) ** -2.0)
    top = 0.25 * np.trace(A.astype(np.float64)) * np.trace(B.astype(np.float64))
    assert loss <= mid * (1 + 1e-12)
    assert mid <= top * (1 + 1e-12)


# ------------------------------------------------------------- brute force
@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("seed", [0, 1, 2, 3, 4])
def test_brute_force_2x3_unique_fixed_point(oracle_mod, bits, seed):
    """2x3 inputs: exactly one code matrix is consistent with the intended-
    output recurrence (induction along the product order), and it is the
    solver's.  The least-loss matrix over all enumerated ones is reported and
    cannot beat... nothing is claimed about optimality beyond loss <= solver."""
    o = oracle_mod
    W, A, B = workloads.random_problem(2, 3, seed=seed)
    if seed % 2:
        W = W * 3  # push some entries into the clamp
    qmin, qmax, s, LA, LB, LtA, LtB = _prep(o, W, A, B, bits=bits)
    cnt, first, best_loss, best = o.brute(W, A, B, LtA, LtB, s, qmin, qmax)
    codes, _ = o.solve(W, LtA, LtB, s, qmin, qmax)
    assert cnt == 1
    assert np.array_equal(first, codes)
    V = s.astype(np.float64)[:, None] * codes
    assert best_loss <= o.proxy_loss(W, V, A, B) + 1e-15


# ------------------------------------------------------------------ factor
def test_factor_definition_and_closed_forms(oracle_mod):
    """L = chol(A^{-1}): lower, positive diagonal, L L^T A = I; diagonal A
    gives diag(1/sqrt(a)); 2x2 gives [[sqrt p, 0],[q/sqrt p, sqrt(r - q^2/p)]]
    with A^{-1} = [[p,q],[q,r]]."""
    o = oracle_mod
    _, A, _ = workloads.random_problem(3, 40, seed=2)
    L = o.factor(A)
    assert np.allclose(np.triu(L, 1), 0) and (np.diag(L) > 0).all()
    np.testing.assert_allclose(L @ L.T @ A.astype(np.float64), np.eye(40), atol=1e-10)
    a = np.array([4.0, 0.25, 9.0])
    np.testing.assert_allclose(o.factor(np.diag(a)), np.diag(1 / np.sqrt(a)), atol=1e-15)
    A2 = np.array([[2.0, 1.0], [1.0, 2.0]])  # inverse = [[2,-1],[-1,2]]/3
    p, q, r = 2 / 3, -1 / 3, 2 / 3
    exp = np.array([[np.sqrt(p), 0], [q / np.sqrt(p), np.sqrt(r - q * q / p)]])
    np.testing.assert_allclose(o.factor(A2), exp, atol=1e-15)
    with pytest.raises(o.NotSPD):
        o.factor(np.array([[1.0, 2.0], [2.0, 1.0]]))


def test_scales_and_decision_reading(oracle_mod):
    """Grid reading: symmetric range, fp32 absmax/qmax step, zero row -> 1,
    round half to even, clamp."""
    o = oracle_mod
    assert o.grid(4) == (-7, 7) and o.grid(3) == (-3, 3) and o.grid(2) == (-1, 1)
    W = np.array([[0.7, -1.4, 0.0], [0.0, 0.0, 0.0]], np.float32)
    s = o.scales(W, 7)
    assert s[0] == np.float32(1.4) / np.float32(7) and s[1] == 1.0
    d = o.decide(np.array([[0.5, 1.5, 2.5, -0.5, 9.0, -9.0]]), np.array([1.0], np.float32), -7, 7)
    assert d.tolist() == [[0, 2, 2, 0, 7, -7]]


# --------------------------------------------------- teacher-forced checker
def test_forced_check_counts(oracle_mod):
    """The forced check finds no mismatch on the oracle's own codes; a planted
    far-from-midpoint flip is a failure; and a candidate that flips the
    nearest-to-midpoint decision but is otherwise consistent with its own
    history (what a solver with slightly different rounding produces) shows
    exactly one mismatch, classified as a tie: adopting the candidate's code
    stops the flip from cascading."""
    o = oracle_mod
    W, A, B = workloads.random_problem(12, 15, seed=11)
    qmin, qmax, s, LA, LB, LtA, LtB = _prep(o, W, A, B)
    codes, Wt = o.solve(W, LtA, LtB, s, qmin, qmax)
    r = o.forced_check(W, LtA, LtB, s, qmin, qmax, codes)
    assert r["mismatches"] == 0
    md = o.midpoint_distance(Wt, s, qmin, qmax)
    bad = codes.copy()
    i, j = np.unravel_index(np.argmax(np.where(np.abs(codes) < qmax, md, -1)), md.shape)
    bad[i, j] += 1 if codes[i, j] < qmax else -1
    r = o.forced_check(W, LtA, LtB, s, qmin, qmax, bad)
    assert r["own"][i, j] != bad[i, j] and r["failures"] >= 1
    # consistent candidate with the nearest-to-midpoint decision flipped
    i, j = np.unravel_index(np.argmin(md), md.shape)
    x = Wt[i, j] / float(s[i])
    flipped = int(np.floor(x)) if codes[i, j] == int(np.floor(x)) + 1 else int(np.floor(x)) + 1
    cand = codes.copy()
    cand[i, j] = flipped
    for _ in range(W.size):
        own = o.forced_check(W, LtA, LtB, s, qmin, qmax, cand)["own"]
        nxt = own.copy()
        nxt[i, j] = flipped
        if np.array_equal(nxt, cand):
            break
        cand = nxt
    r = o.forced_check(W, LtA, LtB, s, qmin, qmax, cand, tie_eps=float(md[i, j]) * 1.01 + 1e-15)
    assert r["mismatches"] == 1 and r["ties"] == 1 and r["failures"] == 0
    r = o.forced_check(W, LtA, LtB, s, qmin, qmax, cand, tie_eps=float(md[i, j]) * 0.5)
    assert r["mismatches"] == 1 and r["failures"] == 1


def test_planted_mistakes_are_caught(oracle_mod):
    """Mistakes planted in the oracle's inputs (transposed factor, swapped
    sides, un-normalised factor) change the codes versus the literal mn x mn
    GPTQ, so the pins above would catch them."""
    o = oracle_mod
    W, A, B = workloads.random_problem(10, 12, seed=21)
    qmin, qmax, s, LA, LB, LtA, LtB = _prep(o, W, A, B)
    ref = o.naive(W, A, B, s, qmin, qmax)[0]
    _, Wt_ref = o.solve(W, LtA, LtB, s, qmin, qmax)
    for bad_A, bad_B in ((LtA.T, LtB), (LtA, np.tril(LB)), (LtA, LtB.T)):
        codes, Wt = o.solve(W, np.tril(bad_A), np.tril(bad_B), s, qmin, qmax)
        assert np.abs(Wt - Wt_ref).max() > 1e-6
    # swapping sides needs a square problem to be well formed
    W2, A2, B2 = workloads.random_problem(12, 12, seed=22)
    qmin, qmax, s2, LA2, LB2, LtA2, LtB2 = _prep(o, W2, A2, B2)
    ref2 = o.naive(W2, A2, B2, s2, qmin, qmax)[0]
    assert not np.array_equal(o.solve(W2, LtB2, LtA2, s2, qmin, qmax)[0], ref2)
    assert np.array_equal(o.solve(W2, LtA2, LtB2, s2, qmin, qmax)[0], ref2)
    del ref


# ---------------------------------------------------------------------------
# Per-row step searched for the least round-to-nearest error ("per-row
# scaling factor (shrink) up to factor 2, MSE search": review, free parameters)
# ---------------------------------------------------------------------------
def test_shrink_candidates_span_one_to_one_half(oracle_mod):
    oracle = oracle_mod
    c = oracle.shrink_candidates(100)
    assert c[0] == np.float32(1.0) and c[-1] == np.float32(0.5)
    assert np.all(np.diff(c) < 0) and c.dtype == np.float32
    assert list(oracle.shrink_candidates(2)) == [1.0, 0.5]


def test_shrink_search_hand_examples(oracle_mod):
    oracle = oracle_mod
    # INT2 (q in {-1, 0, 1}), candidates {1, 1/2}.
    # [0.7, 0.34, 0.34]: step 0.7 rounds the small entries to 0 (error
    # 2 * 0.34^2 = 0.2312); step 0.35 keeps 0.7 at the clamp (error 0.35^2) and
    # rounds 0.34 to 0.35 (error 2 * 0.01^2): 0.1227 < 0.2312, so 0.35.
    # [0.7, 0.3, 0]: step 0.7 costs 0.3^2 = 0.09; step 0.35 costs
    # 0.35^2 + 0.05^2 = 0.125, so 0.7.
    W = np.array([[0.7, 0.34, 0.34], [0.7, 0.3, 0.0]], np.float32)
    s, gap = oracle.scales_mse(W, -1, 1, 2)
    assert s[0] == np.float32(np.float32(0.5) * np.float32(0.7)) / np.float32(1)
    assert s[1] == np.float32(0.7)
    err = oracle.row_mse(W, s, -1, 1)
    assert abs(err[0] - (0.35 ** 2 + 2 * 0.01 ** 2)) < 1e-6 and abs(err[1] - 0.09) < 1e-6


def test_shrink_search_on_grid_row_keeps_absmax_step(oracle_mod):
    oracle = oracle_mod
    # a row that already lies on its absmax grid has zero error at c = 1, the
    # first candidate, so the search keeps s = absmax / qmax
    rng = np.random.default_rng(4)
    qmax = 7
    s0 = np.float32(0.0123)
    ints = rng.integers(-qmax, qmax + 1, size=(5, 40)).astype(np.float32)
    ints[:, 0] = qmax
    W = (ints * s0).astype(np.float32)
    s, _ = oracle.scales_mse(W, -qmax, qmax, 50)
    assert np.array_equal(s, oracle.scales(W, qmax))
    assert np.all(oracle.row_mse(W, s, -qmax, qmax) < 1e-18)


def test_shrink_search_never_worse_than_absmax_and_scales_with_rows(oracle_mod):
    oracle = oracle_mod
    rng = np.random.default_rng(5)
    W = (rng.standard_t(3, size=(20, 64)) * 0.02).astype(np.float32)
    s, _ = oracle.scales_mse(W, -7, 7, 40)
    assert np.all(oracle.row_mse(W, s, -7, 7) <= oracle.row_mse(W, oracle.scales(W, 7), -7, 7))
    assert np.all(s <= oracle.scales(W, 7)) and np.all(s >= oracle.scales(W, 7) * np.float32(0.5))
    # a power-of-two scaling of a row scales its step exactly
    s2, _ = oracle.scales_mse((W * np.float32(8)).astype(np.float32), -7, 7, 40)
    assert np.array_equal(s2, (s * np.float32(8)).astype(np.float32))


def test_gram_closed_forms(oracle_mod):
    oracle = oracle_mod
    # X = [[1, 2], [3, 4]]: X^T X / 2 = [[5, 7], [7, 10]], mean diagonal 7.5
    X = np.array([[1.0, 2.0], [3.0, 4.0]])
    assert np.allclose(oracle.gram(X), [[5.0, 7.0], [7.0, 10.0]], rtol=0, atol=1e-15)
    assert np.allclose(oracle.gram(X, 0.1), [[5.75, 7.0], [7.0, 10.75]], rtol=0, atol=1e-15)
    # orthogonal columns give a diagonal factor; sample order does not matter
    Q, _ = np.linalg.qr(np.random.default_rng(6).standard_normal((50, 6)))
    X = Q * np.array([1.0, 2.0, 3.0, 4.0, 5.0, 6.0])
    A = oracle.gram(X)
    assert np.allclose(A, np.diag(np.array([1, 4, 9, 16, 25, 36]) / 50.0), atol=1e-14)
    assert np.allclose(oracle.gram(X[::-1]), A, atol=1e-14)
