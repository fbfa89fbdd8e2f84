"""Leaf structure 7 (two tile diagonals per launch) replayed on the host,
over whole multi-tile problems.

The tile-diagonal recursion (Algorithm 6 over tile-diagonal key ranges,
midpoint split) is replayed with three kinds of step:
* leaves, each tile by the cluster leaf's phase schedule;
* band updates as plain products, tile by tile;
* the pair form for every range of exactly two tile diagonals K, K+1.

In the pair form, the node's update from K to K+1 does not run as a band
product. Each tile (I', J') on K+1 instead applies its two neighbours' shares
itself:
* left share: (R_left LtA[J',J'-1]^T) is subtracted from its staged Wt, where
  R_left is the left tile's in-tile R;
* upper share: S_up = LtB[I',I'-1] D_up is added into S before each sub-tile,
  so the sweep's row-side sums apply the LtA factor to it.

The codes and pre-rounding values must equal the oracle's sequential pull
(Theorem 3.2), with and without the pair form.  Leaving out either share
must move the replay off the pull.
"""
import math

import numpy as np
import pytest

import oracle
import workloads
from test_cluster_schedule import T, sweep_tile


def solve_replay(W, LtA, LtB, s, qmin, qmax, pair=True, mistake=None):
    m, n = W.shape
    Mt, Nt = math.ceil(m / T), math.ceil(n / T)
    Mp, Np = Mt * T, Nt * T
    Wt = np.zeros((Mp, Np))
    Wt[:m, :n] = W
    LA = np.zeros((Np, Np))
    LA[:n, :n] = LtA
    LB = np.zeros((Mp, Mp))
    LB[:m, :m] = LtB
    step = np.ones(Mp, np.float32)
    step[:m] = s
    D = np.zeros((Mp, Np))
    R_in = np.zeros((Mp, Np))  # every tile's in-tile R
    codes = np.zeros((Mp, Np), np.int64)
    wt = np.zeros((Mp, Np))

    def tb(i):
        return slice(T * i, T * (i + 1))

    def tiles(k):
        return [(I, k - I) for I in range(Mt) if 0 <= k - I < Nt]

    def leaf_tile(I, J, S_extra=None):
        c, w, d, r = sweep_tile(Wt[tb(I), tb(J)].copy(), LA[tb(J), tb(J)], LB[tb(I), tb(I)], step[tb(I)],
                                min(T, m - T * I), min(T, n - T * J), qmin, qmax, S_extra=S_extra)
        codes[tb(I), tb(J)] = c
        wt[tb(I), tb(J)] = w
        D[tb(I), tb(J)] = d
        R_in[tb(I), tb(J)] = r

    def update(k0, h, k1, l1):
        """Wt of the tiles on diagonals [k1, k1 + l1) loses the contributions
        of the tiles on [k0, k0 + h) (the node's two band products)."""
        for kt in range(k1, k1 + l1):
            for I2, J2 in tiles(kt):
                acc = np.zeros((T, T))
                for ks in range(k0, k0 + h):
                    for I, J in tiles(ks):
                        if I <= I2 and J <= J2:
                            acc += LB[tb(I2), tb(I)] @ D[tb(I), tb(J)] @ LA[tb(J2), tb(J)].T
                Wt[tb(I2), tb(J2)] -= acc

    def pair_leaf(k):
        for I, J in tiles(k):
            leaf_tile(I, J)
        for I2, J2 in tiles(k + 1):
            if J2 >= 1 and mistake != "no_left_share":
                Wt[tb(I2), tb(J2)] -= R_in[tb(I2), tb(J2 - 1)] @ LA[tb(J2), tb(J2 - 1)].T
            S_up = None
            if I2 >= 1 and mistake != "no_upper_share":
                S_up = LB[tb(I2), tb(I2 - 1)] @ D[tb(I2 - 1), tb(J2)]
            leaf_tile(I2, J2, S_up)

    def rec(k, length):
        if length == 1:
            for I, J in tiles(k):
                leaf_tile(I, J)
        elif length == 2 and pair:
            pair_leaf(k)
        else:
            h = length // 2
            rec(k, h)
            update(k, h, k + h, length - h)
            rec(k + h, length - h)

    rec(0, Mt + Nt - 1)
    return codes[:m, :n], wt[:m, :n]


def _problem(m, n, seed):
    W, A, B = workloads.random_problem(m, n, seed=seed)
    LtA = oracle.normalize(oracle.factor(A))
    LtB = oracle.normalize(oracle.factor(B))
    qmin, qmax = oracle.grid(4)
    s = oracle.scales(W, qmax)
    return W, LtA, LtB, s, qmin, qmax


@pytest.mark.parametrize("pair", [True, False])
@pytest.mark.parametrize("shape", [(256, 256), (384, 256), (300, 200)])
def test_tile_recursion_with_pair_leaves_equals_sequential_pull(shape, pair):
    m, n = shape
    W, LtA, LtB, s, qmin, qmax = _problem(m, n, seed=7 * m + n)
    codes, wt = solve_replay(W, LtA, LtB, s, qmin, qmax, pair=pair)
    ref_codes, ref_wt = oracle.solve(W, LtA, LtB, s, qmin, qmax, mode="pull")
    # no entry of these seeded problems lies within 1e-9 of a rounding midpoint
    assert oracle.midpoint_distance(ref_wt, s, qmin, qmax).min() > 1e-9
    assert np.array_equal(codes, ref_codes)
    assert np.abs(wt - ref_wt).max() <= 1e-9 * max(1.0, np.abs(ref_wt).max())


@pytest.mark.parametrize("mistake", ["no_left_share", "no_upper_share"])
def test_pair_replay_needs_both_neighbour_shares(mistake):
    W, LtA, LtB, s, qmin, qmax = _problem(256, 256, seed=3)
    _, ref_wt = oracle.solve(W, LtA, LtB, s, qmin, qmax, mode="pull")
    _, wt = solve_replay(W, LtA, LtB, s, qmin, qmax, pair=True, mistake=mistake)
    assert np.abs(wt - ref_wt).max() > 1e-6
