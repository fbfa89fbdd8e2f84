"""The phase schedule of the default cluster leaf (structure 6), replayed on
the host.

Each 128 x 128 tile runs on four CTAs, CTA p owning row block p.  In phase
e = p + q CTA p sweeps its sub-tile (p, q) in 63 entry anti-diagonal steps.
Before the sweep, the sub-tile's staged Wt loses two products:
    S[p,q]  = sum_{p' < p} LtB[p,p'] D[p',q]       (column side, older row blocks),
    U[p,q]  = sum_{q' < q} R[p,q'] LtA[q,q']^T     (row side, older sub-tiles).
The product warp forms the parts that need only phases <= e - 2 during phase
e - 1 (O_S over p' <= p - 2, O_U over q' <= q - 2).  The newest 32-deep parts
(p' = p - 1, q' = q - 1) are formed after the cluster barrier that opens
phase e.  Inside the sweep, an entry's sums are the sub-tile's own row and
column terms: the side warps form all but the newest, and the entry warp adds
those.  R's block (p, q) starts as S and ends as S plus this block's column
sums plus D.

The replay computes every part at the time the kernel computes it, and
asserts that every value it reads was produced early enough (phase and
step).  Codes and pre-rounding values must equal the oracle's sequential pull
(Proposition 3.1's updates in anti-diagonal order; Theorem 3.2).
"""
import numpy as np
import pytest

import oracle
import workloads

T, S3, NB = 128, 32, 4


def sweep_tile(Wp, LA, LB, step, m, n, qmin, qmax, S_extra=None, mistake=None):
    """One 128 x 128 tile by the phase schedule: staged Wt ``Wp``, the tile's
    diagonal factor blocks ``LA`` (columns) and ``LB`` (rows), row steps, the
    extent (m, n) inside the matrix.  ``S_extra`` (the pair form's upper
    neighbour share) is added into S before each sub-tile.  Returns (codes,
    pre-rounding values, D, in-tile R), all 128 x 128."""
    D = np.zeros((T, T))
    R = np.zeros((T, T))
    phase_of = np.full((T, T), 1 << 20)  # phase that produced D / R (block-wise)
    codes = np.zeros((T, T), np.int64)
    wt_out = np.zeros((T, T))
    blk = lambda i: slice(S3 * i, S3 * (i + 1))  # noqa: E731

    def older(e, p, q):
        """O_S and O_U of sub-tile (p, q), formed during phase e - 1 from
        phases <= e - 2."""
        os_ = np.zeros((S3, S3))
        ou = np.zeros((S3, S3))
        for pr in range(p - 1):
            assert phase_of[S3 * pr, S3 * q] <= e - 2
            os_ += LB[blk(p), blk(pr)] @ D[blk(pr), blk(q)]
        for qr in range(q - 1):
            assert phase_of[S3 * p, S3 * qr] <= e - 2
            ou += R[blk(p), blk(qr)] @ LA[blk(q), blk(qr)].T
        return os_, ou

    for e in range(2 * NB - 1):
        # the product warp's part for this phase, formed during the last one
        staged = {}
        for p in range(NB):
            q = e - p
            if 0 <= q < NB:
                staged[p] = older(e, p, q)
        # cluster barrier: phases <= e - 1 visible; the newest terms, then W0
        W0 = {}
        for p, (os_, ou) in staged.items():
            q = e - p
            S = os_.copy()
            U = ou.copy()
            if p >= 1 and mistake != "drop_newest_column_block":
                assert phase_of[S3 * (p - 1), S3 * q] == e - 1
                S += LB[blk(p), blk(p - 1)] @ D[blk(p - 1), blk(q)]
            if q >= 1:
                assert phase_of[S3 * p, S3 * (q - 1)] == e - 1
                U += R[blk(p), blk(q - 1)] @ LA[blk(q), blk(q - 1)].T
            if S_extra is not None:
                S += S_extra[blk(p), blk(q)]
            W0[p] = Wp[blk(p), blk(q)] - U - S
            R[blk(p), blk(q)] = S  # R's block starts as S
        # the sweeps: 63 steps, every CTA of the phase in parallel
        for p in W0:
            q = e - p
            mrb = max(0, min(S3, m - p * S3))
            rstep = np.full((S3, S3), 1 << 20)  # step that rounded (a, b) in this sweep
            for d in range(2 * S3 - 1):
                for b in range(S3):
                    a = d - b
                    if not 0 <= a < S3:
                        continue
                    r, c = S3 * p + a, S3 * q + b
                    valid = a < mrb and c < n
                    # row side: columns <= b-2 of the sub-tile (side warp), b-1 (entry)
                    cs_ = np.arange(0, max(b - 1, 0))
                    assert np.all(rstep[a, cs_] <= d - 2)
                    pu = R[r, S3 * q + cs_] @ LA[c, S3 * q + cs_]
                    r_new = R[r, c - 1] if b > 0 else 0.0
                    la_new = (LA[c - 1, c] if mistake == "transposed_factor" else LA[c, c - 1]) if b > 0 else 0.0
                    # column side: rows <= a-2 of the row block (side warp), a-1 (entry)
                    rs_ = np.arange(0, max(a - 1, 0))
                    assert np.all(rstep[rs_, b] <= d - 2)
                    ps = LB[r, S3 * p + rs_] @ D[S3 * p + rs_, c]
                    d_prev = D[r - 1, c] if a > 0 else 0.0
                    lb_new = LB[r, r - 1] if a > 0 else 0.0
                    s_ab = R[r, c]  # S[a][b] until this entry overwrites it
                    if mistake == "R_without_S":
                        s_ab = 0.0
                    sc = lb_new * d_prev + ps
                    wt = W0[p][a, b] - (r_new * la_new + pu) - sc
                    cq = int(np.clip(np.rint(np.float32(wt) / step[r]), qmin, qmax))
                    if valid:
                        dl = wt - float(step[r]) * cq
                        D[r, c] = dl
                        R[r, c] = s_ab + sc + dl
                        codes[r, c] = cq
                        wt_out[r, c] = wt
                    rstep[a, b] = d
            phase_of[blk(p), blk(q)] = e
    return codes, wt_out, D, R


def replay(W, LtA, LtB, s_rows, qmin, qmax, mistake=None):
    """Codes and pre-rounding values of one tile (m, n <= 128).  ``mistake``
    plants one error in the replay (for the sensitivity test)."""
    m, n = W.shape
    Wp = np.zeros((T, T))
    Wp[:m, :n] = W
    LA = np.zeros((T, T))
    LA[:n, :n] = LtA
    LB = np.zeros((T, T))
    LB[:m, :m] = LtB
    step = np.ones(T, np.float32)
    step[:m] = s_rows
    codes, wt, _, _ = sweep_tile(Wp, LA, LB, step, m, n, qmin, qmax, mistake=mistake)
    return codes[:m, :n], wt[:m, :n]


@pytest.mark.parametrize("shape", [(128, 128), (100, 77), (33, 128), (128, 5)])
def test_phase_schedule_equals_sequential_pull(shape):
    m, n = shape
    W, A, B = workloads.random_problem(m, n, seed=13 * m + n)
    LtA = oracle.normalize(oracle.factor(A))
    LtB = oracle.normalize(oracle.factor(B))
    qmin, qmax = oracle.grid(4)
    s = oracle.scales(W, qmax)
    codes, wt = replay(W, LtA, LtB, s, qmin, qmax)
    ref_codes, ref_wt = oracle.solve(W, LtA, LtB, s, qmin, qmax, mode="pull")
    # no entry of these seeded problems lies within 1e-9 of a rounding midpoint
    assert oracle.midpoint_distance(ref_wt, s, qmin, qmax).min() > 1e-9
    assert np.array_equal(codes, ref_codes)
    assert np.abs(wt - ref_wt).max() <= 1e-9 * max(1.0, np.abs(ref_wt).max())


@pytest.mark.parametrize("mistake", ["drop_newest_column_block", "transposed_factor", "R_without_S"])
def test_phase_schedule_replay_catches_a_planted_mistake(mistake):
    """Each planted error (the newest column-side block left out, the
    sub-diagonal factor entry read transposed, R's block not starting from
    S) moves the replay off the pull, so the replay checks the split."""
    m = n = 128
    W, A, B = workloads.random_problem(m, n, seed=21)
    LtA = oracle.normalize(oracle.factor(A))
    LtB = oracle.normalize(oracle.factor(B))
    qmin, qmax = oracle.grid(4)
    s = oracle.scales(W, qmax)
    _, ref_wt = oracle.solve(W, LtA, LtB, s, qmin, qmax, mode="pull")
    _, wt = replay(W, LtA, LtB, s, qmin, qmax, mistake=mistake)
    assert np.abs(wt - ref_wt).max() > 1e-6
