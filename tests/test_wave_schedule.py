"""The strip-sweep schedule of leaf structure 8, replayed on the host.

The kernel rounds a 128 x 128 tile as four staggered strip sweeps (one per
32-row block).  Each entry's sum is split by where its terms come from (row
side: current sub-tile, previous sub-tile, older sub-tiles, newest column;
column side: this row block, the block above, older row blocks, newest row),
and each part is read at the step the kernel reads it, under the wait that
guards it.  This test replays that schedule in FP64 with the weakest
visibility the waits allow: a value read from another CTA exists only if its
producer's published progress (the wait's threshold, no more) covers it, a
value of this CTA only if it was produced at an earlier step.  Anything the
schedule read too early would read as zero, as it would on the device, and
the codes and pre-rounding values would leave the oracle's sequential pull
(Proposition 3.1's updates in anti-diagonal order; Theorem 3.2).
"""
import numpy as np
import pytest

import oracle
import workloads

T, S3, NB = 128, 32, 4          # tile, strip height, row blocks per tile
K_STEPS = T + S3 - 1            # 159 entry anti-diagonals per strip
LAG, NEED = 48, 33              # start lag; CTA p's step s needs CTA p-1's steps < s + NEED
OS_NEED = 63                    # O_S of sub-tile q waits for the older CTAs' steps < 32 q + OS_NEED
OU_BACK = 17                    # O_U of half h of sub-tile q waits for own steps < 32 q + 16 h - OU_BACK


def _entry(s, b):
    """Entry of lane b at step s: (row in block, column, live)."""
    act = s - b
    live = 0 <= act < T
    ac = min(max(act, 0), T - 1)
    return ac % S3, b + S3 * (ac // S3), live


def replay(W, LtA, LtB, s_rows, qmin, qmax):
    """Codes and pre-rounding values of one tile (m, n <= 128) by the strip
    schedule.  prod[r, c] = the strip-local step that produced D[r, c] and
    R[r, c] (rows are tile rows)."""
    m, n = W.shape
    Wp = np.zeros((T, T))
    Wp[:m, :n] = W
    LA = np.zeros((T, T))
    LA[:n, :n] = LtA
    LB = np.zeros((T, T))
    LB[:m, :m] = LtB
    step = np.ones(T, np.float32)
    step[:m] = s_rows
    D = np.zeros((T, T))
    R = np.zeros((T, T))
    prod = np.full((T, T), 1 << 30)
    codes = np.zeros((T, T), np.int64)
    wt_out = np.zeros((T, T))
    INF = 1 << 30

    def seen_D(rows, c, progress):
        """D[rows, c] as a reader sees it when the producer's progress is
        `progress` (steps < progress are visible)."""
        v = D[rows, c].copy()
        v[prod[rows, c] >= progress] = 0.0
        return v

    for p in range(NB):
        rows = np.arange(p * S3, (p + 1) * S3)
        mrb = max(0, min(S3, m - p * S3))
        # older terms from the product warp: O_S per sub-tile from the CTAs
        # p' <= p-2 (each under its wait on their progress; those CTAs are
        # replayed already), O_U per half sub-tile from this CTA's own R, formed
        # when its own progress reaches the wait's threshold
        OS = np.zeros((S3, T))
        OU = np.zeros((S3, T))
        ou_at = {}
        for q in range(4):
            cols = np.arange(q * S3, (q + 1) * S3)
            if p >= 2:
                P = min(32 * q + OS_NEED, K_STEPS)  # progress of every CTA p' <= p-2
                older = np.arange(0, (p - 1) * S3)
                Dv = np.stack([seen_D(older, c, P) for c in cols], axis=1)
                OS[:, cols] = LB[np.ix_(rows, older)] @ Dv
            for h in range(2):
                if q >= 2:
                    P_own = 32 * q + 16 * h - OU_BACK
                    # the entry warp needs the half's flag at step 32 q + 16 h
                    assert P_own < 32 * q + 16 * h
                    ou_at[P_own] = (q, h)

        def form_ou(q, h, P_own):
            cols = np.arange(q * S3, (q + 1) * S3)
            hr = np.arange(16 * h, 16 * h + 16)
            oc = np.arange(0, S3 * (q - 1))
            Rv = R[np.ix_(rows[hr], oc)].copy()
            Rv[prod[np.ix_(rows[hr], oc)] >= P_own] = 0.0
            OU[np.ix_(hr, cols)] = Rv @ LA[np.ix_(cols, oc)].T

        for s in range(K_STEPS):
            if s in ou_at:  # steps < s are done: own progress = s
                form_ou(*ou_at[s], s)
            # CTA p-1's progress when the block-above sums of step s were read
            # (during step s-1; progress only grows, so the start lag holds too)
            P_up = min(max(LAG, s + NEED), K_STEPS)
            for b in range(S3):
                a, c, live = _entry(s, b)
                r = p * S3 + a
                q = c // S3
                if not live:
                    continue
                valid = a < mrb and c < n
                # row side: current sub-tile up to c-2, previous sub-tile, newest column
                k1 = np.arange(q * S3, c - 1) if c - 1 > q * S3 else np.arange(0)
                k2 = np.arange((q - 1) * S3, q * S3) if q >= 1 else np.arange(0)
                k2 = k2[k2 < c - 1]
                # (entries outside the matrix are never rounded: zero throughout)
                if r < m:
                    for kk in (k1, k2):
                        kk = kk[kk < n]
                        assert np.all(prod[r, kk] <= s - 2)
                w12 = R[r, k1] @ LA[c, k1] + R[r, k2] @ LA[c, k2]
                r_left = R[r, c - 1] if c > 0 else 0.0
                la = LA[c, c - 1] if c > 0 else 0.0
                # column side: this block up to a-2, the block above (pushed), newest row
                rb = np.arange(p * S3, r - 1) if r - 1 > p * S3 else np.arange(0)
                if c < n:
                    assert np.all(prod[rb[rb < m], c] <= s - 2)
                w3 = LB[r, rb] @ D[rb, c]
                w4 = 0.0
                if p >= 1:
                    up = np.arange((p - 1) * S3, p * S3)
                    w4 = LB[r, up] @ seen_D(up, c, P_up)
                d_prev = D[r - 1, c] if a > 0 else 0.0
                lb = LB[r, r - 1] if a > 0 else 0.0
                cs = (lb * d_prev + w3) + w4
                wt = (Wp[r, c] - OU[a, c] - OS[a, c]) - (la * r_left + w12) - cs
                qf = np.float32(wt) / step[r]
                cq = int(np.clip(np.rint(qf), qmin, qmax))
                if valid:
                    dl = wt - float(step[r]) * cq
                    D[r, c] = dl
                    R[r, c] = OS[a, c] + cs + dl
                    prod[r, c] = s
                    codes[r, c] = cq
                    wt_out[r, c] = wt
    assert np.all(prod[:m, :n] < INF)
    return codes[:m, :n], wt_out[:m, :n]


@pytest.mark.parametrize("shape", [(128, 128), (100, 77), (33, 128), (128, 5)])
def test_strip_schedule_equals_sequential_pull(shape):
    m, n = shape
    W, A, B = workloads.random_problem(m, n, seed=11 * m + n)
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


def test_strip_schedule_catches_a_short_wait():
    """The replay is sensitive to the waits: 32 steps is the least the
    column-side wait can ask for (the block above's row 31 of column c is
    rounded at its step 31 + c); with 31 (and the start lag cut to match) the
    pre-rounding values leave the pull."""
    global NEED, LAG
    m = n = 128
    W, A, B = workloads.random_problem(m, n, seed=5)
    LtA = oracle.normalize(oracle.factor(A))
    LtB = oracle.normalize(oracle.factor(B))
    qmin, qmax = oracle.grid(4)
    s = oracle.scales(W, qmax)
    ref_codes, ref_wt = oracle.solve(W, LtA, LtB, s, qmin, qmax, mode="pull")
    saved = NEED, LAG
    try:
        NEED, LAG = 32, 32
        _, wt_ok = replay(W, LtA, LtB, s, qmin, qmax)
        NEED, LAG = 31, 31
        _, wt_short = replay(W, LtA, LtB, s, qmin, qmax)
    finally:
        NEED, LAG = saved
    assert np.abs(wt_ok - ref_wt).max() <= 1e-9 * max(1.0, np.abs(ref_wt).max())
    assert np.abs(wt_short - ref_wt).max() > 1e-6


@pytest.mark.parametrize("knob,ok,short", [("OS_NEED", 63, 62), ("OU_BACK", 17, 18)])
def test_product_warp_thresholds_are_tight(knob, ok, short):
    """The product warp's two waits are exactly sufficient: the older row
    blocks' D of sub-tile q is complete after their step 32 q + 62 (row 31,
    column 32 q + 31), and rows 16 h .. 16 h + 15 of this CTA have finished
    sub-tile q - 2 after step 32 q + 16 h - 18; one step less and the replay
    leaves the pull."""
    m = n = 128
    W, A, B = workloads.random_problem(m, n, seed=9)
    LtA = oracle.normalize(oracle.factor(A))
    LtB = oracle.normalize(oracle.factor(B))
    qmin, qmax = oracle.grid(4)
    s = oracle.scales(W, qmax)
    _, ref_wt = oracle.solve(W, LtA, LtB, s, qmin, qmax, mode="pull")
    saved = globals()[knob]
    try:
        globals()[knob] = ok
        _, wt_ok = replay(W, LtA, LtB, s, qmin, qmax)
        globals()[knob] = short
        _, wt_short = replay(W, LtA, LtB, s, qmin, qmax)
    finally:
        globals()[knob] = saved
    assert np.abs(wt_ok - ref_wt).max() <= 1e-9 * max(1.0, np.abs(ref_wt).max())
    assert np.abs(wt_short - ref_wt).max() > 1e-6
