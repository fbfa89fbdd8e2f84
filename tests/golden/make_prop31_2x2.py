"""Writes prop31_2x2.txt: a 2 x 2 solve worked out by hand from Proposition
3.1 of "BaKron: Efficient Quantization with Kronecker-Factored Hessians" (the
Kronecker update L^B_i Delta_ij (L^A_j)^T, with the factors normalised to a
unit diagonal), in exact rational arithmetic.  It calls neither the oracle nor
the CUDA library.

    A = [[2,1],[1,2]]  ->  LtA[1,0] = -A01/A11 = -1/2
    B = [[4,2],[2,3]]  ->  LtB[1,0] = -B01/B11 = -2/3
    Wt00 = W00
    Wt01 = W01 + D00/2                         (D00 reaches column 1 through LtA[1,0])
    Wt10 = W10 + 2 D00/3                       (D00 reaches row 1 through LtB[1,0])
    Wt11 = W11 - D00/3 + 2 D01/3 + D10/2
with D = Wt - s_i * code and code = clamp(rint(Wt / s_i)), ties to even.

Run:  python tests/golden/make_prop31_2x2.py
"""
import os
from fractions import Fraction as F

A = [[2, 1], [1, 2]]
B = [[4, 2], [2, 3]]
W = [["0.30", "0.41"], ["-0.22", "0.17"]]
S = ["0.125", "0.0625"]  # exact binary steps
QMIN, QMAX = -7, 7


def rnd(x, s):
    q = x / s
    fl = q.numerator // q.denominator
    r = q - fl
    c = fl + 1 if r > F(1, 2) else fl if r < F(1, 2) else (fl if fl % 2 == 0 else fl + 1)
    return max(QMIN, min(QMAX, c))


def solve():
    w = [[F(x) for x in row] for row in W]
    s = [F(x) for x in S]
    la, lb = F(-A[0][1], A[1][1]), F(-B[0][1], B[1][1])
    wt = [[None, None], [None, None]]
    c = [[None, None], [None, None]]
    d = [[None, None], [None, None]]
    order = [(0, 0), (0, 1), (1, 0), (1, 1)]
    for i, j in order:
        if (i, j) == (0, 0):
            v = w[0][0]
        elif (i, j) == (0, 1):
            v = w[0][1] - la * d[0][0]
        elif (i, j) == (1, 0):
            v = w[1][0] - lb * d[0][0]
        else:
            v = w[1][1] - (lb * la * d[0][0] + lb * d[0][1] + la * d[1][0])
        wt[i][j] = v
        c[i][j] = rnd(v, s[i])
        d[i][j] = v - s[i] * c[i][j]
    return la, lb, wt, c


def main():
    la, lb, wt, c = solve()
    lines = [
        "# 2 x 2 BaKron solve worked by hand from Proposition 3.1 (normalised factors,",
        "# Kronecker update L^B_i Delta_ij (L^A_j)^T), exact rationals; written by",
        "# make_prop31_2x2.py (no oracle, no CUDA).",
        f"A {A[0][0]} {A[0][1]} {A[1][0]} {A[1][1]}",
        f"B {B[0][0]} {B[0][1]} {B[1][0]} {B[1][1]}",
        f"W {W[0][0]} {W[0][1]} {W[1][0]} {W[1][1]}",
        f"s {S[0]} {S[1]}",
        f"grid {QMIN} {QMAX}",
        f"LtA10 {la}",
        f"LtB10 {lb}",
        "Wt " + " ".join(str(wt[i][j]) for i in range(2) for j in range(2)),
        "codes " + " ".join(str(c[i][j]) for i in range(2) for j in range(2)),
    ]
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "prop31_2x2.txt")
    with open(path, "w") as f:
        f.write("\n".join(lines) + "\n")
    print(path)


if __name__ == "__main__":
    main()
