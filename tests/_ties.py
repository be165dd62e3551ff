"""Weight blocks that sit exactly on the quantizers' rounding decisions.

They are inputs only (no arithmetic of the method): the CPU pins check the
oracle's codes on them against values fixed by exact arithmetic, and the GPU
quantizer tests feed the same blocks to the device kernels.

Q4_0 (workload statement: d = signed max-abs / -8, q = clamp(int(w/d + 8.5), 0, 15)):
each listed element w has w/d = k - 8.5 exactly, so w/d + 8.5 is the integer k
and the code is k.  d needs more than 11 significant bits, so fp16(d) differs
from d, and the fp32 reciprocal 1/d is inexact: computing q through w * (1/d),
or through the stored fp16 scale, lands just below k and gives k - 1.

Affine (q = round((w - bias)/scale), ties to even): with bias 0 and scale
2^-e exactly, element (j + 1/2)·scale divides to j + 1/2 exactly, so its code is
the even neighbour of j + 1/2.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

# (d, [(element index, k)]) with d = max / -8 in fp32 exactly, max = -8 d at index 0.
Q4_0_TIE_BLOCKS = [
    (0.27227783203125, [(3, 1)]),
    (0.9024658203125, [(5, 1), (9, 2), (17, 3)]),
    (0.230010986328125, [(2, 1), (30, 2)]),
    (0.021488189697265625, [(1, 1), (16, 2)]),
    (0.0581207275390625, [(7, 1), (31, 2)]),
]


def q4_0_tie_matrix():
    """W[N][32] (one block per row) and the expected codes: listed elements map
    to k, the max element (index 0) to 0, and every other element is d·(j - 8)
    for an integer j in [1, 15] (w/d + 8.5 = j + 1/2, code j)."""
    rows, codes = [], []
    for r, (d, ties) in enumerate(Q4_0_TIE_BLOCKS):
        d32 = np.float32(d)
        w = np.zeros(32, np.float32)
        q = np.zeros(32, np.int64)
        w[0] = np.float32(-8.0) * d32
        for j in range(1, 32):
            jj = 1 + (5 * j + r) % 15
            w[j] = np.float32(jj - 8) * d32
            q[j] = jj
        for i, k in ties:
            w[i] = np.float32(k - 8.5) * d32
            q[i] = k
        rows.append(w)
        codes.append(q)
    return np.stack(rows), np.stack(codes)


def q4_0_tie_exactness():
    """Facts the tie blocks rely on, in exact rational arithmetic."""
    w, q = q4_0_tie_matrix()
    for r, (d, ties) in enumerate(Q4_0_TIE_BLOCKS):
        D = Fraction(float(np.float32(d)))
        assert Fraction(float(w[r, 0])) / Fraction(-8) == D           # d = max / -8 exactly
        for i, k in ties:
            assert Fraction(float(w[r, i])) / D == Fraction(2 * k - 17, 2)
        for j in range(32):
            assert abs(Fraction(float(w[r, j]))) <= abs(Fraction(float(w[r, 0])))
    return True


def affine_tie_matrix(bits: int, group: int = 64):
    """W[2][2*group]: per group, bias 0 (the min, element 0), max L·s (element 1)
    with s = 2^-e, and elements (j + 1/2)·s for j = 0 .. L-1, repeated.  Returns
    W, the scale s per row and the expected codes (ties to even)."""
    L = (1 << bits) - 1
    rows, codes, scales = [], [], []
    for r, e in enumerate((6, 9)):
        s = 2.0 ** -e
        w = np.zeros(2 * group, np.float64)
        q = np.zeros(2 * group, np.int64)
        for gi in range(2):
            base = gi * group
            w[base] = 0.0
            w[base + 1] = L * s
            q[base + 1] = L
            for t in range(2, group):
                j = (t - 2 + 3 * gi + r) % L
                w[base + t] = (j + 0.5) * s
                q[base + t] = j if j % 2 == 0 else j + 1
        rows.append(w.astype(np.float32))
        codes.append(q)
        scales.append(s)
    return np.stack(rows), np.array(scales), np.stack(codes)
