"""Instrumented op counter for the IsoQuant rotation (oracle).

[RQ-news] section "妙处不只是压缩，而是不再展开" gives 1,408 FMA-class operations for the
whole structured rotation against 16,384 for a dense one, and 256 stored parameters
per head against 16,384.  [TQ-RQ] section "三种变体" lists 512 FMAs for the SO(4)
stage on its own (d = 128).  The split of the 1,408 is not printed; the reading here
is 7 x 128 = 896 add/sub for the seven WHT butterfly stages plus 32 x 16 = 512 for
the 4x4 block products (each block's 4x4 matrix formed once per head from its
quaternion pair; the 1/sqrt(d) scale folded into it).

The variants without the WHT ([TQ-RQ] section "三种变体"; "RotorQuant" sd114.wiki section
"1. 绕过蝴蝶网络") are printed at 512 FMAs and 128 parameters (quaternion blocks of 4) and
256 FMAs and 128 parameters (Givens blocks of 2); they are counted the same way, each block's
matrix built from its parameters and applied with counted multiply / fused multiply-add.

The counts are obtained by running the transforms on a counting scalar type, not by
formula, so a dropped or duplicated stage changes them.
"""

import numpy as np

from .rotation import D, block_matrices, rotate


class Counter:
    def __init__(self):
        self.add = 0
        self.mul = 0
        self.fma = 0


class CNum:
    """A float that counts the operations applied to it."""

    __slots__ = ("v", "c")

    def __init__(self, v, c):
        self.v = v
        self.c = c

    def __add__(self, o):
        self.c.add += 1
        return CNum(self.v + o.v, self.c)

    def __sub__(self, o):
        self.c.add += 1
        return CNum(self.v - o.v, self.c)


def fma(a, b, acc, c):
    """acc + a*b as one fused multiply-add (a is a plain float, b and acc counted)."""
    c.fma += 1
    return CNum(acc.v + a * b.v, c)


def mul(a, b, c):
    c.mul += 1
    return CNum(a * b.v, c)


def count_wht(d=128):
    c = Counter()
    x = [CNum(float(i), c) for i in range(d)]
    h = 1
    while h < d:
        for i in range(0, d, 2 * h):
            for j in range(i, i + h):
                a, b = x[j], x[j + h]
                x[j], x[j + h] = a + b, a - b
        h *= 2
    return c, [v.v for v in x]


def count_blocks(params, y):
    """Apply the 32 block matrices to y with counted multiply / fused multiply-add."""
    c = Counter()
    mats = block_matrices(params)
    out = []
    for k, m in enumerate(mats):
        yb = [CNum(y[4 * k + i], c) for i in range(4)]
        for r in range(4):
            acc = mul(m[r, 0], yb[0], c)
            for col in range(1, 4):
                acc = fma(m[r, col], yb[col], acc, c)
            out.append(acc.v)
    return c, out


def variant_blocks(params, variant):
    """(first coordinate, matrix) of each block of a variant without the WHT; each matrix is
    the block's action read off column by column on unit vectors."""
    size = 4 if variant == "quat" else 2
    R = rotate(np.eye(D), params, variant).T  # column c = image of unit vector c
    return [(k, R[k:k + size, k:k + size]) for k in range(0, D, size)]


def count_variant_blocks(params, variant, y):
    c = Counter()
    out = []
    for k, m in variant_blocks(params, variant):
        n = m.shape[0]
        yb = [CNum(y[k + i], c) for i in range(n)]
        for r in range(n):
            acc = mul(m[r, 0], yb[0], c)
            for col in range(1, n):
                acc = fma(m[r, col], yb[col], acc, c)
            out.append(acc.v)
    return c, out


def count_dense(d=128):
    """A dense d x d rotation applied to one vector, counted the same way."""
    c = Counter()
    rng = np.random.default_rng(0)
    M = rng.standard_normal((d, d))
    y = [CNum(float(v), c) for v in rng.standard_normal(d)]
    for r in range(d):
        acc = mul(M[r, 0], y[0], c)
        for col in range(1, d):
            acc = fma(M[r, col], y[col], acc, c)
    return c


def rotation_op_counts(params, d=128, variant="iso"):
    """{'wht': add/sub count, 'so4': multiply-class count, 'total', 'dense', 'params'}
    ('blocks' instead of 'so4' and no WHT for the quat / planar variants)."""
    if variant != "iso":
        cb, _ = count_variant_blocks(params, variant, [float(i) for i in range(d)])
        n = cb.mul + cb.fma
        return {"wht": 0, "blocks": n, "total": n, "params": int(np.asarray(params).size)}
    cw, y = count_wht(d)
    cb, _ = count_blocks(params, y)
    cd = count_dense(d)
    so4 = cb.mul + cb.fma
    return {
        "wht": cw.add,
        "so4": so4,
        "total": cw.add + so4,
        "dense": cd.mul + cd.fma,
        "params": int(np.asarray(params).size),
        "dense_params": d * d,
    }
