"""IsoQuant encoder (oracle, fp64), step by step in the pages' order.

[RQ-news] section "妙处不只是压缩，而是不再展开" and [RQ-abs]: rotate first (WHT,
then the block SO(4) rotations) so that energy is spread evenly over coordinates,
then quantise each coordinate with a scalar quantiser to 3 bits.  [TQ-RQ] section
"Beta 分布的魔力": the rotation acts on the unit vector, whose rotated
coordinates are close to N(0, 1/d); section "Lloyd-Max 最优量化": the quantiser is
the Lloyd–Max codebook for that law, applied by lookup.

Steps for one fp16 vector x in R^128:
  1. promote to fp64;           2. n = ||x||_2;
  3. x_hat = x / n (0 if n = 0); 4. y = H_hat x_hat;
  5. z = S y (quaternion blocks); 6. u = sqrt(d) z  (N(0,1) units);
  7. code = #{ j : u > b_j }  (b = N(0,1) Lloyd–Max boundaries, ascending), so a
     value equal to a boundary goes to the lower cell and code k names the k-th
     centroid in ascending order;
  8. norm stored as IEEE binary16, round-to-nearest-even, saturating at 65504.
"""

import math

import numpy as np

from .codebook import codebook
from .rotation import rotate

D = 128
FP16_MAX = 65504.0
BOUNDARY_BAND = 1e-6  # |u - b_j| below this (N(0,1) units) is excluded from bit-exact checks


def norm_to_fp16_bits(n):
    """fp64 norms -> binary16 bit patterns, RNE, saturating at 65504 (and a count of saturations)."""
    n = np.asarray(n, dtype=np.float64)
    with np.errstate(over="ignore"):
        h = n.astype(np.float16)  # numpy rounds fp64 -> fp16 to nearest even in one step
    sat = ~np.isfinite(h)
    h = np.where(sat, np.float16(FP16_MAX), h)
    return h.view(np.uint16), int(sat.sum())


def fp16_bits_to_float(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def encode(x16, params_head, bits=3, variant="iso"):
    """Encode fp16 vectors of one (layer, kv head).

    x16: (N, 128) float16 (or anything exactly representable in it).
    params_head: rotation parameters of that head ((32, 2, 4) for "iso"; see oracle.rotation).
    bits: 2, 3 or 4 (the 2**bits-level Lloyd–Max codebook).
    Returns dict with
      codes  (N, 128) uint8   -- ascending centroid index per rotated coordinate
      norm16 (N,) uint16      -- binary16 bits of ||x||
      u      (N, 128) fp64    -- rotated unit-vector coordinates in N(0,1) units
      near   (N, 128) bool    -- |u - b_j| < 1e-6 for some boundary b_j
      saturated int           -- norms clamped to 65504
    """
    x = np.asarray(x16, dtype=np.float16).astype(np.float64)
    assert x.shape[-1] == D
    n = np.sqrt(np.sum(x * x, axis=-1))
    safe = np.where(n > 0.0, n, 1.0)
    x_hat = np.where((n > 0.0)[..., None], x / safe[..., None], 0.0)
    z = rotate(x_hat, params_head, variant)
    u = math.sqrt(D) * z
    _, b = codebook(bits)
    codes = quantise(u, bits)
    near = np.zeros(u.shape, dtype=bool)
    for bj in b:  # within the band of any boundary
        near |= np.abs(u - bj) < BOUNDARY_BAND
    n16, sat = norm_to_fp16_bits(n)
    return {"codes": codes, "norm16": n16, "u": u, "near": near, "saturated": sat, "norm": n}


def quantise(u, bits=3):
    """Step 7: code = number of boundaries strictly below u (ties go to the lower cell)."""
    _, b = codebook(bits)
    return np.sum(np.asarray(u, dtype=np.float64)[..., None] > b, axis=-1).astype(np.uint8)


def nearest_centroid(u, bits=3):
    """Brute-force nearest centroid index (ties to the lower index); a check on step 7."""
    c, _ = codebook(bits)
    dist = np.abs(np.asarray(u)[..., None] - c)
    return np.argmin(dist, axis=-1).astype(np.uint8)
