"""The IsoQuant rotation R = S . H_hat (oracle, fp64).

[RQ-abs] and [RQ-news] section "妙处不只是压缩，而是不再展开": each head vector is
first mixed globally by a Walsh–Hadamard transform and then by a block-diagonal
SO(4) rotation acting on groups of four coordinates, before scalar quantisation;
the structure stores 256 parameters per head.  [RQ-wiki] section "3. V 缓存的逆旋转
修复": values read back from the rotated basis must go through the inverse of the
forward rotation.

Readings where the pages are silent (each listed in the design notes):
  * H_hat = H / sqrt(d) with H the Sylvester-ordered Hadamard matrix,
    H[i, j] = (-1)**popcount(i & j); no random sign diagonal.
  * Block k acts on coordinates 4k .. 4k+3, read as the quaternion
    (w, x, y, z) = (y[4k], y[4k+1], y[4k+2], y[4k+3]).
  * Block action: v -> qL * v * conj(qR) (Hamilton product) with unit qL, qR.
    Every such pair is an element of SO(4) and every element of SO(4) arises
    this way (isoclinic decomposition); 32 blocks x 2 quaternions x 4 = 256
    parameters per head.
  * Parameter layout per head: [32 blocks][2: qL, qR][4: w, x, y, z], fp32.
    Stored fp32 quaternions are unit only to ~1e-7; every use divides each one by
    its fp64 norm first, so the rotation applied is exactly orthogonal.
  * Seed -> parameters: a counter-based splitmix64 stream per
    (seed, layer, head, block, side) feeding Marsaglia's (1972) method for a
    uniform point on the 3-sphere; computed in fp64 and rounded to fp32.
    (Parity unpinned: the pages publish no parameter values.)
"""

import math

import numpy as np

D = 128
N_BLOCKS = D // 4
MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15


# ----------------------------------------------------------------------------- WHT
def hadamard_matrix(d=D):
    """Sylvester-ordered Hadamard matrix, H[i, j] = (-1)**popcount(i & j), unnormalised."""
    i = np.arange(d)
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


def wht(x):
    """Normalised WHT along the last axis: returns H_hat @ x (H_hat = H/sqrt(d)).

    Written as the log2(d) butterfly stages of the Sylvester construction; stage s
    combines coordinate pairs (i, i + 2**s) into (a + b, a - b).
    """
    y = np.array(x, dtype=np.float64, copy=True)
    d = y.shape[-1]
    h = 1
    while h < d:
        y = y.reshape(y.shape[:-1] + (d // (2 * h), 2, h))
        a = y[..., 0, :].copy()
        b = y[..., 1, :].copy()
        y[..., 0, :] = a + b
        y[..., 1, :] = a - b
        y = y.reshape(y.shape[:-3] + (d,))
        h *= 2
    return y / math.sqrt(d)


# ------------------------------------------------------------------------ quaternions
def quat_mul(p, q):
    """Hamilton product p*q for arrays of quaternions (..., 4) stored as (w, x, y, z)."""
    pw, px, py, pz = p[..., 0], p[..., 1], p[..., 2], p[..., 3]
    qw, qx, qy, qz = q[..., 0], q[..., 1], q[..., 2], q[..., 3]
    return np.stack(
        [
            pw * qw - px * qx - py * qy - pz * qz,
            pw * qx + px * qw + py * qz - pz * qy,
            pw * qy - px * qz + py * qw + pz * qx,
            pw * qz + px * qy - py * qx + pz * qw,
        ],
        axis=-1,
    )


def quat_conj(q):
    return q * np.array([1.0, -1.0, -1.0, -1.0])


def unit_params(params):
    """fp64 copy of the parameters with every quaternion scaled to unit length."""
    p = np.asarray(params, dtype=np.float64)
    return p / np.sqrt(np.sum(p * p, axis=-1, keepdims=True))


def so4_apply(y, params):
    """z = S y: block k maps y[4k:4k+4] to qL_k * y_blk * conj(qR_k).

    y: (..., 128) fp64; params: (32, 2, 4) (qL, qR per block).
    """
    p = unit_params(params)
    yb = np.asarray(y, dtype=np.float64).reshape(y.shape[:-1] + (N_BLOCKS, 4))
    qL = p[:, 0, :]
    qR = p[:, 1, :]
    z = quat_mul(quat_mul(np.broadcast_to(qL, yb.shape), yb), np.broadcast_to(quat_conj(qR), yb.shape))
    return z.reshape(y.shape)


def so4_apply_inverse(z, params):
    """S^T z: block k maps z_blk to conj(qL_k) * z_blk * qR_k (the inverse rotation)."""
    p = unit_params(params)
    zb = np.asarray(z, dtype=np.float64).reshape(z.shape[:-1] + (N_BLOCKS, 4))
    qL = p[:, 0, :]
    qR = p[:, 1, :]
    y = quat_mul(quat_mul(np.broadcast_to(quat_conj(qL), zb.shape), zb), np.broadcast_to(qR, zb.shape))
    return y.reshape(z.shape)


def rotate(x, params):
    """Forward rotation R x = S (H_hat x) along the last axis."""
    return so4_apply(wht(x), params)


def rotate_inverse(z, params):
    """Inverse rotation R^T z = H_hat (S^T z); H_hat is its own inverse."""
    return wht(so4_apply_inverse(z, params))


def block_matrices(params):
    """The 4x4 matrix of each block, built column by column from the quaternion action."""
    p = unit_params(params)
    mats = np.zeros((N_BLOCKS, 4, 4))
    eye = np.eye(4)
    for k in range(N_BLOCKS):
        for col in range(4):
            v = eye[col]
            mats[k][:, col] = quat_mul(quat_mul(p[k, 0], v), quat_conj(p[k, 1]))
    return mats


def rotation_matrix(params, d=D):
    """Explicit d x d matrix R = S H_hat (for brute-force checks on tiny inputs)."""
    S = np.zeros((d, d))
    for k, m in enumerate(block_matrices(params)):
        S[4 * k : 4 * k + 4, 4 * k : 4 * k + 4] = m
    return S @ (hadamard_matrix(d) / math.sqrt(d))


# ------------------------------------------------------------------- seed -> params
def _mix64(z):
    """splitmix64 output function (S. Vigna, splitmix64.c; its finaliser is D. Stafford's "Mix13")."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def stream_id(layer, head, block, side):
    """64-bit identifier of the parameter stream of one quaternion."""
    return ((((layer * 65536) + head) * 64 + block) * 2 + side) & MASK64


class _Stream:
    """Counter-based uniform doubles: u_i = top 53 bits of mix64(key + (i+1)*GOLDEN) / 2**53,
    key = mix64(seed + GOLDEN) XOR mix64(stream_id + 2*GOLDEN)."""

    def __init__(self, seed, sid):
        self.key = _mix64((seed + GOLDEN) & MASK64) ^ _mix64((sid + 2 * GOLDEN) & MASK64)
        self.i = 0

    def uniform(self):
        self.i += 1
        r = _mix64((self.key + self.i * GOLDEN) & MASK64)
        return (r >> 11) * (1.0 / 9007199254740992.0)


def random_unit_quaternion(seed, sid):
    """Marsaglia's method for a uniform point on S^3, in fp64.

    Draw (x1, x2) uniform in the open unit disc (rejection: s1 = x1^2 + x2^2 < 1),
    then (x3, x4) the same way with 0 < s2 < 1; t = sqrt((1 - s1) / s2);
    q = (x1, x2, x3 t, x4 t).
    """
    st = _Stream(seed, sid)
    while True:
        x1 = 2.0 * st.uniform() - 1.0
        x2 = 2.0 * st.uniform() - 1.0
        s1 = x1 * x1 + x2 * x2
        if s1 < 1.0:
            break
    while True:
        x3 = 2.0 * st.uniform() - 1.0
        x4 = 2.0 * st.uniform() - 1.0
        s2 = x3 * x3 + x4 * x4
        if 0.0 < s2 < 1.0:
            break
    t = math.sqrt((1.0 - s1) / s2)
    return (x1, x2, x3 * t, x4 * t)


def init_rotation(seed, n_layers, n_kv_heads):
    """Rotation parameters [L][Hkv][32][2][4], fp32 (fp64 values rounded to nearest)."""
    out = np.zeros((n_layers, n_kv_heads, N_BLOCKS, 2, 4), dtype=np.float32)
    for l in range(n_layers):
        for h in range(n_kv_heads):
            for k in range(N_BLOCKS):
                for side in range(2):
                    q = random_unit_quaternion(seed, stream_id(l, h, k, side))
                    out[l, h, k, side, :] = np.array(q, dtype=np.float64).astype(np.float32)
    return out
