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

Two block rotations without the WHT are the variants of the same idea ("压缩与速度的
博弈" [TQ-RQ] section "三种变体": quaternion SO(4) blocks of 4 at 512 FMAs and 128
parameters, Givens 2D blocks of 2 at 256 FMAs and 128 parameters; [RQ-wiki] section
"1. 绕过蝴蝶网络": an independent 2D Givens or 4D quaternion rotation per pair or group of
coordinates, no butterfly network, 128 rotation parameters):
  * "quat":   block k maps y[4k..4k+3] to q_k * y_blk (left multiplication by one unit
              quaternion, a left-isoclinic rotation); parameters [32][4] per head.
  * "planar": pair i maps (y[2i], y[2i+1]) to (c y0 - s y1, s y0 + c y1), the Givens
              rotation by the angle with cosine c and sine s; parameters [64][2] = (c, s)
              per head, rescaled to unit length at use.
The original structure is "iso" (WHT then quaternion pairs, [32][2][4] per head).
Their parameters come from the same counter streams with the variant's index in the
stream identifier; a Givens pair is a uniform point on the unit circle obtained by
normalising a point drawn uniformly from the unit disc (rejection sampling).
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


VARIANTS = ("iso", "quat", "planar")
PARAMS_PER_HEAD = {"iso": 256, "quat": 128, "planar": 128}
PARAM_SHAPE = {"iso": (N_BLOCKS, 2, 4), "quat": (N_BLOCKS, 4), "planar": (D // 2, 2)}


def quat_left_apply(y, params):
    """Block k maps y[4k:4k+4] to q_k * y_blk (params (32, 4), each row rescaled to unit)."""
    q = unit_params(params)
    yb = np.asarray(y, dtype=np.float64).reshape(y.shape[:-1] + (N_BLOCKS, 4))
    return quat_mul(np.broadcast_to(q, yb.shape), yb).reshape(y.shape)


def quat_left_apply_inverse(z, params):
    """The inverse: conj(q_k) * z_blk."""
    q = unit_params(params)
    zb = np.asarray(z, dtype=np.float64).reshape(z.shape[:-1] + (N_BLOCKS, 4))
    return quat_mul(np.broadcast_to(quat_conj(q), zb.shape), zb).reshape(z.shape)


def givens_apply(y, params):
    """Pair i maps (y[2i], y[2i+1]) to (c y0 - s y1, s y0 + c y1) (params (64, 2) = (c, s))."""
    p = unit_params(params)
    yp = np.asarray(y, dtype=np.float64).reshape(y.shape[:-1] + (D // 2, 2))
    c, s = p[:, 0], p[:, 1]
    out = np.stack([c * yp[..., 0] - s * yp[..., 1], s * yp[..., 0] + c * yp[..., 1]], axis=-1)
    return out.reshape(y.shape)


def givens_apply_inverse(z, params):
    """The transpose: (c z0 + s z1, -s z0 + c z1)."""
    p = unit_params(params)
    zp = np.asarray(z, dtype=np.float64).reshape(z.shape[:-1] + (D // 2, 2))
    c, s = p[:, 0], p[:, 1]
    out = np.stack([c * zp[..., 0] + s * zp[..., 1], -s * zp[..., 0] + c * zp[..., 1]], axis=-1)
    return out.reshape(z.shape)


def rotate(x, params, variant="iso"):
    """Forward rotation along the last axis: iso R x = S (H_hat x); quat / planar: the block
    rotation alone (no WHT)."""
    if variant == "iso":
        return so4_apply(wht(x), params)
    if variant == "quat":
        return quat_left_apply(np.asarray(x, dtype=np.float64), params)
    if variant == "planar":
        return givens_apply(np.asarray(x, dtype=np.float64), params)
    raise ValueError(variant)


def rotate_inverse(z, params, variant="iso"):
    """Inverse rotation: iso R^T z = H_hat (S^T z) (H_hat is its own inverse); quat / planar:
    the inverse block rotation."""
    if variant == "iso":
        return wht(so4_apply_inverse(z, params))
    if variant == "quat":
        return quat_left_apply_inverse(np.asarray(z, dtype=np.float64), params)
    if variant == "planar":
        return givens_apply_inverse(np.asarray(z, dtype=np.float64), params)
    raise ValueError(variant)


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


def rotation_matrix(params, d=D, variant="iso"):
    """Explicit d x d matrix of the forward rotation, built column by column by applying it to
    the unit vectors (for "iso" also assembled as S H_hat from the block matrices)."""
    if variant == "iso":
        S = np.zeros((d, d))
        for k, m in enumerate(block_matrices(params)):
            S[4 * k : 4 * k + 4, 4 * k : 4 * k + 4] = m
        return S @ (hadamard_matrix(d) / math.sqrt(d))
    return rotate(np.eye(d), params, variant).T


# ------------------------------------------------------------------- seed -> params
def _mix64(z):
    """splitmix64 output function (S. Vigna, splitmix64.c; its finaliser is D. Stafford's "Mix13")."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def stream_id(layer, head, block, side, variant=0):
    """64-bit identifier of the parameter stream of one quaternion (or Givens pair); variant 0
    ("iso") uses block 0..31 and side 0 (qL) / 1 (qR), 1 ("quat") block 0..31, 2 ("planar")
    pair 0..63 as the block, both with side 0."""
    return (((((variant * 65536 + layer) * 65536) + head) * 64 + block) * 2 + side) & MASK64


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


def random_unit_circle(seed, sid):
    """A uniform point (c, s) on the unit circle, in fp64: (x, y) uniform in the open unit disc
    without the origin (rejection: 0 < r2 = x^2 + y^2 < 1), then (x / r, y / r), r = sqrt(r2)."""
    st = _Stream(seed, sid)
    while True:
        x = 2.0 * st.uniform() - 1.0
        y = 2.0 * st.uniform() - 1.0
        r2 = x * x + y * y
        if 0.0 < r2 < 1.0:
            break
    r = math.sqrt(r2)
    return (x / r, y / r)


def init_rotation(seed, n_layers, n_kv_heads, variant="iso"):
    """Rotation parameters [L][Hkv][*PARAM_SHAPE[variant]], fp32 (fp64 values rounded to
    nearest): iso [32][2][4] (qL, qR per block), quat [32][4], planar [64][2] (c, s)."""
    out = np.zeros((n_layers, n_kv_heads) + PARAM_SHAPE[variant], dtype=np.float32)
    vi = VARIANTS.index(variant)
    for l in range(n_layers):
        for h in range(n_kv_heads):
            if variant == "iso":
                for k in range(N_BLOCKS):
                    for side in range(2):
                        q = random_unit_quaternion(seed, stream_id(l, h, k, side))
                        out[l, h, k, side, :] = np.array(q, dtype=np.float64).astype(np.float32)
            elif variant == "quat":
                for k in range(N_BLOCKS):
                    q = random_unit_quaternion(seed, stream_id(l, h, k, 0, vi))
                    out[l, h, k, :] = np.array(q, dtype=np.float64).astype(np.float32)
            else:
                for i in range(D // 2):
                    out[l, h, i, :] = np.array(random_unit_circle(seed, stream_id(l, h, i, 0, vi)),
                                               dtype=np.float64).astype(np.float32)
    return out
