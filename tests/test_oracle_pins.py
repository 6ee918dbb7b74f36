"""Pins for the CPU oracle: each check ties it to something other than itself --
printed values, textbook tables, closed forms, library routines, brute force."""

import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.optimize
import scipy.stats
import torch

from oracle import attention, codebook, encode, opcount, packing, rotation

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, *v = line.split()
        vals[k] = v
    return vals


def _params(seed=1, layer=0, head=0):
    return rotation.init_rotation(seed, layer + 1, head + 1)[layer, head]


# ------------------------------------------------------------------ codebook
def test_lloyd_max_matches_textbook_table():
    g = _golden("lloyd_max_gaussian_3bit.txt")
    c, b = codebook.codebook(3)
    def half_unit(v):  # 0.6 units of the last printed digit (the 1960 table's own rounding slack)
        return 0.6 * 10.0 ** -(len(v.split(".")[1]) if "." in v else 0)

    for got, printed in [(c[4:], g["output_levels"]), (-c[:4][::-1], g["output_levels"]), (b[3:], g["decision_levels"])]:
        for x, v in zip(got, printed):
            assert abs(x - float(v)) <= half_unit(v) + 1e-12, (x, v)
    assert abs(codebook.gaussian_mse(c, b) - float(g["mse"][0])) <= half_unit(g["mse"][0])


def test_lloyd_max_is_a_minimum_of_mse():
    """An independent optimiser (Nelder-Mead on the MSE functional) finds the same levels."""
    c, b = codebook.codebook(3)

    def mse(pos):
        levels = np.sort(np.concatenate([-pos[::-1], pos]))
        bounds = 0.5 * (levels[1:] + levels[:-1])
        return codebook.gaussian_mse(levels, bounds)

    res = scipy.optimize.minimize(mse, x0=np.array([0.3, 0.9, 1.5, 2.4]), method="Nelder-Mead",
                                  options={"xatol": 1e-10, "fatol": 1e-14, "maxiter": 20000})
    np.testing.assert_allclose(np.sort(res.x), c[4:], atol=1e-5)


def test_gaussian_mse_against_monte_carlo():
    c, b = codebook.codebook(3)
    x = np.random.default_rng(7).standard_normal(2_000_000)
    q = c[np.searchsorted(b, x, side="left")]
    assert abs(np.mean((x - q) ** 2) - codebook.gaussian_mse(c, b)) < 2e-4


def test_codebook_scaled_for_dimension():
    c, b = codebook.codebook(3)
    ct, bt = codebook.codebook_for_dim(128, 3)
    np.testing.assert_allclose(ct * math.sqrt(128), c, rtol=0, atol=1e-15)
    assert b[3] == 0.0 and np.all(np.diff(c) > 0)


# ------------------------------------------------------------------ WHT
def test_hadamard_matches_scipy_and_orthogonality():
    H = rotation.hadamard_matrix(128)
    np.testing.assert_array_equal(H, scipy.linalg.hadamard(128))
    np.testing.assert_array_equal(H @ H.T, 128 * np.eye(128))


def test_fast_wht_equals_matrix():
    x = np.random.default_rng(1).standard_normal((5, 128))
    H = scipy.linalg.hadamard(128) / math.sqrt(128)
    np.testing.assert_allclose(rotation.wht(x), x @ H.T, atol=1e-13)
    np.testing.assert_allclose(rotation.wht(rotation.wht(x)), x, atol=1e-13)


# ------------------------------------------------------------------ SO(4) blocks
def test_hamilton_product_against_textbook_table():
    """i*j = k, j*k = i, k*i = j, i*i = -1 (Hamilton's rules)."""
    one, i, j, k = np.eye(4)
    np.testing.assert_array_equal(rotation.quat_mul(i, j), k)
    np.testing.assert_array_equal(rotation.quat_mul(j, k), i)
    np.testing.assert_array_equal(rotation.quat_mul(k, i), j)
    np.testing.assert_array_equal(rotation.quat_mul(i, i), -one)
    np.testing.assert_array_equal(rotation.quat_mul(j, i), -k)


def test_sandwich_is_rodrigues_rotation():
    """q v q^-1 with q = (cos t, sin t a) rotates the vector part by 2t about a (Rodrigues)."""
    rng = np.random.default_rng(3)
    for _ in range(10):
        a = rng.standard_normal(3)
        a /= np.linalg.norm(a)
        t = rng.uniform(-math.pi, math.pi)
        v = rng.standard_normal(3)
        q = np.concatenate([[math.cos(t)], math.sin(t) * a])
        params = np.zeros((32, 2, 4))
        params[:] = np.eye(4)[0]
        params[0, 0] = q
        params[0, 1] = q
        z = rotation.so4_apply(np.concatenate([[0.0], v, np.zeros(124)]), params)
        th = 2 * t
        rod = v * math.cos(th) + np.cross(a, v) * math.sin(th) + a * np.dot(a, v) * (1 - math.cos(th))
        np.testing.assert_allclose(z[1:4], rod, atol=1e-13)
        assert abs(z[0]) < 1e-13


def test_blocks_are_so4_and_match_left_right_matrices():
    p = rotation.unit_params(_params())
    mats = rotation.block_matrices(p)

    def Lmat(q):  # left multiplication by q, explicit
        w, x, y, z = q
        return np.array([[w, -x, -y, -z], [x, w, -z, y], [y, z, w, -x], [z, -y, x, w]])

    def Rmat(q):  # right multiplication by q, explicit
        w, x, y, z = q
        return np.array([[w, -x, -y, -z], [x, w, z, -y], [y, -z, w, x], [z, y, -x, w]])

    for kk, m in enumerate(mats):
        qL, qR = p[kk]
        qRc = qR * np.array([1, -1, -1, -1])
        np.testing.assert_allclose(m, Lmat(qL) @ Rmat(qRc), atol=1e-14)
        np.testing.assert_allclose(m.T @ m, np.eye(4), atol=1e-14)
        assert abs(np.linalg.det(m) - 1.0) < 1e-13
        # left and right isoclinic factors commute
        np.testing.assert_allclose(Lmat(qL) @ Rmat(qRc), Rmat(qRc) @ Lmat(qL), atol=1e-14)


def test_round_trip_and_explicit_matrix():
    p = _params(1, 3, 2)
    x = np.random.default_rng(5).standard_normal((7, 128))
    R = rotation.rotation_matrix(p)
    np.testing.assert_allclose(R @ R.T, np.eye(128), atol=1e-13)
    np.testing.assert_allclose(rotation.rotate(x, p), x @ R.T, atol=1e-13)
    assert np.abs(rotation.rotate_inverse(rotation.rotate(x, p), p) - x).max() <= 1e-12
    # the inverse is the transpose, written out
    np.testing.assert_allclose(rotation.rotate_inverse(x, p), x @ R, atol=1e-13)


def test_params_unit_deterministic_and_spread():
    P = rotation.init_rotation(1, 2, 3)
    assert P.shape == (2, 3, 32, 2, 4) and P.dtype == np.float32
    n = np.linalg.norm(P.astype(np.float64), axis=-1)
    assert np.abs(n - 1).max() < 3e-7
    np.testing.assert_array_equal(P, rotation.init_rotation(1, 2, 3))
    assert not np.array_equal(P, rotation.init_rotation(2, 2, 3))
    # Haar measure on S^3: each coordinate has mean 0 and second moment 1/4
    Q = rotation.init_rotation(9, 8, 8).reshape(-1, 4).astype(np.float64)
    assert np.abs(Q.mean(0)).max() < 0.03
    assert np.abs((Q ** 2).mean(0) - 0.25).max() < 0.02


def test_rotated_unit_vectors_have_variance_one_over_d():
    """Coordinates of rotated random unit vectors: mean 0, variance 1/d; near N(0, 1/d)."""
    p = _params()
    x = np.random.default_rng(2).standard_normal((4000, 128))
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    z = rotation.rotate(x, p)
    assert abs(z.var() * 128 - 1) < 0.01
    ks = scipy.stats.kstest(z.ravel() * math.sqrt(128), "norm")
    assert ks.statistic < 0.01


# ------------------------------------------------------------------ op counts
def test_op_counts_match_the_printed_figures():
    g = _golden("rotation_op_counts.txt")
    cnt = opcount.rotation_op_counts(_params())
    assert cnt["total"] == int(g["total_fma"][0])
    assert cnt["so4"] == int(g["so4_fma"][0])
    assert cnt["dense"] == int(g["dense_fma"][0])
    assert cnt["params"] == int(g["params_per_head"][0])
    assert cnt["dense_params"] == int(g["dense_params"][0])
    assert cnt["wht"] == 7 * 128


def test_counted_transforms_compute_the_rotation():
    p = _params()
    _, y = opcount.count_wht(128)
    _, z = opcount.count_blocks(p, y)
    x = np.arange(128, dtype=np.float64)
    np.testing.assert_allclose(np.array(z), rotation.rotate(x, p) * math.sqrt(128), atol=1e-9)


# ------------------------------------------------------------------ encoder
def test_quantise_tie_rule_and_brute_force():
    c, b = codebook.codebook(3)
    for j, bj in enumerate(b):
        assert encode.quantise(np.array([bj]))[0] == j  # a boundary goes to the lower cell
    u = np.random.default_rng(4).standard_normal(100000) * 1.3
    np.testing.assert_array_equal(encode.quantise(u), encode.nearest_centroid(u))


def test_encode_constructed_centroid_vectors():
    """x = n R^T c~[k*] (rounded to fp16) must encode to k* with norm ~ n ||c~[k*]||.

    The encoder rescales to unit length, so u = f c[k*] with f = sqrt(d)/||c[k*]||; the
    codes are preserved while f keeps every level inside its cell (0.82 < f < 1.29), which
    holds when k* is drawn with the Gaussian cell probabilities."""
    p = _params(1, 0, 0)
    c, b = codebook.codebook(3)
    ct, _ = codebook.codebook_for_dim(128)
    e_ = np.concatenate([[-np.inf], b, [np.inf]])
    mass = scipy.stats.norm.cdf(e_[1:]) - scipy.stats.norm.cdf(e_[:-1])
    rng = np.random.default_rng(11)
    for _ in range(20):
        kstar = rng.choice(8, size=128, p=mass / mass.sum())
        f = math.sqrt(128) / np.linalg.norm(c[kstar])
        assert 0.85 < f < 1.25
        n = rng.uniform(0.5, 300.0)
        x = (n * rotation.rotate_inverse(ct[kstar], p)).astype(np.float16)
        e = encode.encode(x[None], p)
        np.testing.assert_array_equal(e["codes"][0], kstar)
        assert abs(e["norm"][0] - n * np.linalg.norm(ct[kstar])) < 1e-2 * n


def test_encode_zero_vector_and_saturation():
    p = _params()
    e = encode.encode(np.zeros((1, 128), np.float16), p)
    assert np.all(e["codes"] == 3) and e["norm16"][0] == 0
    big = np.full((1, 128), 60000.0, np.float16)
    e = encode.encode(big, p)
    assert e["saturated"] == 1 and e["norm16"][0] == np.float16(65504).view(np.uint16)


def test_norm_fp16_rounding_is_nearest_even():
    # 1 + 2^-11 lies halfway between 1 and 1 + 2^-10: ties to even -> 1.0
    bits, _ = encode.norm_to_fp16_bits(np.array([1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2049.0]))
    np.testing.assert_array_equal(bits.view(np.float16).astype(np.float64), [1.0, 1.0 + 2 * 2.0 ** -10, 2048.0])


# ------------------------------------------------------------------ packing
def test_chunk_golden_fixtures():
    g = _golden("packing_chunks.txt")
    ya = [s % 8 for s in range(32)]
    assert packing.pack_chunk(ya).hex() == g["chunk_mod8"][0]
    yb = [7 if s % 4 == 0 else 0 for s in range(32)]
    assert packing.pack_chunk(yb).hex() == g["chunk_slot_mod4_0_is_7"][0]
    assert packing.unpack_chunk(bytes.fromhex(g["chunk_mod8"][0])) == ya


def test_v_block_golden_fixtures():
    g = _golden("packing_chunks.txt")
    c = np.zeros((16, 128), np.uint8)
    c[0] = 7
    rec = packing.pack_v(c)[0]
    assert rec[:192].tobytes().hex() == g["vblock_token0_7_head"][0]
    # chunks (g, 0, h) are the Case B chunk, every other chunk is zero
    for q in range(64):
        want = g["chunk_slot_mod4_0_is_7"][0] if (q // 2) % 4 == 0 else "00" * 12
        assert rec[12 * q : 12 * q + 12].tobytes().hex() == want, q
    m = np.tile(np.arange(128) % 8, (16, 1)).astype(np.uint8)
    rec = packing.pack_v(m)[0]
    for tq in range(4):
        for h in range(2):
            q = 2 * (4 * 5 + tq) + h
            assert rec[12 * q : 12 * q + 12].tobytes().hex() == g["vblock_coordmod8_chunk_g5"][0]


def test_pack_round_trip_and_ownership():
    rng = np.random.default_rng(12)
    codes = rng.integers(0, 8, (37, 128)).astype(np.uint8)
    np.testing.assert_array_equal(packing.unpack_k(packing.pack_k(codes)), codes)
    np.testing.assert_array_equal(packing.unpack_v(packing.pack_v(codes), 37), codes)
    np.testing.assert_array_equal(packing.pack_k_fast(codes), packing.pack_k(codes))
    np.testing.assert_array_equal(packing.pack_v_fast(codes), packing.pack_v(codes))
    np.testing.assert_array_equal(packing.unpack_v_fast(packing.pack_v(codes), 37), codes)
    # the bits of a V block that change with token u are exactly the bits the owner map
    # gives to u: nibbles j(u) and j(u)+4 of the words of chunks (g, tq(u), h)
    own = packing.v_bit_owner()
    assert np.all(np.bincount(own, minlength=16) == 384)
    base = rng.integers(0, 8, (16, 128)).astype(np.uint8)
    bits0 = np.unpackbits(packing.pack_v(base)[0], bitorder="little")
    for u in (0, 5, 10, 15):
        alt = base.copy()
        alt[u] = 7 - alt[u]  # flips every code bit of token u
        bits1 = np.unpackbits(packing.pack_v(alt)[0], bitorder="little")
        np.testing.assert_array_equal(np.nonzero(bits0 != bits1)[0], np.nonzero(own == u)[0])
        for t in range(16):
            if t != u:
                assert not np.any(bits0[own == t] != bits1[own == t])
        j, tq = 2 * (u // 8) + (u % 2), (u % 8) // 2
        for q in np.unique(np.nonzero(own == u)[0] // 96):
            assert (q // 2) % 4 == tq
        nib = (np.nonzero(own == u)[0] % 32) // 4
        assert set(nib.tolist()) == {j, j + 4}
    # K record for codes = coordinate mod 8 is four copies of the mod-8 fixture
    k = packing.pack_k(np.array([np.arange(128) % 8], np.uint8))[0].tobytes().hex()
    assert k == _golden("packing_chunks.txt")["chunk_mod8"][0] * 4


# ------------------------------------------------------------------ attention
def _cache(Hkv, T, seed=0):
    rng = np.random.default_rng(seed)
    P = rotation.init_rotation(1, 1, Hkv)[0]
    kc = rng.integers(0, 8, (Hkv, T, 128)).astype(np.uint8)
    vc = rng.integers(0, 8, (Hkv, T, 128)).astype(np.uint8)
    kn, _ = encode.norm_to_fp16_bits(rng.uniform(1, 60, (Hkv, T)))
    vn, _ = encode.norm_to_fp16_bits(rng.uniform(1, 10, (Hkv, T)))
    return P, kc, kn, vc, vn


def test_rotated_equals_dequantised_attention():
    P, kc, kn, vc, vn = _cache(2, 37)
    q = np.random.default_rng(1).standard_normal((8, 128))
    a = attention.attention_rotated(q, kc, kn, vc, vn, P)
    b = attention.attention_dequant(q, kc, kn, vc, vn, P)
    assert np.abs(a - b).max() / np.abs(b).max() < 1e-10


def test_dequantised_attention_matches_torch_sdpa():
    P, kc, kn, vc, vn = _cache(2, 29)
    q = np.random.default_rng(2).standard_normal((6, 128))
    out = attention.attention_dequant(q, kc, kn, vc, vn, P)
    for kv in range(2):
        K = torch.from_numpy(attention.dequantise(kc[kv], kn[kv], P[kv]))
        V = torch.from_numpy(attention.dequantise(vc[kv], vn[kv], P[kv]))
        Q = torch.from_numpy(q[3 * kv : 3 * kv + 3])
        ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None])[0]
        np.testing.assert_allclose(out[3 * kv : 3 * kv + 3], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    P, kc, kn, vc, vn = _cache(1, 16)
    q = np.random.default_rng(3).standard_normal((2, 128))
    V0 = attention.dequantise(vc[0], vn[0], P[0])
    one = attention.attention_rotated(q, kc[:, :1], kn[:, :1], vc[:, :1], vn[:, :1], P)
    np.testing.assert_allclose(one, np.repeat(V0[:1], 2, 0), atol=1e-12)
    zero_q = attention.attention_rotated(np.zeros((1, 128)), kc, kn, vc, vn, P)
    np.testing.assert_allclose(zero_q[0], V0.mean(0), atol=1e-12)
    same_k = attention.attention_rotated(q, np.repeat(kc[:, :1], 16, 1), np.repeat(kn[:, :1], 16, 1), vc, vn, P)
    np.testing.assert_allclose(same_k, np.repeat(V0.mean(0)[None], 2, 0), atol=1e-12)
    empty = attention.attention_rotated(q, kc[:, :0], kn[:, :0], vc[:, :0], vn[:, :0], P)
    assert np.all(empty == 0)


def test_gqa_head_mapping():
    P, kc, kn, vc, vn = _cache(2, 10)
    q = np.random.default_rng(4).standard_normal((4, 128))
    out = attention.attention_rotated(q, kc, kn, vc, vn, P)
    swapped = attention.attention_rotated(q[[2, 3, 0, 1]], kc[::-1], kn[::-1], vc[::-1], vn[::-1], P[::-1])
    np.testing.assert_allclose(out, swapped[[2, 3, 0, 1]], atol=1e-13)


def test_planted_mistakes_are_caught():
    """A dropped inverse rotation or a transposed block must break the pins above."""
    P, kc, kn, vc, vn = _cache(1, 8)
    q = np.random.default_rng(5).standard_normal((1, 128))
    good = attention.attention_dequant(q, kc, kn, vc, vn, P)
    ct, _ = codebook.codebook_for_dim(128)
    # mistake 1: accumulate V in the rotated basis and forget the inverse rotation
    nk = encode.fp16_bits_to_float(kn[0])
    nv = encode.fp16_bits_to_float(vn[0])
    s = nk * (ct[kc[0].astype(int)] @ rotation.rotate(q[0], P[0])) / math.sqrt(128)
    p = np.exp(s - s.max())
    no_inverse = (p * nv) @ ct[vc[0].astype(int)] / p.sum()
    assert np.abs(no_inverse - good[0]).max() > 0.1 * np.abs(good).max()
    # mistake 2: transposed blocks (conj on the wrong side) is not the same rotation
    Pbad = P.copy()
    Pbad[..., 0, :], Pbad[..., 1, :] = P[..., 1, :], P[..., 0, :]
    x = np.random.default_rng(6).standard_normal(128)
    assert np.abs(rotation.rotate(x, Pbad[0]) - rotation.rotate(x, P[0])).max() > 1e-3


# ------------------------------------------------------------------ other bit widths
@pytest.mark.parametrize("bits,tag", [(2, "n4"), (4, "n16")])
def test_lloyd_max_2_and_4_bit_match_textbook_table(bits, tag):
    g = _golden("lloyd_max_gaussian_2bit_4bit.txt")
    c, b = codebook.codebook(bits)
    n = 1 << bits

    def slack(v):
        return 0.6 * 10.0 ** -(len(v.split(".")[1]) if "." in v else 0)

    for got, printed in [(c[n // 2:], g[f"{tag}_output_levels"]), (-c[:n // 2][::-1], g[f"{tag}_output_levels"]),
                         (b[n // 2 - 1:], g[f"{tag}_decision_levels"])]:
        assert len(got) == len(printed)
        for x, v in zip(got, printed):
            assert abs(x - float(v)) <= slack(v) + 1e-12, (x, v)
    mse = codebook.gaussian_mse(c, b)
    tol = 1e-5 if bits == 4 else slack(g[f"{tag}_mse"][0])
    assert abs(mse - float(g[f"{tag}_mse"][0])) <= tol, mse


@pytest.mark.parametrize("bits", [2, 4])
def test_lloyd_max_2_and_4_bit_are_minima_of_mse(bits):
    """An independent optimiser (Nelder-Mead on the MSE functional) finds the same levels, and
    a Monte Carlo estimate of the error agrees with the closed form."""
    c, b = codebook.codebook(bits)
    n = 1 << bits

    def mse(pos):
        levels = np.sort(np.concatenate([-pos[::-1], pos]))
        return codebook.gaussian_mse(levels, 0.5 * (levels[1:] + levels[:-1]))

    x0 = np.linspace(0.2, 2.5, n // 2)
    res = scipy.optimize.minimize(mse, x0=x0, method="Nelder-Mead",
                                  options={"xatol": 1e-11, "fatol": 1e-15, "maxiter": 200000, "maxfev": 200000})
    np.testing.assert_allclose(np.sort(res.x), c[n // 2:], atol=2e-5)
    x = np.random.default_rng(8).standard_normal(2_000_000)
    q = c[np.searchsorted(b, x, side="left")]
    assert abs(np.mean((x - q) ** 2) - codebook.gaussian_mse(c, b)) < 3e-4


@pytest.mark.parametrize("bits", [2, 4])
def test_chunk_golden_fixtures_other_widths(bits):
    g = _golden("packing_chunks.txt")
    if bits == 4:
        y = [s % 16 for s in range(32)]
        assert packing.pack_chunk(y, 4).hex() == g["chunk4_mod16"][0]
        assert packing.unpack_chunk(bytes.fromhex(g["chunk4_mod16"][0]), 4) == y
    else:
        y = [s % 4 for s in range(32)]
        assert packing.pack_chunk(y, 2).hex() == g["chunk2_mod4"][0]
        assert packing.unpack_chunk(bytes.fromhex(g["chunk2_mod4"][0]), 2) == y
        y = [3 if 8 <= s < 16 else 0 for s in range(32)]
        assert packing.pack_chunk(y, 2).hex() == g["chunk2_slots8to15_are_3"][0]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_round_trip_and_ownership_all_widths(bits):
    rng = np.random.default_rng(13)
    top = (1 << bits) - 1
    codes = rng.integers(0, top + 1, (37, 128)).astype(np.uint8)
    np.testing.assert_array_equal(packing.unpack_k(packing.pack_k(codes, bits), bits), codes)
    np.testing.assert_array_equal(packing.unpack_v(packing.pack_v(codes, bits), 37, bits), codes)
    np.testing.assert_array_equal(packing.pack_k_fast(codes, bits), packing.pack_k(codes, bits))
    np.testing.assert_array_equal(packing.pack_v_fast(codes, bits), packing.pack_v(codes, bits))
    np.testing.assert_array_equal(packing.unpack_v_fast(packing.pack_v(codes, bits), 37, bits), codes)
    np.testing.assert_array_equal(packing.unpack_k_fast(packing.pack_k(codes, bits), bits), codes)
    own = packing.v_bit_owner(bits)
    assert np.all(np.bincount(own, minlength=16) == 128 * bits)
    base = rng.integers(0, top + 1, (16, 128)).astype(np.uint8)
    bits0 = np.unpackbits(packing.pack_v(base, bits)[0], bitorder="little")
    cbits = 32 * bits  # bits per chunk
    for u in (0, 6, 9, 15):
        alt = base.copy()
        alt[u] = top - alt[u]  # flips every code bit of token u
        bits1 = np.unpackbits(packing.pack_v(alt, bits)[0], bitorder="little")
        np.testing.assert_array_equal(np.nonzero(bits0 != bits1)[0], np.nonzero(own == u)[0])
        # in every width token u owns nibbles j and j+4 of every word of its 16 chunks
        j, tq = 2 * (u // 8) + (u % 2), (u % 8) // 2
        pos = np.nonzero(own == u)[0]
        assert set(((pos // cbits) // 2 % 4).tolist()) == {tq}
        assert set(((pos % 32) // 4).tolist()) == {j, j + 4}


# ------------------------------------------------------------------ rotation variants
def test_variant_params_shapes_units_and_streams():
    for v in ("quat", "planar"):
        P = rotation.init_rotation(1, 2, 3, v)
        assert P.shape == (2, 3) + rotation.PARAM_SHAPE[v] and P.dtype == np.float32
        assert P[0, 0].size == rotation.PARAMS_PER_HEAD[v] == 128
        n = np.linalg.norm(P.astype(np.float64), axis=-1)
        assert np.abs(n - 1).max() < 3e-7
        np.testing.assert_array_equal(P, rotation.init_rotation(1, 2, 3, v))
    # Givens angles are uniform on the circle: mean of (c, s) ~ 0, E[c^2] = 1/2
    G = rotation.init_rotation(5, 8, 8, "planar").reshape(-1, 2).astype(np.float64)
    assert np.abs(G.mean(0)).max() < 0.03 and abs((G[:, 0] ** 2).mean() - 0.5) < 0.02
    # the variants' streams differ from the iso streams
    Q = rotation.init_rotation(1, 1, 1, "quat")[0, 0]
    I = rotation.init_rotation(1, 1, 1, "iso")[0, 0]
    assert not np.array_equal(Q, I[:, 0])


def test_planar_blocks_are_givens_rotations():
    """Each 2x2 block equals the matrix exponential of the skew generator of its angle
    (scipy.linalg.expm), an independent construction of the Givens rotation."""
    P = rotation.init_rotation(3, 1, 1, "planar")[0, 0].astype(np.float64)
    R = rotation.rotation_matrix(P, variant="planar")
    for i in range(64):
        c, s = P[i] / np.linalg.norm(P[i])
        th = math.atan2(s, c)
        ref = scipy.linalg.expm(np.array([[0.0, -th], [th, 0.0]]))
        np.testing.assert_allclose(R[2 * i:2 * i + 2, 2 * i:2 * i + 2], ref, atol=1e-14)
    off = R.copy()
    for i in range(64):
        off[2 * i:2 * i + 2, 2 * i:2 * i + 2] = 0
    assert np.all(off == 0)


def test_quat_blocks_are_left_isoclinic():
    """Each 4x4 block is left multiplication by its unit quaternion (the explicit matrix of
    Hamilton's product), lies in SO(4), and commutes with every right multiplication."""
    P = rotation.init_rotation(4, 1, 1, "quat")[0, 0].astype(np.float64)
    R = rotation.rotation_matrix(P, variant="quat")

    def Lmat(q):
        w, x, y, z = q
        return np.array([[w, -x, -y, -z], [x, w, -z, y], [y, z, w, -x], [z, -y, x, w]])

    def Rmat(q):
        w, x, y, z = q
        return np.array([[w, -x, -y, -z], [x, w, z, -y], [y, -z, w, x], [z, y, -x, w]])

    rng = np.random.default_rng(9)
    for k in range(32):
        q = P[k] / np.linalg.norm(P[k])
        m = R[4 * k:4 * k + 4, 4 * k:4 * k + 4]
        np.testing.assert_allclose(m, Lmat(q), atol=1e-14)
        assert abs(np.linalg.det(m) - 1) < 1e-13
        p = rng.standard_normal(4)
        np.testing.assert_allclose(m @ Rmat(p), Rmat(p) @ m, atol=1e-13)


@pytest.mark.parametrize("variant", ["quat", "planar"])
def test_variant_round_trip_orthogonal(variant):
    P = rotation.init_rotation(2, 1, 1, variant)[0, 0]
    R = rotation.rotation_matrix(P, variant=variant)
    np.testing.assert_allclose(R @ R.T, np.eye(128), atol=1e-13)
    assert abs(np.linalg.det(R) - 1) < 1e-10
    x = np.random.default_rng(5).standard_normal((7, 128))
    assert np.abs(rotation.rotate_inverse(rotation.rotate(x, P, variant), P, variant) - x).max() <= 1e-12
    np.testing.assert_allclose(rotation.rotate_inverse(x, P, variant), x @ R, atol=1e-13)


def test_variant_op_counts_match_the_printed_figures():
    g = _golden("rotation_op_counts.txt")
    q = opcount.rotation_op_counts(rotation.init_rotation(1, 1, 1, "quat")[0, 0], variant="quat")
    p = opcount.rotation_op_counts(rotation.init_rotation(1, 1, 1, "planar")[0, 0], variant="planar")
    assert q["total"] == int(g["quat_fma"][0]) and q["wht"] == 0
    assert p["total"] == int(g["planar_fma"][0]) and p["wht"] == 0
    assert q["params"] == p["params"] == int(g["variant_params"][0])


@pytest.mark.parametrize("variant,bits", [("iso", 2), ("iso", 4), ("quat", 3), ("planar", 3), ("planar", 4)])
def test_encode_constructed_centroid_vectors_all_forms(variant, bits):
    """x = n R^T c~[k*] (rounded to fp16) encodes to k* for every width and rotation (k* drawn
    with the cell probabilities so that the unit-length rescaling keeps each level in its cell)."""
    P = rotation.init_rotation(1, 1, 1, variant)[0, 0]
    c, b = codebook.codebook(bits)
    ct, _ = codebook.codebook_for_dim(128, bits)
    e_ = np.concatenate([[-np.inf], b, [np.inf]])
    mass = scipy.stats.norm.cdf(e_[1:]) - scipy.stats.norm.cdf(e_[:-1])
    rng = np.random.default_rng(17)
    done = 0
    while done < 10:
        kstar = rng.choice(1 << bits, size=128, p=mass / mass.sum())
        u = math.sqrt(128) / np.linalg.norm(c[kstar]) * c[kstar]
        if np.any(encode.quantise(u, bits) != kstar):  # rescaling crossed a boundary: draw again
            continue
        n = rng.uniform(0.5, 300.0)
        x = (n * rotation.rotate_inverse(ct[kstar], P, variant)).astype(np.float16)
        e = encode.encode(x[None], P, bits, variant)
        ok = e["codes"][0] == kstar
        assert np.all(ok | e["near"][0]), np.nonzero(~ok)
        done += 1


@pytest.mark.parametrize("variant,kb,vb", [("iso", 4, 2), ("iso", 4, 3), ("quat", 3, 3), ("planar", 3, 2)])
def test_rotated_equals_dequantised_attention_all_forms(variant, kb, vb):
    rng = np.random.default_rng(21)
    Hkv, T = 2, 29
    P = rotation.init_rotation(1, 1, Hkv, variant)[0]
    kc = rng.integers(0, 1 << kb, (Hkv, T, 128)).astype(np.uint8)
    vc = rng.integers(0, 1 << vb, (Hkv, T, 128)).astype(np.uint8)
    kn, _ = encode.norm_to_fp16_bits(rng.uniform(1, 60, (Hkv, T)))
    vn, _ = encode.norm_to_fp16_bits(rng.uniform(1, 10, (Hkv, T)))
    q = rng.standard_normal((6, 128))
    a = attention.attention_rotated(q, kc, kn, vc, vn, P, kb, vb, variant)
    b = attention.attention_dequant(q, kc, kn, vc, vn, P, kb, vb, variant)
    assert np.abs(a - b).max() / np.abs(b).max() < 1e-10
    for kv in range(Hkv):  # and the dequantised form is plain softmax attention (torch SDPA, fp64)
        K = torch.from_numpy(attention.dequantise(kc[kv], kn[kv], P[kv], kb, variant))
        V = torch.from_numpy(attention.dequantise(vc[kv], vn[kv], P[kv], vb, variant))
        Q = torch.from_numpy(q[3 * kv:3 * kv + 3])
        ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None])[0]
        np.testing.assert_allclose(b[3 * kv:3 * kv + 3], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_planted_variant_mistakes_are_caught():
    """A Givens pair applied with the sign of its sine flipped, or a quaternion applied on the
    right instead of the left, is a different rotation: the explicit-matrix pins would fail."""
    x = np.random.default_rng(6).standard_normal(128)
    Pp = rotation.init_rotation(1, 1, 1, "planar")[0, 0].astype(np.float64)
    flipped = Pp * np.array([1.0, -1.0])
    assert np.abs(rotation.rotate(x, flipped, "planar") - rotation.rotate(x, Pp, "planar")).max() > 1e-3
    Pq = rotation.init_rotation(1, 1, 1, "quat")[0, 0].astype(np.float64)
    q = rotation.unit_params(Pq)
    right = rotation.quat_mul(x.reshape(32, 4), q).reshape(128)
    assert np.abs(right - rotation.rotate(x, Pq, "quat")).max() > 1e-3


def test_prefill_attention_is_causal_sdpa():
    """The oracle's chunked prefill equals torch SDPA (fp64) on the dequantised cache with an
    explicit causal mask (query i of the chunk sees keys 0 .. start + i)."""
    rng = np.random.default_rng(31)
    Hkv, G, start, C = 2, 3, 11, 7
    T = start + C
    P = rotation.init_rotation(1, 1, Hkv)[0]
    kc = rng.integers(0, 8, (Hkv, T, 128)).astype(np.uint8)
    vc = rng.integers(0, 8, (Hkv, T, 128)).astype(np.uint8)
    kn, _ = encode.norm_to_fp16_bits(rng.uniform(1, 40, (Hkv, T)))
    vn, _ = encode.norm_to_fp16_bits(rng.uniform(1, 10, (Hkv, T)))
    q = rng.standard_normal((C, Hkv * G, 128))
    out = attention.prefill_attention(q, kc, kn, vc, vn, P, start)
    mask = torch.from_numpy(np.arange(T)[None, :] <= start + np.arange(C)[:, None])
    for kv in range(Hkv):
        K = torch.from_numpy(attention.dequantise(kc[kv], kn[kv], P[kv]))
        V = torch.from_numpy(attention.dequantise(vc[kv], vn[kv], P[kv]))
        for g in range(G):
            h = kv * G + g
            Q = torch.from_numpy(q[:, h])
            ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None], attn_mask=mask[None])[0]
            np.testing.assert_allclose(out[:, h], ref.numpy(), rtol=1e-12, atol=1e-12)
    # the last query token sees the whole cache: plain decode attention
    np.testing.assert_allclose(out[-1], attention.attention_rotated(q[-1], kc, kn, vc, vn, P), atol=1e-13)


def test_mixed_attention_pins():
    """Attention over an fp16 prefix plus packed positions: equals torch SDPA (fp64) on the
    concatenated keys and values; with no prefix it is the packed attention; with no packed
    positions it is plain attention on the fp16 vectors."""
    rng = np.random.default_rng(41)
    Hkv, G, P, T2 = 2, 4, 13, 9
    Pr = rotation.init_rotation(3, 1, Hkv)[0]
    k16 = (rng.standard_normal((Hkv, P, 128)) * 2).astype(np.float16)
    v16 = rng.standard_normal((Hkv, P, 128)).astype(np.float16)
    kc = rng.integers(0, 8, (Hkv, T2, 128)).astype(np.uint8)
    vc = rng.integers(0, 8, (Hkv, T2, 128)).astype(np.uint8)
    kn, _ = encode.norm_to_fp16_bits(rng.uniform(1, 30, (Hkv, T2)))
    vn, _ = encode.norm_to_fp16_bits(rng.uniform(1, 10, (Hkv, T2)))
    q = rng.standard_normal((Hkv * G, 128))
    out = attention.attention_mixed(q, k16, v16, kc, kn, vc, vn, Pr)
    for kv in range(Hkv):
        K = torch.from_numpy(np.concatenate([k16[kv].astype(np.float64), attention.dequantise(kc[kv], kn[kv], Pr[kv])]))
        V = torch.from_numpy(np.concatenate([v16[kv].astype(np.float64), attention.dequantise(vc[kv], vn[kv], Pr[kv])]))
        Q = torch.from_numpy(q[kv * G:(kv + 1) * G])
        ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None])[0]
        np.testing.assert_allclose(out[kv * G:(kv + 1) * G], ref.numpy(), rtol=1e-12, atol=1e-12)
    none = attention.attention_mixed(q, k16[:, :0], v16[:, :0], kc, kn, vc, vn, Pr)
    np.testing.assert_allclose(none, attention.attention_rotated(q, kc, kn, vc, vn, Pr), atol=1e-12)
    only = attention.attention_mixed(q, k16, v16, kc[:, :0], kn[:, :0], vc[:, :0], vn[:, :0], Pr)
    for kv in range(Hkv):
        K = torch.from_numpy(k16[kv].astype(np.float64))
        V = torch.from_numpy(v16[kv].astype(np.float64))
        Q = torch.from_numpy(q[kv * G:(kv + 1) * G])
        ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None])[0]
        np.testing.assert_allclose(only[kv * G:(kv + 1) * G], ref.numpy(), rtol=1e-12, atol=1e-12)
