"""Shared test utilities: oracle-side encoding of seeded inputs, cache upload, guard bands and
the record of parity margins."""

import numpy as np

from oracle import attention, encode, packing, rotation
from rotated_bit_kv_iq_b200 import inputs

TILE = 32


def oracle_params(seed, n_layers, n_kv_heads, variant="iso"):
    """Rotation parameters drawn by the oracle's own generator (the product's generator is
    checked against it bit for bit in the host tests; the oracle never uses the product's)."""
    return rotation.init_rotation(seed, n_layers, n_kv_heads, variant)


def oracle_encode_stream(params_head, layer, head, which, t0, n, n_outliers=4, heavy_frac=0.0, seed=inputs.DATA_SEED):
    """Seeded fp16 tokens of one (layer, kv head, K|V) stream and their oracle encoding."""
    x = inputs.kv_tokens(seed, layer, head, which, t0, n, n_outliers=n_outliers, heavy_frac=heavy_frac)
    return x, encode.encode(x, params_head)


def tile_records(k_codes, k_n16, v_codes, v_n16, k_bits=3, v_bits=3):
    """Oracle-packed tile records of tokens 0..T-1 of one (sequence, kv head):
    (ceil(T/32), tile bytes) uint8; slots past T are zero."""
    T = k_codes.shape[0]
    nt = (T + TILE - 1) // TILE
    kr, vbk = packing.k_record_bytes(k_bits), packing.v_block_bytes(v_bits)
    krec = np.zeros((nt * TILE, kr), np.uint8)
    krec[:T] = packing.pack_k_fast(k_codes, k_bits)
    vrec = np.zeros((nt * 2, vbk), np.uint8)
    vb = packing.pack_v_fast(v_codes, v_bits)
    vrec[:vb.shape[0]] = vb
    kn = np.zeros(nt * TILE, np.uint16)
    vn = np.zeros(nt * TILE, np.uint16)
    kn[:T] = k_n16
    vn[:T] = v_n16
    rec = np.concatenate([krec.reshape(nt, TILE * kr), vrec.reshape(nt, 2 * vbk),
                          kn.reshape(nt, TILE).view(np.uint8), vn.reshape(nt, TILE).view(np.uint8)], axis=1)
    assert rec.shape[1] == TILE * kr + 2 * vbk + 128
    return rec


def upload_sequence(cache, layer, seq_pages, head, k_codes, k_n16, v_codes, v_n16):
    """Write oracle-packed records of tokens 0..T-1 of one sequence/head into the device pool
    (one host-to-device copy) in the cache's code widths.  seq_pages: physical page ids of the
    sequence, in order."""
    import torch

    ps = cache.page_size
    T = k_codes.shape[0]
    if T == 0:
        return
    kb, vb = cache.k_bits, cache.v_bits
    rec = torch.from_numpy(tile_records(k_codes, k_n16, v_codes, v_n16, kb, vb)).to(cache.pool.device)
    nt = rec.shape[0]
    t0 = np.arange(nt) * TILE
    pages = torch.as_tensor(np.asarray(seq_pages)[t0 // ps].astype(np.int64), device=cache.pool.device)
    tiles = torch.as_tensor((t0 % ps) // TILE, dtype=torch.int64, device=cache.pool.device)
    tv = cache.tiles()
    # a partial last tile keeps the pool's bytes of the slots past T
    full = nt if T % TILE == 0 else nt - 1
    if full:
        tv[layer, pages[:full], head, tiles[:full]] = rec[:full]
    if full < nt:
        m = T - full * TILE
        last = tv[layer, pages[full], head, tiles[full]].clone()
        r = rec[full]
        kr, vbk = packing.k_record_bytes(kb), packing.v_block_bytes(vb)
        kv0 = TILE * kr
        kn0 = kv0 + 2 * vbk
        last[:kr * m] = r[:kr * m]
        nblk = (m + 15) // 16
        last[kv0:kv0 + vbk * nblk] = r[kv0:kv0 + vbk * nblk]
        last[kn0:kn0 + 2 * m] = r[kn0:kn0 + 2 * m]
        last[kn0 + 64:kn0 + 64 + 2 * m] = r[kn0 + 64:kn0 + 64 + 2 * m]
        tv[layer, pages[full], head, tiles[full]] = last


def max_rel_err(out, ref):
    """Per row: ||o - r||_inf / ||r||_inf; returns the maximum over rows."""
    out = np.asarray(out, dtype=np.float64).reshape(-1, 128)
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, 128)
    den = np.abs(ref).max(axis=1)
    den = np.where(den > 0, den, 1.0)
    return float((np.abs(out - ref).max(axis=1) / den).max())


def oracle_attention(q, k_codes, k_n16, v_codes, v_n16, params):
    return attention.attention_rotated(q, k_codes, k_n16, v_codes, v_n16, params)


PARITY_RECORDS = []


def record_parity(case, max_rel_err=None, excluded=None, codes=None, norm_ulp=None):
    """Keep one case's parity margins for the terminal summary (tests/conftest.py)."""
    PARITY_RECORDS.append({"case": case, "max_rel_err": max_rel_err, "excluded": excluded, "codes": codes,
                                    "norm_ulp": norm_ulp})


# ------------------------------------------------------------------ guard bands
CANARY = 0x5A  # byte written before and after every output and workspace a GPU test hands to a kernel
GUARD = 4096


class Guarded:
    """A device buffer with GUARD bytes of canary on each side; `.t` is the usable view."""

    def __init__(self, shape, dtype, fill=None, device="cuda"):
        import torch

        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + ((n + 255) // 256) * 256 + GUARD,), CANARY, dtype=torch.uint8, device=device)
        self.n = n
        body = self.raw[GUARD:GUARD + n]
        self.t = body.view(dtype).view(*shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, label=""):
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.n:]
        assert bool((head == CANARY).all()), f"{label}: bytes written before the buffer"
        assert bool((tail == CANARY).all()), f"{label}: bytes written after the buffer"
