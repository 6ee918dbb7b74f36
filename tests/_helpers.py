"""Shared test utilities: oracle-side encoding of seeded inputs and cache upload."""

import numpy as np

from oracle import attention, encode, packing
from rotated_bit_kv_iq_b200 import inputs


def oracle_encode_stream(params_head, layer, head, which, t0, n, n_outliers=4, heavy_frac=0.0, seed=inputs.DATA_SEED):
    """Seeded fp16 tokens of one (layer, kv head, K|V) stream and their oracle encoding."""
    x = inputs.kv_tokens(seed, layer, head, which, t0, n, n_outliers=n_outliers, heavy_frac=heavy_frac)
    return x, encode.encode(x, params_head)


def upload_sequence(cache, layer, seq_pages, head, k_codes, k_n16, v_codes, v_n16):
    """Write oracle-packed records of tokens 0..T-1 of one sequence/head into the device pools.

    seq_pages: physical page ids of the sequence, in order."""
    import torch

    ps = cache.page_size
    T = k_codes.shape[0]
    krec = packing.pack_k_fast(k_codes)
    vrec = packing.pack_v_fast(v_codes)
    kv_k = cache.k_code_view()
    kv_v = cache.v_code_view()
    kn = cache.k_norm_view()
    vn = cache.v_norm_view()
    for pi in range((T + ps - 1) // ps):
        page = int(seq_pages[pi])
        lo, hi = pi * ps, min(T, (pi + 1) * ps)
        kv_k[layer, page, head, : hi - lo] = torch.from_numpy(krec[lo:hi]).to(kv_k.device)
        blo, bhi = lo // 16, (hi + 15) // 16  # pages hold whole 16-token V blocks
        kv_v[layer, page, head, : bhi - blo] = torch.from_numpy(vrec[blo:bhi]).to(kv_v.device)
        kn[layer, page, head, : hi - lo] = torch.from_numpy(k_n16[lo:hi].view(np.int16)).to(kn.device)
        vn[layer, page, head, : hi - lo] = torch.from_numpy(v_n16[lo:hi].view(np.int16)).to(vn.device)


def max_rel_err(out, ref):
    """Per row: ||o - r||_inf / ||r||_inf; returns the maximum over rows."""
    out = np.asarray(out, dtype=np.float64).reshape(-1, 128)
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, 128)
    den = np.abs(ref).max(axis=1)
    den = np.where(den > 0, den, 1.0)
    return float((np.abs(out - ref).max(axis=1) / den).max())


def oracle_attention(q, k_codes, k_n16, v_codes, v_n16, params):
    return attention.attention_rotated(q, k_codes, k_n16, v_codes, v_n16, params)
