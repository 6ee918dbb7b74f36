"""Shared test utilities: oracle-side encoding of seeded inputs and cache upload."""

import numpy as np

from oracle import attention, encode, packing
from rotated_bit_kv_iq_b200 import inputs


def oracle_encode_stream(params_head, layer, head, which, t0, n, n_outliers=4, heavy_frac=0.0, seed=inputs.DATA_SEED):
    """Seeded fp16 tokens of one (layer, kv head, K|V) stream and their oracle encoding."""
    x = inputs.kv_tokens(seed, layer, head, which, t0, n, n_outliers=n_outliers, heavy_frac=heavy_frac)
    return x, encode.encode(x, params_head)


def upload_sequence(cache, layer, seq_pages, head, k_codes, k_n16, v_codes, v_n16):
    """Write oracle-packed records of tokens 0..T-1 of one sequence/head into the device pool.

    seq_pages: physical page ids of the sequence, in order."""
    import torch

    ps = cache.page_size
    T = k_codes.shape[0]
    krec = torch.from_numpy(packing.pack_k_fast(k_codes))
    vrec = torch.from_numpy(packing.pack_v_fast(v_codes))
    kn = torch.from_numpy(np.asarray(k_n16).view(np.int16).copy())
    vn = torch.from_numpy(np.asarray(v_n16).view(np.int16).copy())
    kv_k, kv_v = cache.k_code_view(), cache.v_code_view()
    k_nv, v_nv = cache.k_norm_view(), cache.v_norm_view()
    for t0 in range(0, T, 32):  # one tile record (32 slots of one page) at a time
        page, slot = int(seq_pages[t0 // ps]), t0 % ps
        tile, m = slot // 32, min(32, T - t0)
        kv_k[layer, page, head, tile, :m] = krec[t0:t0 + m].to(kv_k.device)
        nb = (m + 15) // 16
        kv_v[layer, page, head, tile, :nb] = vrec[t0 // 16:t0 // 16 + nb].to(kv_v.device)
        k_nv[layer, page, head, tile, :m] = kn[t0:t0 + m].to(k_nv.device)
        v_nv[layer, page, head, tile, :m] = vn[t0:t0 + m].to(v_nv.device)


def max_rel_err(out, ref):
    """Per row: ||o - r||_inf / ||r||_inf; returns the maximum over rows."""
    out = np.asarray(out, dtype=np.float64).reshape(-1, 128)
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, 128)
    den = np.abs(ref).max(axis=1)
    den = np.where(den > 0, den, 1.0)
    return float((np.abs(out - ref).max(axis=1) / den).max())


def oracle_attention(q, k_codes, k_n16, v_codes, v_n16, params):
    return attention.attention_rotated(q, k_codes, k_n16, v_codes, v_n16, params)
