"""Decode attention over the packed cache (oracle, fp64), written two ways.

[TQ-RQ] section "为什么压缩 KV 缓存这么难？": attention is softmax(Q K^T / sqrt(d)) V.
[RQ-news] section "妙处不只是压缩，而是不再展开" and [RQ-abs]: the packed pipeline
scores the query against the packed keys, runs softmax, accumulates the packed
values, and applies the inverse rotation last, never building full-precision K/V.
[RQ-wiki] section "3. V 缓存的逆旋转修复": values must be mapped back with the
inverse of the forward rotation.

Because the encoder stores x ~ n * R^T c~[codes] (c~ = Lloyd–Max centroids of
N(0, 1/d)), the method computes exactly (up to rounding order) ordinary attention
on the dequantised cache
    K_hat_t = n_k,t R^T c~[codes_k,t],   V_hat_t = n_v,t R^T c~[codes_v,t],
with n the stored binary16 norms.  `attention_dequant` is that definition written
out; `attention_rotated` follows the packed pipeline's order (rotate q once, score
in the rotated basis, softmax, accumulate in the rotated basis, rotate back once).
They must agree to ~1e-10.

GQA (q heads sharing a kv head): q head h reads kv head h // G, G = Hq / Hkv.
An empty context (ctx = 0) yields a zero output vector (the pages are silent).
K and V may use different codebook widths ([TQ-RQ] section "K 和 V 的非对称需求": keys need
more bits than values) and any rotation variant of oracle.rotation.
"""

import math

import numpy as np

from .codebook import codebook_for_dim
from .encode import fp16_bits_to_float
from .rotation import rotate, rotate_inverse

D = 128


def dequantise(codes, norm16, params_head, bits=3, variant="iso"):
    """Explicit fp64 vectors n * R^T c~[codes] for one kv head: (T, 128)."""
    ct, _ = codebook_for_dim(D, bits)
    n = fp16_bits_to_float(norm16)
    return n[:, None] * rotate_inverse(ct[np.asarray(codes, dtype=np.int64)], params_head, variant)


def attention_dequant(q, k_codes, k_norm16, v_codes, v_norm16, params, bits=3, v_bits=None, variant="iso"):
    """Plain softmax attention on the explicitly dequantised cache.

    q: (Hq, 128); k_codes/v_codes: (Hkv, T, 128); k_norm16/v_norm16: (Hkv, T);
    params: (Hkv, ...) per-head rotation parameters.  bits: K codebook width; v_bits: V width
    (default: bits).  Returns (Hq, 128) fp64.
    """
    v_bits = bits if v_bits is None else v_bits
    q = np.asarray(q, dtype=np.float64)
    Hq = q.shape[0]
    Hkv, T = np.asarray(k_codes).shape[:2]
    G = Hq // Hkv
    out = np.zeros((Hq, D))
    if T == 0:
        return out
    for kv in range(Hkv):
        Kh = dequantise(k_codes[kv], k_norm16[kv], params[kv], bits, variant)
        Vh = dequantise(v_codes[kv], v_norm16[kv], params[kv], v_bits, variant)
        for h in range(kv * G, (kv + 1) * G):
            s = Kh @ q[h] / math.sqrt(D)
            p = np.exp(s - s.max())
            out[h] = (p / p.sum()) @ Vh
    return out


def attention_rotated(q, k_codes, k_norm16, v_codes, v_norm16, params, bits=3, v_bits=None, variant="iso"):
    """The packed pipeline's order: same inputs and output as `attention_dequant`."""
    v_bits = bits if v_bits is None else v_bits
    q = np.asarray(q, dtype=np.float64)
    Hq = q.shape[0]
    Hkv, T = np.asarray(k_codes).shape[:2]
    G = Hq // Hkv
    ct_k, _ = codebook_for_dim(D, bits)
    ct_v, _ = codebook_for_dim(D, v_bits)
    out = np.zeros((Hq, D))
    if T == 0:
        return out
    for kv in range(Hkv):
        nk = fp16_bits_to_float(k_norm16[kv])
        nv = fp16_bits_to_float(v_norm16[kv])
        Ck = ct_k[np.asarray(k_codes[kv], dtype=np.int64)]  # (T, 128) rotated-basis keys (unit scale)
        Cv = ct_v[np.asarray(v_codes[kv], dtype=np.int64)]
        for h in range(kv * G, (kv + 1) * G):
            q_r = rotate(q[h], params[kv], variant)  # rotate the query once
            s = nk * (Ck @ q_r) / math.sqrt(D)  # scores straight from codes and norms
            p = np.exp(s - s.max())
            acc = (p * nv) @ Cv  # accumulate values in the rotated basis
            out[h] = rotate_inverse(acc / p.sum(), params[kv], variant)  # one inverse rotation per output
    return out


def prefill_attention(q, k_codes, k_norm16, v_codes, v_norm16, params, start, bits=3, v_bits=None, variant="iso"):
    """Chunked prefill on the packed cache: q (n_tok, Hq, 128) are the queries of tokens at
    positions start .. start + n_tok - 1 of one sequence; query token i attends to cache
    positions 0 .. start + i (causal).  k_codes etc. hold at least start + n_tok positions.
    Each query token is one decode-attention problem over its own prefix.  Returns
    (n_tok, Hq, 128) fp64."""
    q = np.asarray(q, dtype=np.float64)
    out = np.zeros(q.shape)
    for i in range(q.shape[0]):
        T = start + i + 1
        out[i] = attention_rotated(q[i], k_codes[:, :T], k_norm16[:, :T], v_codes[:, :T], v_norm16[:, :T], params,
                                   bits, v_bits, variant)
    return out


def attention_mixed(q, k16_prefix, v16_prefix, k_codes, k_norm16, v_codes, v_norm16, params, bits=3, v_bits=None,
                    variant="iso"):
    """Deferred quantisation ("RotorQuant" sd114.wiki section "2. 延迟量化策略"; [TQ-RQ] section
    "延迟量化（Deferred Quantization）"): the prompt's K/V are kept in fp16 and only later tokens
    are quantised.  Attention over positions 0 .. P-1 held as fp16 vectors (k16_prefix,
    v16_prefix: (Hkv, P, 128)) followed by packed positions P .. T-1 (k_codes etc.: (Hkv, T-P,
    ...)): plain softmax attention over the concatenation of the fp16 keys and values, promoted
    to fp64, and the dequantised packed ones.  Returns (Hq, 128) fp64."""
    v_bits = bits if v_bits is None else v_bits
    q = np.asarray(q, dtype=np.float64)
    Hq = q.shape[0]
    Hkv = np.asarray(k16_prefix).shape[0]
    G = Hq // Hkv
    out = np.zeros((Hq, D))
    for kv in range(Hkv):
        K = np.concatenate([np.asarray(k16_prefix[kv], dtype=np.float16).astype(np.float64),
                            dequantise(k_codes[kv], k_norm16[kv], params[kv], bits, variant)])
        V = np.concatenate([np.asarray(v16_prefix[kv], dtype=np.float16).astype(np.float64),
                            dequantise(v_codes[kv], v_norm16[kv], params[kv], v_bits, variant)])
        if K.shape[0] == 0:
            continue
        for h in range(kv * G, (kv + 1) * G):
            s = K @ q[h] / math.sqrt(D)
            p = np.exp(s - s.max())
            out[h] = (p / p.sum()) @ V
    return out
