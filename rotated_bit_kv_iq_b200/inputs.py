"""Seeded synthetic workloads for the packed-3-bit KV path.

This module only draws random numbers and fixes shapes; it holds none of the
method's arithmetic, so both the CUDA path's callers and the CPU oracle's tests
may use it.

Recipe (one independent substream per (layer, kv head, K|V); PCG64 seeded with a
numpy SeedSequence of integer words):
  * per-channel scale s_c ~ LogNormal(mu=0, sigma=0.5), 128 channels;
  * `n_outliers` channels (without replacement) multiplied by 20;
  * z ~ N(0,1) per coordinate; optionally a fraction of tokens (Bernoulli per
    token) drawn instead from Student-t with 3 degrees of freedom;
  * x = z * s, clamped to +-65504 and rounded to binary16 (round to nearest even).
Tokens are generated in blocks of 1024 from their own substreams, so any token
range can be regenerated without producing the ones before it.
Queries: q ~ N(0,1) per (layer, batch, q head), stored as fp16 (or fp32).

These stand in for K/V activations of real checkpoints (Llama-3.1-8B, Qwen3-30B-A3B
shaped decode); no model weights or evaluation data are used.
"""

import numpy as np

D = 128
BLOCK = 1024
FP16_MAX = 65504.0

# Workload definitions (shapes only).
CONFIGS = {
    "tiny": dict(batch=1, n_q_heads=1, n_kv_heads=1, n_layers=1, ctx=512, q_dtype="f32", n_outliers=2,
                 heavy_frac=0.0, page_size=512),
    "llama8b_8k": dict(batch=1, n_q_heads=32, n_kv_heads=8, n_layers=1, ctx=8192, q_dtype="f16", n_outliers=4,
                       heavy_frac=0.0, page_size=8192),
    "qwen30b_32k": dict(batch=1, n_q_heads=32, n_kv_heads=4, n_layers=48, ctx=32768, q_dtype="f16", n_outliers=4,
                        heavy_frac=0.0, page_size=32768),
    "serve_b16": dict(batch=16, n_q_heads=32, n_kv_heads=8, n_layers=32, ctx_lo=2048, ctx_hi=32768, q_dtype="f16",
                      n_outliers=4, heavy_frac=0.0, page_size=64),
    "ingest_32k": dict(batch=1, n_q_heads=8, n_kv_heads=8, n_layers=32, ctx=32768, q_dtype="f16", n_outliers=4,
                       heavy_frac=0.01, page_size=32768),
}
DATA_SEED = 0
ROTATION_SEED = 1


def _rng(*words):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(w) for w in words])))


def channel_scales(seed, layer, head, which, n_outliers):
    """Per-channel scales of one (layer, kv head, K=0|V=1) stream: (128,) float64."""
    r = _rng(seed, 1, layer, head, which)
    s = r.lognormal(mean=0.0, sigma=0.5, size=D)
    if n_outliers:
        idx = r.choice(D, size=n_outliers, replace=False)
        s[idx] *= 20.0
    return s


def kv_tokens(seed, layer, head, which, t0, n, n_outliers=4, heavy_frac=0.0):
    """Tokens [t0, t0+n) of one (layer, kv head, K|V) stream as float16 (n, 128)."""
    s = channel_scales(seed, layer, head, which, n_outliers)
    out = np.empty((n, D), dtype=np.float16)
    t = t0
    while t < t0 + n:
        blk = t // BLOCK
        r = _rng(seed, 2, layer, head, which, blk)
        z = r.standard_normal((BLOCK, D))
        if heavy_frac > 0.0:
            heavy = r.random(BLOCK) < heavy_frac
            zt = r.standard_t(3.0, size=(BLOCK, D))
            z = np.where(heavy[:, None], zt, z)
        lo = t - blk * BLOCK
        hi = min(BLOCK, t0 + n - blk * BLOCK)
        x = np.clip(z[lo:hi] * s, -FP16_MAX, FP16_MAX)
        out[t - t0 : t - t0 + (hi - lo)] = x.astype(np.float16)
        t += hi - lo
    return out


def queries(seed, layer, batch, n_q_heads, dtype="f16"):
    """Decode queries of one layer: (batch, n_q_heads, 128), fp16 or fp32."""
    r = _rng(seed, 3, layer)
    q = r.standard_normal((batch, n_q_heads, D))
    return q.astype(np.float16 if dtype == "f16" else np.float32)


def context_lengths(seed, batch, lo, hi):
    """Per-sequence context lengths, uniform integers in [lo, hi]."""
    r = _rng(seed, 4)
    return r.integers(lo, hi + 1, size=batch).astype(np.int32)


def page_permutation(seed, n_pages):
    """A random permutation of physical page ids."""
    r = _rng(seed, 5)
    return r.permutation(n_pages).astype(np.int32)


# ------------------------------------------------------------------ device-side generator
def _torch_gen(device, *words):
    import torch

    h = 1469598103934665603
    for w in words:  # FNV-1a over the words -> a 63-bit seed
        h = ((h ^ (int(w) & 0xFFFFFFFF)) * 1099511628211) & 0xFFFFFFFFFFFFFFFF
    return torch.Generator(device=device).manual_seed(h & 0x7FFFFFFFFFFFFFFF)


def kv_tokens_device(seed, layer, n_kv_heads, which, n, n_outliers=4, heavy_frac=0.0, device="cuda"):
    """Same recipe as `kv_tokens`, drawn on the device with torch's generator (a different
    stream): fp16 tensor (n, n_kv_heads, 128).  Used to fill full-size caches quickly; the
    parity tests use the host generator."""
    import torch

    g = _torch_gen(device, seed, 6, layer, which)
    s = torch.exp(0.5 * torch.randn((n_kv_heads, D), generator=g, device=device, dtype=torch.float32))
    if n_outliers:
        for h in range(n_kv_heads):
            idx = torch.randperm(D, generator=g, device=device)[:n_outliers]
            s[h, idx] *= 20.0
    z = torch.randn((n, n_kv_heads, D), generator=g, device=device, dtype=torch.float32)
    if heavy_frac > 0.0:
        heavy = torch.rand((n, 1, 1), generator=g, device=device) < heavy_frac
        chi2 = (torch.randn((n, n_kv_heads, D, 3), generator=g, device=device) ** 2).sum(-1)
        t3 = torch.randn((n, n_kv_heads, D), generator=g, device=device) / torch.sqrt(chi2 / 3.0)
        z = torch.where(heavy, t3, z)
    return torch.clamp(z * s, -FP16_MAX, FP16_MAX).to(torch.float16)


def queries_device(seed, layer, batch, n_q_heads, device="cuda"):
    import torch

    g = _torch_gen(device, seed, 7, layer)
    return torch.randn((batch, n_q_heads, D), generator=g, device=device).to(torch.float16)
