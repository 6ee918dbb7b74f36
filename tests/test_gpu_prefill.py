"""GPU parity of chunked-prefill attention over the packed cache (iq_prefill_attention) against
the fp64 oracle: every query token of the chunk attends causally to its own prefix."""

import numpy as np
import pytest
import torch

from oracle import attention, encode
from rotated_bit_kv_iq_b200 import binding as B
from rotated_bit_kv_iq_b200 import inputs
from tests._helpers import Guarded, max_rel_err, oracle_params, record_parity, upload_sequence

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rotated_bit_kv_iq_b200 import build

    build.build()
    B.lib()


def _pd(P):
    return torch.from_numpy(np.ascontiguousarray(P)).to(DEV)


def _oracle_seq(P_layer, layer, Hkv, T, seed, kb=3, vb=3, rot="iso"):
    kc, kn, vc, vn = [], [], [], []
    for h in range(Hkv):
        ek = encode.encode(inputs.kv_tokens(seed, layer, h, 0, 0, T), P_layer[h], kb, rot)
        ev = encode.encode(inputs.kv_tokens(seed, layer, h, 1, 0, T), P_layer[h], vb, rot)
        kc.append(ek["codes"]); kn.append(ek["norm16"]); vc.append(ev["codes"]); vn.append(ev["norm16"])
    return np.stack(kc), np.stack(kn), np.stack(vc), np.stack(vn)


def _prefill(cache, q, start, max_ctx, P):
    Bn, C, Hq = q.shape[0], q.shape[1], q.shape[2]
    out = Guarded((Bn, C, Hq, 128), torch.float32, fill=float("nan"))
    ws = Guarded((B.iq_prefill_workspace_size(Bn, C, cache.n_kv_heads, max_ctx),), torch.uint8)
    B.iq_prefill_attention(cache, 0, torch.from_numpy(q).to(DEV), torch.tensor(start, dtype=torch.int32, device=DEV),
                           max_ctx, _pd(P), out.t, ws.t)
    torch.cuda.synchronize()
    out.check("out")
    ws.check("workspace")
    return out.t.cpu().numpy()


@pytest.mark.parametrize("kb,vb,rot,G", [(3, 3, "iso", 4), (3, 3, "iso", 8), (3, 3, "iso", 1), (4, 3, "iso", 8),
                                         (3, 2, "planar", 4), (3, 3, "quat", 2), (3, 3, "iso", 3),
                                         (3, 3, "iso", 6), (2, 2, "iso", 4), (4, 4, "iso", 5),
                                         (4, 2, "quat", 7)])
def test_prefill_ragged_chunks_match_oracle(kb, vb, rot, G):
    """Two sequences with different prefixes (0 and 300 tokens) and a 37-token chunk (a ragged last
    block of query tokens) over shuffled 64-token pages; every query token compared."""
    Hkv = 2
    Hq = G * Hkv
    starts, C, ps, maxp = [0, 300], 37, 64, 6
    P = oracle_params(9, 1, Hkv, rot)
    table_np = inputs.page_permutation(4, 2 * maxp).reshape(2, maxp)
    cache = B.PagedCache(1, Hkv, ps, 2 * maxp, block_table=torch.from_numpy(table_np).to(DEV), k_bits=kb, v_bits=vb,
                         rotation=rot)
    q = np.stack([inputs.queries(20 + b, 0, C, Hq) for b in range(2)])  # [batch][C][Hq][128]
    refs = []
    for b, s0 in enumerate(starts):
        kc, kn, vc, vn = _oracle_seq(P[0], 0, Hkv, s0 + C, 70 + b, kb, vb, rot)
        for h in range(Hkv):
            upload_sequence(cache, 0, table_np[b], h, kc[h], kn[h], vc[h], vn[h])
        refs.append(attention.prefill_attention(q[b].astype(np.float64), kc, kn, vc, vn, P[0], s0, kb, vb, rot))
    o = _prefill(cache, q, starts, maxp * ps, P)
    err = max(max_rel_err(o[b], refs[b]) for b in range(2))
    record_parity(f"prefill ragged chunks K{kb}/V{vb} {rot} (G={G})", max_rel_err=err)
    assert err < TOL, err
    assert cache.status.item() == 0


def test_prefill_llama8b_chunk_sampled():
    """The bench's prefill shape: a 512-token chunk at prefix 7680 of a Llama-3.1-8B-shaped layer
    (32 q / 8 kv heads, contiguous 8192-token cache); 16 sampled query tokens of every head."""
    Hq, Hkv, T, C = 32, 8, 8192, 512
    s0 = T - C
    P = oracle_params(inputs.ROTATION_SEED, 1, Hkv)
    cache = B.PagedCache(1, Hkv, T, 1)
    kc, kn, vc, vn = _oracle_seq(P[0], 0, Hkv, T, 0)
    for h in range(Hkv):
        upload_sequence(cache, 0, [0], h, kc[h], kn[h], vc[h], vn[h])
    q = inputs.queries(5, 0, C, Hq)[None]
    o = _prefill(cache, q, [s0], T, P)
    sample = np.unique(np.concatenate([np.arange(0, C, 37), [C - 1, 7, 8]]))
    err = 0.0
    for i in sample:
        ref = attention.attention_rotated(q[0, i].astype(np.float64), kc[:, :s0 + i + 1], kn[:, :s0 + i + 1],
                                          vc[:, :s0 + i + 1], vn[:, :s0 + i + 1], P[0])
        err = max(err, max_rel_err(o[0, i], ref))
    record_parity("prefill llama8b 512-token chunk at 7680, 17 sampled tokens", max_rel_err=err)
    assert err < TOL, err
    assert np.isfinite(o).all()


def test_prefill_after_gpu_encode_end_to_end():
    """The chunk's K/V are appended by iq_encode_append (GPU), then iq_prefill_attention runs over
    prefix + chunk; against the oracle's own encoding and causal attention."""
    Hq, Hkv, s0, C = 16, 2, 200, 64
    T = s0 + C
    P = oracle_params(2, 1, Hkv)
    cache = B.PagedCache(1, Hkv, 320, 1)
    X = {w: np.stack([inputs.kv_tokens(33, 0, h, w, 0, T) for h in range(Hkv)], axis=1)[None] for w in (0, 1)}
    zero = torch.zeros(1, dtype=torch.int32, device=DEV)
    B.iq_encode_append(cache, 0, torch.from_numpy(X[0][:, :s0]).to(DEV), torch.from_numpy(X[1][:, :s0]).to(DEV), zero,
                       _pd(P))
    B.iq_encode_append(cache, 0, torch.from_numpy(X[0][:, s0:].copy()).to(DEV),
                       torch.from_numpy(X[1][:, s0:].copy()).to(DEV), torch.full((1,), s0, dtype=torch.int32,
                                                                                device=DEV), _pd(P))
    q = inputs.queries(34, 0, C, Hq)[None]
    o = _prefill(cache, q, [s0], T, P)
    enc = {w: [encode.encode(X[w][0, :, h], P[0, h]) for h in range(Hkv)] for w in (0, 1)}
    ref = attention.prefill_attention(
        q[0].astype(np.float64), np.stack([e["codes"] for e in enc[0]]), np.stack([e["norm16"] for e in enc[0]]),
        np.stack([e["codes"] for e in enc[1]]), np.stack([e["norm16"] for e in enc[1]]), P[0], s0)
    err = max_rel_err(o[0], ref)
    record_parity("GPU encode -> GPU prefill vs oracle (64-token chunk)", max_rel_err=err)
    assert err < TOL, err
