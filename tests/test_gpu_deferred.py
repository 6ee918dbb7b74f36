"""GPU parity of deferred quantisation (iq_decode_step_deferred) against the fp64 oracle: the
prompt's K/V stay fp16, later tokens are packed, the step appends its new token quantised and
attends over both."""

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


def _case(G, lens, ctxs, kb=3, vb=3, rot="iso", ps=64, seed=0):
    """fp16 prefixes and packed tails of several sequences; returns everything the call and the
    oracle need.  The packed pool's positions below each prefix hold other data (they must be
    ignored)."""
    Hkv = 2
    Hq = G * Hkv
    Bn = len(ctxs)
    maxp = (max(ctxs) + ps - 1) // ps
    max_len = max(max(lens), 1)
    P = oracle_params(seed + 5, 1, Hkv, rot)
    table_np = inputs.page_permutation(seed + 2, Bn * maxp).reshape(Bn, maxp)
    cache = B.PagedCache(1, Hkv, ps, Bn * maxp, block_table=torch.from_numpy(table_np).to(DEV), k_bits=kb, v_bits=vb,
                         rotation=rot)
    k16 = np.zeros((Bn, Hkv, max_len, 128), np.float16)
    v16 = np.zeros((Bn, Hkv, max_len, 128), np.float16)
    knew = np.zeros((Bn, Hkv, 128), np.float16)
    vnew = np.zeros((Bn, Hkv, 128), np.float16)
    q = inputs.queries(seed + 7, 0, Bn, Hq)
    refs = []
    for b, (L, T) in enumerate(zip(lens, ctxs)):
        s = 500 + 10 * b + seed
        X = {w: np.stack([inputs.kv_tokens(s, 0, h, w, 0, T) for h in range(Hkv)]) for w in (0, 1)}  # (Hkv, T, 128)
        k16[b, :, :L] = X[0][:, :L]
        v16[b, :, :L] = X[1][:, :L]
        knew[b] = X[0][:, T - 1]
        vnew[b] = X[1][:, T - 1]
        ek = [encode.encode(X[0][h, L:], P[0, h], kb, rot) for h in range(Hkv)]
        ev = [encode.encode(X[1][h, L:], P[0, h], vb, rot) for h in range(Hkv)]
        # packed pool: positions 0 .. T-2; below L other tokens' codes (must be masked)
        junk_k = [encode.encode(inputs.kv_tokens(s + 1, 0, h, 0, 0, L), P[0, h], kb, rot) for h in range(Hkv)]
        junk_v = [encode.encode(inputs.kv_tokens(s + 1, 0, h, 1, 0, L), P[0, h], vb, rot) for h in range(Hkv)]
        for h in range(Hkv):
            kc = np.concatenate([junk_k[h]["codes"], ek[h]["codes"]])[:T - 1]
            kn = np.concatenate([junk_k[h]["norm16"], ek[h]["norm16"]])[:T - 1]
            vc = np.concatenate([junk_v[h]["codes"], ev[h]["codes"]])[:T - 1]
            vn = np.concatenate([junk_v[h]["norm16"], ev[h]["norm16"]])[:T - 1]
            upload_sequence(cache, 0, table_np[b], h, kc, kn, vc, vn)
        refs.append(attention.attention_mixed(
            q[b].astype(np.float64), X[0][:, :L], X[1][:, :L],
            np.stack([e["codes"] for e in ek]), np.stack([e["norm16"] for e in ek]),
            np.stack([e["codes"] for e in ev]), np.stack([e["norm16"] for e in ev]), P[0], kb, vb, rot))
    return cache, P, q, k16, v16, knew, vnew, refs, maxp * ps


def _run(cache, P, q, k16, v16, lens, knew, vnew, ctxs, max_ctx):
    Bn, Hq = q.shape[0], q.shape[1]
    out = Guarded((Bn, Hq, 128), torch.float32, fill=float("nan"))
    ws = Guarded((B.iq_decode_deferred_workspace_size(Bn, Hq, cache.n_kv_heads, max_ctx, k16.shape[2]),), torch.uint8,
                 fill=0)
    B.iq_decode_step_deferred(cache, 0, torch.from_numpy(k16).to(DEV), torch.from_numpy(v16).to(DEV),
                              torch.tensor(lens, dtype=torch.int32, device=DEV), torch.from_numpy(q).to(DEV),
                              torch.from_numpy(knew).to(DEV), torch.from_numpy(vnew).to(DEV),
                              torch.tensor(ctxs, dtype=torch.int32, device=DEV), max_ctx, _pd(P), out.t, ws.t)
    torch.cuda.synchronize()
    out.check("out")
    ws.check("workspace")
    return out.t.cpu().numpy(), ws


@pytest.mark.parametrize("G,kb,vb,rot", [(4, 3, 3, "iso"), (8, 3, 3, "iso"), (8, 4, 3, "iso"), (4, 3, 2, "planar"),
                                         (1, 3, 3, "quat"), (3, 3, 3, "iso"), (5, 3, 3, "iso"), (7, 3, 3, "iso"),
                                         (2, 3, 3, "iso"), (6, 3, 3, "iso")])
def test_deferred_step_matches_oracle(G, kb, vb, rot):
    """Prefixes of 0, 5, 64 (a whole tile) and 300 tokens; contexts 1, 40, 100, 777; the positions
    of the packed pool below each prefix hold other tokens' codes."""
    lens, ctxs = [0, 5, 64, 300], [1, 40, 100, 777]
    cache, P, q, k16, v16, knew, vnew, refs, max_ctx = _case(G, lens, ctxs, kb, vb, rot)
    o, ws = _run(cache, P, q, k16, v16, lens, knew, vnew, ctxs, max_ctx)
    err = max(max_rel_err(o[b], refs[b]) for b in range(len(ctxs)))
    record_parity(f"deferred step K{kb}/V{vb} {rot} (G={G})", max_rel_err=err)
    assert err < TOL, err
    assert cache.status.item() == 0
    # the counters are left at zero: a second call on the same workspace gives the same result
    out2 = torch.empty_like(torch.from_numpy(o)).to(DEV)
    B.iq_decode_step_deferred(cache, 0, torch.from_numpy(k16).to(DEV), torch.from_numpy(v16).to(DEV),
                              torch.tensor(lens, dtype=torch.int32, device=DEV), torch.from_numpy(q).to(DEV),
                              torch.from_numpy(knew).to(DEV), torch.from_numpy(vnew).to(DEV),
                              torch.tensor(ctxs, dtype=torch.int32, device=DEV), max_ctx, _pd(P), out2, ws.t)
    torch.cuda.synchronize()
    assert max(max_rel_err(out2.cpu().numpy()[b], refs[b]) for b in range(len(ctxs))) < TOL


def test_deferred_flags_out_of_range_prefix_length():
    """A prefix length equal to the context length (it must be below: the step's new token is
    packed) or far above the arrays' capacity is clamped and flagged with IQ_DEVERR_CTX; the
    guard bands stay intact and every output is finite."""
    lens, ctxs = [5, 64], [40, 100]
    cache, P, q, k16, v16, knew, vnew, refs, max_ctx = _case(4, lens, ctxs)
    o, ws = _run(cache, P, q, k16, v16, [40, 10**6], knew, vnew, ctxs, max_ctx)
    assert np.isfinite(o).all()
    assert cache.status.item() & B.IQ_DEVERR_CTX


def test_deferred_llama8b_layer_full():
    """The bench's deferred shape: one Llama-3.1-8B-shaped layer (32 q / 8 kv heads), an 8192-token
    fp16 prompt and 512 generated tokens packed (the step appends the last), every head compared."""
    Hq, Hkv, Lp, T = 32, 8, 8192, 8704
    P = oracle_params(inputs.ROTATION_SEED, 1, Hkv)
    cache = B.PagedCache(1, Hkv, T, 1)
    X = {w: np.stack([inputs.kv_tokens(0, 0, h, w, 0, T) for h in range(Hkv)]) for w in (0, 1)}
    ek = [encode.encode(X[0][h, Lp:], P[0, h]) for h in range(Hkv)]
    ev = [encode.encode(X[1][h, Lp:], P[0, h]) for h in range(Hkv)]
    for h in range(Hkv):  # packed tail at positions Lp .. T-2 (the pool's first pages stay unwritten)
        pad = np.zeros((Lp, 128), np.uint8)
        z = np.zeros(Lp, np.uint16)
        upload_sequence(cache, 0, [0], h, np.concatenate([pad, ek[h]["codes"][:-1]]), np.concatenate([z, ek[h]["norm16"][:-1]]),
                        np.concatenate([pad, ev[h]["codes"][:-1]]), np.concatenate([z, ev[h]["norm16"][:-1]]))
    q = inputs.queries(0, 0, 1, Hq)
    k16 = X[0][None, :, :Lp].copy()
    v16 = X[1][None, :, :Lp].copy()
    o, _ = _run(cache, P, q, k16, v16, [Lp], X[0][None, :, T - 1], X[1][None, :, T - 1], [T], T)
    ref = attention.attention_mixed(q[0].astype(np.float64), X[0][:, :Lp], X[1][:, :Lp],
                                    np.stack([e["codes"] for e in ek]), np.stack([e["norm16"] for e in ek]),
                                    np.stack([e["codes"] for e in ev]), np.stack([e["norm16"] for e in ev]), P[0])
    err = max_rel_err(o[0], ref)
    record_parity("deferred step llama8b: 8192 fp16 + 512 packed, full layer", max_rel_err=err)
    assert err < TOL, err
    assert cache.status.item() == 0
