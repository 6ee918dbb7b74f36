"""Benchmark of the packed-3-bit KV path on B200 (one JSON line on rank 0).

Headline workload (qwen30b_32k): one decode step of a Qwen3-30B-A3B-shaped stack -- batch 1,
32 query / 4 kv heads, d = 128, 48 layers back to back, context 32768.  A step appends the
new token's K and V to every layer's packed cache (encode) and runs decode attention over
the 32768 cached tokens of every layer; the 48 layers are replayed as one CUDA graph.
value = algorithmic packed-KV bytes of the step / step time (GB/s); the step reads 629 MB
of packed cache, far more than L2, so no flush is needed between steps.

Also reported: the ingest workload (quantise-and-append 32768 tokens x 8 kv heads x 32
layers of K and V, 16.8 M vectors: encode Mvec/s and GB/s) and the batched serving workload
(16 paged sequences, contexts in [2048, 32768], 32 layers).

--impl reference times the fp64 CPU oracle on a bounded sample of the headline workload.
"""

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

BYTES_PER_TOKEN_HEAD = 100  # 48 B K codes + 2 B K norm + 48 B V codes + 2 B V norm
BYTES_PER_VECTOR_ENCODE = 306  # 256 B fp16 in + 48 B codes + 2 B norm out
# DRAM bytes (read + write) of one decode_kernel launch of the headline layer and of the serving
# layer, from ncu captures (dram__bytes_read.sum + dram__bytes_write.sum), valid only for the
# kernel sources they were taken on: reported as roofline.traffic while their code hash matches.
DECODE_SOURCES = ["rotated_bit_kv_iq_b200/csrc/iq_decode_impl.cuh", "rotated_bit_kv_iq_b200/csrc/iq_decode.cu",
                  "rotated_bit_kv_iq_b200/csrc/iq_decode_k3v3.cu", "rotated_bit_kv_iq_b200/csrc/iq_device.cuh",
                  "rotated_bit_kv_iq_b200/csrc/iq_internal.h", "include/iq.h"]
DECODE_TRAFFIC = {"sources": DECODE_SOURCES, "sha256": "7ba6ae650784f6e0ba812196dc3e845d881487cb82b12c68bbeb3366c0018506", "bytes": 13245696}
SERVING_TRAFFIC = {"sources": DECODE_SOURCES, "sha256": "7ba6ae650784f6e0ba812196dc3e845d881487cb82b12c68bbeb3366c0018506", "bytes": 235564544 + 6204160}
# DRAM bytes of one encode_kernel launch of the ingest layer (one-pass capture; the records still
# in L2 at kernel end are not counted as written)
ENCODE_SOURCES = ["rotated_bit_kv_iq_b200/csrc/iq_encode.cu", "rotated_bit_kv_iq_b200/csrc/iq_device.cuh",
                  "rotated_bit_kv_iq_b200/csrc/iq_internal.h", "include/iq.h"]
ENCODE_TRAFFIC = {"sources": ENCODE_SOURCES, "sha256": "1a281353eb9deaa2c5eff367972e97a7d2d4016b02a1136dfe08f033120b9e9c", "bytes": 134295296 + 12922368}


def kernel_source_hash(paths):
    """SHA-256 of the code in the given C/C++/CUDA sources, comments and blank space removed
    (a comment edit does not change the kernel the counters were taken on)."""
    import hashlib
    import re

    h = hashlib.sha256()
    here = os.path.dirname(os.path.abspath(__file__))
    for f in paths:
        with open(os.path.join(here, f), encoding="utf-8") as fh:
            txt = fh.read()
        txt = re.sub(r"/\*.*?\*/", " ", txt, flags=re.S)
        txt = re.sub(r"//[^\n]*", " ", txt)
        h.update(" ".join(txt.split()).encode())
    return h.hexdigest()


def decode_traffic(rec=None):
    """Captured DRAM bytes per launch of a kernel, or None once its sources have changed."""
    rec = rec or DECODE_TRAFFIC
    try:
        digest = kernel_source_hash(rec["sources"])
    except OSError:
        return None
    return rec["bytes"] if digest == rec["sha256"] else None


HEADLINE = "qwen30b_32k"
METRIC = "packed-KV decode attention GB/s & % HBM peak at 32K ctx; encode Mvec/s"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples (200 ms) of the SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[2:6]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ workloads
class DecodeStack:
    """Packed caches of an L-layer stack, filled by the library's own encoder."""

    def __init__(self, B, Hq, Hkv, L, ctx, page_size, device, seed=0, block_table=None, n_pages=None):
        import torch

        from rotated_bit_kv_iq_b200 import binding as Bd
        from rotated_bit_kv_iq_b200 import inputs

        self.Bd, self.torch = Bd, torch
        self.B, self.Hq, self.Hkv, self.L = B, Hq, Hkv, L
        self.ctx = np.asarray(ctx, dtype=np.int32)
        self.max_ctx = int(self.ctx.max())
        self.dev = device
        n_pages = n_pages if n_pages is not None else B
        self.cache = Bd.PagedCache(L, Hkv, page_size, n_pages, block_table=block_table, device=device)
        self.params = torch.from_numpy(Bd.iq_init_rotation(inputs.ROTATION_SEED, L, Hkv)).to(device)
        # prefill: tokens 0..ctx-2 of every sequence and layer, encoded by iq_encode_append
        pre = self.ctx - 1
        n_max = int(pre.max())
        start = torch.zeros(B, dtype=torch.int32, device=device)
        for l in range(L):
            k = inputs.kv_tokens_device(seed, l, Hkv, 0, n_max * B, device=device).view(B, n_max, Hkv, 128)
            v = inputs.kv_tokens_device(seed, l, Hkv, 1, n_max * B, device=device).view(B, n_max, Hkv, 128)
            Bd.iq_encode_append(self.cache, l, k, v, start, self.params)
        # the step's inputs: the new token (position ctx-1) and the queries, per layer
        self.new_pos = torch.from_numpy(pre).to(device)
        self.ctx_dev = torch.from_numpy(self.ctx).to(device)
        self.knew = torch.stack([inputs.kv_tokens_device(seed + 1, l, Hkv, 0, B, device=device) for l in range(L)]).view(
            L, B, 1, Hkv, 128)
        self.vnew = torch.stack([inputs.kv_tokens_device(seed + 1, l, Hkv, 1, B, device=device) for l in range(L)]).view(
            L, B, 1, Hkv, 128)
        self.q = torch.stack([inputs.queries_device(seed, l, B, Hq, device=device) for l in range(L)])
        self.out = torch.empty((L, B, Hq, 128), dtype=torch.float32, device=device)
        self.ws = torch.zeros(Bd.iq_decode_workspace_size(B, Hq, Hkv, self.max_ctx), dtype=torch.uint8, device=device)
        torch.cuda.synchronize()

    @property
    def bytes_per_step(self):
        return int(self.ctx.sum()) * self.Hkv * self.L * BYTES_PER_TOKEN_HEAD + \
            self.B * self.Hkv * 2 * self.L * BYTES_PER_VECTOR_ENCODE

    def layer(self, l, stream=None):
        """One layer of the decode step: append the new token and attend (iq_decode_step)."""
        self.Bd.iq_decode_step(self.cache, l, self.q[l], self.knew[l], self.vnew[l], self.ctx_dev, self.max_ctx,
                               self.params, self.out[l], self.ws, stream)

    def step(self, stream=None):
        for l in range(self.L):
            self.layer(l, stream)

    launches_per_layer = 1  # one kernel: append, split attention, merge and inverse rotation


def time_graph(stack, steps, warmup, stream):
    """Replay the whole step as one CUDA graph; device time per step via events."""
    torch = stack.torch
    with torch.cuda.stream(stream):
        for _ in range(max(1, warmup)):
            stack.step(stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        stack.step(stream)
    # replay() launches on torch's current stream: make it the timed stream
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
        e1.synchronize()
    return e0.elapsed_time(e1) / steps, graph


def time_e2e(stack, steps, warmup, stream):
    """Same step through the public API with host buffers: every step copies the new K/V and
    the queries of all layers from pinned host memory (one copy per tensor), runs the
    layers' iq_decode_step calls and copies all attention outputs back to pinned host memory.
    Returned twice: with the layers' calls captured once as a CUDA graph (like the device-timed
    step), and with every call made through the C ABI each step (host marshalling and argument
    checks of 48 calls inside the timed region)."""
    torch = stack.torch
    hk = stack.knew.cpu().pin_memory()
    hv = stack.vnew.cpu().pin_memory()
    hq = stack.q.cpu().pin_memory()
    ho = torch.empty(stack.out.shape, dtype=torch.float32).pin_memory()
    dk, dv, dq = torch.empty_like(stack.knew), torch.empty_like(stack.vnew), torch.empty_like(stack.q)
    dout = torch.empty_like(stack.out)
    Bd = stack.Bd

    def layers():
        for l in range(stack.L):
            Bd.iq_decode_step(stack.cache, l, dq[l], dk[l], dv[l], stack.ctx_dev, stack.max_ctx, stack.params,
                              dout[l], stack.ws, stream)

    def timed(step):
        for _ in range(max(1, warmup)):
            step()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / steps

    with torch.cuda.stream(stream):
        layers()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            layers()

        def copy_in():
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            dq.copy_(hq, non_blocking=True)

        def step_graph():
            copy_in()
            graph.replay()
            ho.copy_(dout, non_blocking=True)

        def step_direct():
            copy_in()
            layers()
            ho.copy_(dout, non_blocking=True)

        ms = timed(step_graph)
        ms_direct = timed(step_direct)
    del graph
    h2d = hk.numel() * 2 + hv.numel() * 2 + hq.numel() * 2
    d2h = ho.numel() * 4
    return ms, ms_direct, h2d, d2h


def bench_encode(steps, warmup, device, stream):
    """Ingest workload: 32 layers x (32768 tokens x 8 kv heads) of K and V per step."""
    import torch

    from rotated_bit_kv_iq_b200 import binding as Bd
    from rotated_bit_kv_iq_b200 import inputs

    L, Hkv, T = 32, 8, 32768
    cache = Bd.PagedCache(L, Hkv, T, 1, device=device)
    params = torch.from_numpy(Bd.iq_init_rotation(inputs.ROTATION_SEED, L, Hkv)).to(device)
    K = [inputs.kv_tokens_device(0, l, Hkv, 0, T, heavy_frac=0.01, device=device).view(1, T, Hkv, 128) for l in range(L)]
    V = [inputs.kv_tokens_device(0, l, Hkv, 1, T, heavy_frac=0.01, device=device).view(1, T, Hkv, 128) for l in range(L)]
    start = torch.zeros(1, dtype=torch.int32, device=device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(L)]
    with torch.cuda.stream(stream):
        for _ in range(max(1, warmup)):
            for l in range(L):
                Bd.iq_encode_append(cache, l, K[l], V[l], start, params, stream)
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            for l in range(L):
                Bd.iq_encode_append(cache, l, K[l], V[l], start, params, stream)
        e1.record(stream)
        e1.synchronize()
        step_ms = e0.elapsed_time(e1) / steps
        tot = 0.0
        for _ in range(steps):
            for l in range(L):
                evs[l][0].record(stream)
                Bd.iq_encode_append(cache, l, K[l], V[l], start, params, stream)
                evs[l][1].record(stream)
            stream.synchronize()
            tot += sum(a.elapsed_time(b) for a, b in evs)
    launch_ms = tot / (steps * L)
    vecs = L * T * Hkv * 2
    return {"vectors_per_step": vecs, "ms_per_step": step_ms, "launch_ms": launch_ms,
            "bytes_per_launch": T * Hkv * 2 * BYTES_PER_VECTOR_ENCODE}


def bench_prefill(steps, warmup, device, stream, world=1):
    """Chunked prefill of one Llama-3.1-8B-shaped layer (32 q / 8 kv heads): an 8192-token prompt
    in 16 chunks of 512; each chunk appends its K/V (iq_encode_append) and attends causally over the
    packed cache (iq_prefill_attention).  The 48 launches of a step are replayed as one CUDA graph."""
    import torch

    from rotated_bit_kv_iq_b200 import binding as Bd
    from rotated_bit_kv_iq_b200 import inputs

    Hq, Hkv, T, C = 32, 8, 8192, 512
    cache = Bd.PagedCache(1, Hkv, T, 1, device=device)
    params = torch.from_numpy(Bd.iq_init_rotation(inputs.ROTATION_SEED, 1, Hkv)).to(device)
    K = inputs.kv_tokens_device(0, 0, Hkv, 0, T, device=device).view(1, T, Hkv, 128)
    V = inputs.kv_tokens_device(0, 0, Hkv, 1, T, device=device).view(1, T, Hkv, 128)
    g = inputs._torch_gen(device, 0, 8)
    q = torch.randn((1, T, Hq, 128), generator=g, device=device).to(torch.float16)
    out = torch.empty((1, T, Hq, 128), dtype=torch.float32, device=device)
    ws = torch.empty(Bd.iq_prefill_workspace_size(1, C, Hkv, T), dtype=torch.uint8, device=device)
    starts = [torch.full((1,), c, dtype=torch.int32, device=device) for c in range(0, T, C)]
    chunks = [(K[:, c:c + C].contiguous(), V[:, c:c + C].contiguous(), q[:, c:c + C].contiguous()) for c in range(0, T, C)]
    outs = [torch.empty((1, C, Hq, 128), dtype=torch.float32, device=device) for _ in chunks]

    def step():
        for (k, v, qq), st, o in zip(chunks, starts, outs):
            Bd.iq_encode_append(cache, 0, k, v, st, params, stream)
            Bd.iq_prefill_attention(cache, 0, qq, st, T, params, o, ws, stream)

    with torch.cuda.stream(stream):
        for _ in range(max(1, warmup)):
            step()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        for _ in range(warmup):
            graph.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
        e1.synchronize()
        # the attention calls alone (prefill kernel + split merge), chunk by chunk, outside the graph
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in chunks]
        for (k, v, qq), st, o in zip(chunks, starts, outs):
            Bd.iq_encode_append(cache, 0, k, v, st, params, stream)
        for _ in range(steps):
            for (k, v, qq), st, o, ev in zip(chunks, starts, outs, evs):
                ev[0].record(stream)
                Bd.iq_prefill_attention(cache, 0, qq, st, T, params, o, ws, stream)
                ev[1].record(stream)
        stream.synchronize()
        att_ms = sum(a.elapsed_time(b) for a, b in evs)  # the last step's 16 calls
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, device)
    att_ms = max_over_ranks(att_ms, device)
    del graph
    # algorithmic attention work: query token at position p reads p + 1 keys; 2 flops per
    # multiply-add, 2 x 128 multiply-adds per (query head, key) for scores and values
    flops = sum(p + 1 for p in range(T)) * Hq * 4 * 128
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16 = float(json.load(f)["bf16_tflops"])
        peak_kind = "measured bf16 (binary16 operands run at the bf16 rate)"
    except Exception:
        bf16, peak_kind = 1590.0, "fallback bf16 (binary16 operands run at the bf16 rate)"
    ach = flops / (att_ms * 1e-3) / 1e12
    return {"workload": "llama8b_prefill_8k: one layer, 32 q / 8 kv heads, 8192-token prompt in 16 chunks of 512 "
                        "(append + causal attention over the packed cache per chunk)",
            "value": world * T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "dtype": "binary16 hi/lo operands on tcgen05 (three products per contraction), fp32 accumulation",
            "roofline": {"bound": "tensor", "achieved": ach, "peak": bf16, "unit": "TFLOP/s",
                         "frac": ach / bf16, "traffic": None, "peak_kind": peak_kind,
                         "kernel": "prefill attention (prefill_kernel + prefill_merge_kernel) of the 16 chunks, "
                                   "algorithmic flops (4 x 128 per query head and key) / their CUDA-event time",
                         "attention_ms_per_step": att_ms},
            "launches": 48 * steps}


def bench_deferred(steps, warmup, device, stream, world=1, n_layers=32):
    """Deferred quantisation on a Llama-3.1-8B-shaped stack (32 layers, 32 q / 8 kv heads): the
    8192-token prompt stays fp16, 512 generated tokens are packed; one decode step appends the
    next token (quantised) and attends over fp16 prefix + packed tail in every layer
    (iq_decode_step_deferred), replayed as one CUDA graph."""
    import torch

    from rotated_bit_kv_iq_b200 import binding as Bd
    from rotated_bit_kv_iq_b200 import inputs

    Hq, Hkv, Lp, T = 32, 8, 8192, 8704
    L = n_layers
    cache = Bd.PagedCache(L, Hkv, T, 1, device=device)
    params = torch.from_numpy(Bd.iq_init_rotation(inputs.ROTATION_SEED, L, Hkv)).to(device)
    k16, v16, qs, kn, vn = [], [], [], [], []
    start = torch.full((1,), Lp, dtype=torch.int32, device=device)
    for l in range(L):
        K = inputs.kv_tokens_device(0, l, Hkv, 0, T, device=device)  # (T, Hkv, 128)
        V = inputs.kv_tokens_device(0, l, Hkv, 1, T, device=device)
        k16.append(K[:Lp].permute(1, 0, 2).contiguous()[None])
        v16.append(V[:Lp].permute(1, 0, 2).contiguous()[None])
        Bd.iq_encode_append(cache, l, K[Lp:T - 1][None].contiguous(), V[Lp:T - 1][None].contiguous(), start, params,
                            stream)
        kn.append(K[T - 1][None].contiguous())
        vn.append(V[T - 1][None].contiguous())
        qs.append(inputs.queries_device(0, l, 1, Hq, device=device))
    torch.cuda.synchronize()
    plen = torch.full((1,), Lp, dtype=torch.int32, device=device)
    ctx = torch.full((1,), T, dtype=torch.int32, device=device)
    out = torch.empty((L, 1, Hq, 128), dtype=torch.float32, device=device)
    ws = torch.zeros(Bd.iq_decode_deferred_workspace_size(1, Hq, Hkv, T, Lp), dtype=torch.uint8, device=device)

    def step():
        for l in range(L):
            Bd.iq_decode_step_deferred(cache, l, k16[l], v16[l], plen, qs[l], kn[l], vn[l], ctx, T, params, out[l], ws,
                                       stream)

    with torch.cuda.stream(stream):
        for _ in range(max(1, warmup)):
            step()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        for _ in range(warmup):
            graph.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
        e1.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, device)
    del graph
    layer_bytes = Hkv * (Lp * 2 * 256 + (T - Lp) * BYTES_PER_TOKEN_HEAD)  # fp16 K+V prefix, packed tail
    peak, peak_kind = _peaks()
    kern_ms = ms / L
    ach = layer_bytes / (kern_ms * 1e-3) / 1e9
    return {"workload": f"llama8b_deferred: {L} layers, 32 q / 8 kv heads, 8192-token fp16 prompt + 512 packed "
                        "tokens, decode step appending the next token (deferred quantisation)",
            "value": world * layer_bytes * L / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms,
            "us_per_layer": kern_ms * 1e3,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                         "traffic": None, "peak_kind": peak_kind, "bytes_per_launch": layer_bytes,
                         "kernel": "prefix_kernel + decode_kernel per layer, CUDA-graph step time / layers"},
            "launches": 2 * L * steps}


def max_over_ranks(x, device=None):
    """Max of a float over the ranks of the default process group (x itself without one).
    Every timed quantity of a multi-rank run goes through this, so that the job's time is
    that of its slowest rank."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world, bytes_per_rank_step, ms):
    """Whole-job rate: every rank moves bytes_per_rank_step per step; ms is the max over ranks."""
    return world * bytes_per_rank_step / (ms * 1e-3) / 1e9


def bench_serving(steps, warmup, device, stream, seed=0, world=1, n_layers=0):
    """Batched serving workload: one decode step of a 32-layer stack for 16 sequences with
    seeded contexts uniform in [2048, 32768], 64-token pages in a shuffled pool, 32 q / 8 kv
    heads; replayed as one CUDA graph."""
    import torch

    from rotated_bit_kv_iq_b200 import inputs

    cfg = inputs.CONFIGS["serve_b16"]
    B, ps = cfg["batch"], cfg["page_size"]
    ctx = inputs.context_lengths(inputs.DATA_SEED, B, cfg["ctx_lo"], cfg["ctx_hi"])
    maxp = (int(ctx.max()) + ps - 1) // ps
    table = torch.from_numpy(inputs.page_permutation(inputs.DATA_SEED, B * maxp).reshape(B, maxp)).to(device)
    stack = DecodeStack(B, cfg["n_q_heads"], cfg["n_kv_heads"], n_layers or cfg["n_layers"], ctx, ps, device,
                        seed=seed, block_table=table, n_pages=B * maxp)
    ms, graph = time_graph(stack, steps, warmup, stream)
    del graph
    ms = max_over_ranks(ms, device)
    peak, peak_kind = _peaks()
    layer_bytes = int(stack.ctx.sum()) * stack.Hkv * BYTES_PER_TOKEN_HEAD
    kern_ms = ms / stack.L
    achieved = layer_bytes / (kern_ms * 1e-3) / 1e9
    out = {
        "workload": f"serve_b16: decode step of 16 paged sequences (contexts {int(ctx.min())}..{int(ctx.max())}, "
                    f"sum {int(ctx.sum())}), 32 q / 8 kv heads, d=128, {stack.L} layers, 64-token pages",
        "value": job_gbs(world, stack.bytes_per_step, ms), "unit": "GB/s", "ms_per_step": ms,
        "bytes_per_step": stack.bytes_per_step,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": decode_traffic(SERVING_TRAFFIC), "kernel": "decode_kernel, CUDA-graph step time / layers",
                     "peak_kind": peak_kind, "bytes_per_launch": layer_bytes, "launch_ms": kern_ms},
        "launches": stack.L * DecodeStack.launches_per_layer * steps,
    }
    del stack
    return out


# ------------------------------------------------------------------ oracle baseline
def _cpu_info():
    """CPU model and the cores this process may run on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        affinity = len(os.sched_getaffinity(0))
    except AttributeError:
        affinity = os.cpu_count()
    return model, affinity


def oracle_decode_sample(seconds=12.0):
    """fp64 oracle decode attention on slices of the headline workload (one kv head, 8 query
    heads, 32768 tokens per slice) until about `seconds` of CPU time; returns GB/s.  The oracle
    draws its own rotation parameters and encodes the host generator's tokens itself."""
    from oracle import attention, encode, rotation
    from rotated_bit_kv_iq_b200 import inputs

    T, G = 32768, 8
    P = rotation.init_rotation(inputs.ROTATION_SEED, 1, 4)
    slices = []
    for h in range(2):  # encode outside the timed part
        ek = encode.encode(inputs.kv_tokens(0, 0, h, 0, 0, T), P[0, h])
        ev = encode.encode(inputs.kv_tokens(0, 0, h, 1, 0, T), P[0, h])
        slices.append((h, ek, ev))
    q = inputs.queries(0, 0, 1, 32)[0].astype(np.float64)
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=1):  # one core: the figure reported as `cores`
        t0 = time.perf_counter()
        n = 0
        while True:
            h, ek, ev = slices[n % len(slices)]
            attention.attention_rotated(q[h * G:(h + 1) * G], ek["codes"][None], ek["norm16"][None],
                                        ev["codes"][None], ev["norm16"][None], P[0, h:h + 1])
            n += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    gbs = n * T * BYTES_PER_TOKEN_HEAD / el / 1e9
    return gbs, n, el


def oracle_config_rates():
    """The oracle, single-threaded, on bounded samples of the other workloads (a few seconds):
    encode Mvec/s on the tiny workload (512 tokens x K,V) and on one (layer, kv head) slice of the
    ingest workload (32768 tokens x K,V = 65536 vectors, 1% Student-t tokens); decode attention
    microseconds per layer on the tiny workload, one llama8b_8k layer (8 kv heads x 8192 tokens,
    4 q heads each) and one qwen30b_32k layer (4 kv heads x 32768 tokens, 8 q heads each), each
    extrapolated to the stack depth."""
    from threadpoolctl import threadpool_limits

    from oracle import attention, encode, rotation
    from rotated_bit_kv_iq_b200 import inputs

    out = {"encode_mvec_s": {}, "decode_us_per_layer": {}}
    with threadpool_limits(limits=1):
        P1 = rotation.init_rotation(inputs.ROTATION_SEED, 1, 8)
        # encode: tiny workload in full
        x = [inputs.kv_tokens(0, 0, 0, w, 0, 512, n_outliers=2) for w in (0, 1)]
        t0 = time.perf_counter()
        enc_tiny = [encode.encode(xi, P1[0, 0]) for xi in x]
        out["encode_mvec_s"]["tiny (1024 vectors)"] = 1024 / (time.perf_counter() - t0) / 1e6
        # encode: one (layer, kv head) slice of the ingest workload
        x = [inputs.kv_tokens(0, 0, 0, w, 0, 32768, heavy_frac=0.01) for w in (0, 1)]
        t0 = time.perf_counter()
        for xi in x:
            encode.encode(xi, P1[0, 0])
        el = time.perf_counter() - t0
        out["encode_mvec_s"]["ingest_32k slice (65536 vectors)"] = 65536 / el / 1e6
        out["encode_full_ingest_s_extrapolated"] = 16777216 / (65536 / el)
        # decode: tiny
        q = inputs.queries(0, 0, 1, 1, dtype="f32")[0].astype(np.float64)
        t0 = time.perf_counter()
        attention.attention_rotated(q, enc_tiny[0]["codes"][None], enc_tiny[0]["norm16"][None],
                                    enc_tiny[1]["codes"][None], enc_tiny[1]["norm16"][None], P1[0, :1])
        out["decode_us_per_layer"]["tiny (ctx 512, 1 head)"] = (time.perf_counter() - t0) * 1e6
        # decode: one layer of the 8K and 32K workloads (encoding outside the timed part)
        for name, Hkv, T, Hq, L in (("llama8b_8k", 8, 8192, 32, 1), ("qwen30b_32k", 4, 32768, 32, 48)):
            ek = [encode.encode(inputs.kv_tokens(0, 0, h, 0, 0, T), P1[0, h]) for h in range(Hkv)]
            ev = [encode.encode(inputs.kv_tokens(0, 0, h, 1, 0, T), P1[0, h]) for h in range(Hkv)]
            q = inputs.queries(0, 0, 1, Hq)[0].astype(np.float64)
            t0 = time.perf_counter()
            attention.attention_rotated(q, np.stack([e["codes"] for e in ek]), np.stack([e["norm16"] for e in ek]),
                                        np.stack([e["codes"] for e in ev]), np.stack([e["norm16"] for e in ev]),
                                        P1[0, :Hkv])
            us = (time.perf_counter() - t0) * 1e6
            out["decode_us_per_layer"][f"{name} (one layer)"] = us
            if L > 1:
                out[f"decode_ms_per_step_{name}_extrapolated"] = us * L / 1e3
    return out


def oracle_parity_sample(stack, layer, head, seed=0):
    """Parity of the timed step on one (layer, kv head): the oracle encodes the same fp16 tokens
    the bench's cache was filled with (tokens 0..ctx-2, regenerated from their device generator)
    plus the step's new token, its codes and norms are compared with the GPU's records
    (iq_export_codes), and its attention for the group's query heads with the step's output."""
    import torch

    from oracle import attention, encode, rotation
    from rotated_bit_kv_iq_b200 import inputs

    assert stack.B == 1
    Bd, dev = stack.Bd, stack.dev
    T = int(stack.ctx[0])
    G = stack.Hq // stack.Hkv
    P = rotation.init_rotation(inputs.ROTATION_SEED, stack.L, stack.Hkv)[layer, head]
    x = {}
    for w, new in ((0, stack.knew), (1, stack.vnew)):
        old = inputs.kv_tokens_device(seed, layer, stack.Hkv, w, T - 1, device=dev)[:, head].cpu().numpy()
        x[w] = np.concatenate([old, new[layer, 0, 0, head:head + 1].cpu().numpy()])
    enc = {w: encode.encode(x[w], P) for w in (0, 1)}
    codes = torch.empty((stack.Hkv, T, 128), dtype=torch.uint8, device=dev)
    norms = torch.empty((stack.Hkv, T), dtype=torch.int16, device=dev)
    excluded = mismatched = 0
    ulp = 0
    for w in (0, 1):
        Bd.iq_export_codes(stack.cache, layer, w, 0, 0, T, codes, norms)
        torch.cuda.synchronize()
        gc = codes[head].cpu().numpy()
        gn = norms[head].cpu().numpy().view(np.uint16)
        near = enc[w]["near"]
        excluded += int(near.sum())
        mismatched += int(((gc != enc[w]["codes"]) & ~near).sum())
        ulp = max(ulp, int(np.abs(gn.astype(np.int64) - enc[w]["norm16"].astype(np.int64)).max()))
    q = stack.q[layer, 0, head * G:(head + 1) * G].cpu().numpy().astype(np.float64)
    ref = attention.attention_rotated(q, enc[0]["codes"][None], enc[0]["norm16"][None], enc[1]["codes"][None],
                                      enc[1]["norm16"][None], P[None])
    got = stack.out[layer, 0, head * G:(head + 1) * G].cpu().numpy().astype(np.float64)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-300)
    err = float((np.abs(got - ref).max(axis=1) / den).max())
    n_codes = 2 * T * 128
    return {"sample": f"layer {layer}, kv head {head} ({G} q heads), {T} tokens of K and V, timed step's output",
            "max_rel_err": err, "tolerance": 2e-3, "code_mismatches_outside_band": mismatched,
            "excluded_codes": excluded, "codes_checked": n_codes, "exclusion_rate": excluded / n_codes,
            "norm_ulp_max": ulp, "pass": bool(err < 2e-3 and mismatched == 0 and ulp <= 1)}


def reference_arm(args):
    """--impl reference: the oracle on bounded samples of the headline workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = []
    for i in range(args.warmup + args.steps):
        gbs, n, el = oracle_decode_sample(seconds=2.0)
        if i >= args.warmup:
            per_step.append((gbs, el))
    gbs = float(np.mean([g for g, _ in per_step]))
    model, affinity = _cpu_info()
    sample = ("fp64 oracle decode attention, 1 kv head x 8 q heads x 32768 tokens per slice; each 'step' is a "
              "~2 s sampling window of repeated slices (ms_per_step is that window, not a decode step)")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean([e for _, e in per_step]) * 1e3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": HEADLINE + " (oracle sample)"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
                         "cpu_model": model, "affinity_cores": affinity},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="headline workload only")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline leg")
    ap.add_argument("--no-parity", action="store_true", help="skip the oracle check of the timed step's output")
    ap.add_argument("--layers", type=int, default=0, help="override the stack depth (profiling runs)")
    ap.add_argument("--only", default="", choices=["", "serving", "encode", "prefill", "deferred"],
                    help="run one secondary workload alone (profiling runs); no headline line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return reference_arm(args)

    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from rotated_bit_kv_iq_b200 import build

    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    from rotated_bit_kv_iq_b200 import binding as Bd
    from rotated_bit_kv_iq_b200 import inputs

    Bd.lib()
    stream = torch.cuda.Stream(device=dev)
    if args.only:
        if args.only == "serving":
            res = bench_serving(args.steps, args.warmup, dev, stream, seed=rank, world=world, n_layers=args.layers)
        elif args.only == "prefill":
            res = bench_prefill(args.steps, args.warmup, dev, stream, world=world)
        elif args.only == "deferred":
            res = bench_deferred(args.steps, args.warmup, dev, stream, world=world, n_layers=args.layers or 32)
        else:
            res = bench_encode(args.steps, args.warmup, dev, stream)
        if rank == 0:
            print(json.dumps({"only": args.only, **res}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return
    cfg = inputs.CONFIGS[HEADLINE]
    n_layers = args.layers or cfg["n_layers"]
    stack = DecodeStack(cfg["batch"], cfg["n_q_heads"], cfg["n_kv_heads"], n_layers, [cfg["ctx"]],
                        cfg["page_size"], dev, seed=rank)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    barrier()
    with ClockSampler(local) as clk:
        ms, graph = time_graph(stack, args.steps, args.warmup, stream)
    barrier()
    ms = max_over_ranks(ms, dev)
    value = job_gbs(world, stack.bytes_per_step, ms)

    # dominant kernel: the per-layer decode step (one kernel: append, split attention, merge,
    # inverse rotation), timed inside the step graph: step time / layers
    kern_ms = ms / stack.L
    layer_bytes = int(stack.ctx.sum()) * stack.Hkv * BYTES_PER_TOKEN_HEAD
    peak, peak_kind = _peaks()
    achieved = layer_bytes / (kern_ms * 1e-3) / 1e9
    e2e_ms, e2e_direct_ms, h2d, d2h = time_e2e(stack, args.steps, args.warmup, stream)
    e2e_ms = max_over_ranks(e2e_ms, dev)
    e2e_direct_ms = max_over_ranks(e2e_direct_ms, dev)
    del graph

    result = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 hi/lo tensor-core products (s32 accumulate); fp32 softmax, scaling and accumulation "
                 "across tiles; 3-bit codes, binary16 norms", "data": "synthetic",
        "config": {"workload": "qwen30b_32k: decode step (append + attend) B=1, 32 q / 4 kv heads, d=128, "
                               "48 layers, ctx 32768, packed 3-bit cache", "l2": "inputs larger than L2 (629 MB/step)",
                   "graph": f"{stack.L}-layer step replayed as one CUDA graph", "layers": stack.L,
                   "bytes_per_step": stack.bytes_per_step},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": decode_traffic(),
                     "kernel": "decode_kernel (one launch per layer: append + split attention + merge), CUDA-graph step time / layers",
                     "peak_kind": peak_kind, "bytes_per_launch": layer_bytes, "launch_ms": kern_ms},
        "e2e": {"value": job_gbs(world, stack.bytes_per_step, e2e_ms), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "calls": "48 iq_decode_step calls captured once as a CUDA graph, replayed each step",
                "direct_calls": {"value": job_gbs(world, stack.bytes_per_step, e2e_direct_ms), "unit": "GB/s",
                                 "ms_per_step": e2e_direct_ms,
                                 "calls": "48 iq_decode_step calls through the C ABI every step"}},
        "gpu_launches": stack.L * DecodeStack.launches_per_layer * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_parity:
        # the timed step's own output and records against the oracle, on one (layer, kv head)
        result["parity"] = oracle_parity_sample(stack, stack.L - 1, 1 % stack.Hkv, seed=rank)
    del stack
    torch.cuda.empty_cache()

    if not args.no_extras:
        srv = bench_serving(args.steps, args.warmup, dev, stream, seed=rank, world=world)
        result["serving"] = srv
        result["gpu_launches"] += srv["launches"]
        torch.cuda.empty_cache()
        enc = bench_encode(args.steps, args.warmup, dev, stream)
        enc["ms_per_step"] = max_over_ranks(enc["ms_per_step"], dev)
        enc["launch_ms"] = max_over_ranks(enc["launch_ms"], dev)
        mvec = world * enc["vectors_per_step"] / (enc["ms_per_step"] * 1e-3) / 1e6
        enc_ach = enc["bytes_per_launch"] / (enc["launch_ms"] * 1e-3) / 1e9
        result["encode"] = {
            "workload": "ingest_32k: 32768 tokens x 8 kv heads x 32 layers of K and V (16.8 M vectors), 1% Student-t",
            "value": mvec, "unit": "Mvec/s", "GBps": mvec * 1e6 * BYTES_PER_VECTOR_ENCODE / 1e9,
            "ms_per_step": enc["ms_per_step"],
            "roofline": {"bound": "hbm", "achieved": enc_ach, "peak": peak, "unit": "GB/s", "frac": enc_ach / peak,
                         "traffic": decode_traffic(ENCODE_TRAFFIC), "kernel": "encode (one layer, K and V)",
                         "peak_kind": peak_kind},
        }
        result["gpu_launches"] += 32 * args.steps
        torch.cuda.empty_cache()
        pre = bench_prefill(args.steps, args.warmup, dev, stream, world=world)
        result["prefill"] = pre
        result["gpu_launches"] += pre["launches"]
        torch.cuda.empty_cache()
        dfr = bench_deferred(args.steps, args.warmup, dev, stream, world=world)
        result["deferred"] = dfr
        result["gpu_launches"] += dfr["launches"]
        torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_cpu:
        gbs, n, el = oracle_decode_sample(args.cpu_seconds)
        model, affinity = _cpu_info()
        result["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                  "sample": f"{n} x (1 kv head, 8 q heads, 32768 tokens) decode slices in {el:.1f} s",
                                  "cpu_model": model, "affinity_cores": affinity, **oracle_config_rates()}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
