#!/usr/bin/env python
"""Benchmark of the KV-COBRA transform-coded KV cache on B200.

Headline (the metric): decode-attention effective HBM GB/s (and % of the measured HBM
peak) over a 32-layer Llama-3.1-8B-shaped cache (32 query / 8 KV heads, d = 128) of
131072 tokens compressed at a joint 1 bit per dimension; plus encode Mtok/s for the
28-layer Qwen2.5-7B-shaped prefill of 131072 tokens at 2 bits per dimension.

One step = one decode step of the whole model: for each of the 32 layers, append the
new token's K/V (encode: project, quantize, pack) and run decode attention over the
131072-token cache (q into the key basis, unpack + scores, online softmax, value
accumulation in the latent basis, split merge, back-projection).  The 32 layers are
captured in one CUDA graph and replayed; inputs are resident in HBM.  GB/s counts the
algorithmic bytes of a step: packed codes of every cached token plus the projection
bases (fp32 M_K and M_V) of every KV head.  roofline: the decode call of one layer, timed
as the mean call of a graph of the 32 decode calls alone.

Beside the headline the same line carries the other workloads of the method's scope:
layer32k (one 32k-token layer at 2 bpd, L2 evicted before every call), sweep (16
sequences x 32k tokens, 32 layers, at 0.5 / 1 / 2 / 4 bpd), k_only (keys coded, values
fp16), prerope (the same cache read as keys coded before the rotary embedding), encode (the 28-layer Qwen-shaped prefill of 131072 tokens, tensor cores) and
qwen_decode (one decode step over that cache, 7 query heads per KV head), sdpa_context
(torch fp16 SDPA at the headline shape) and cpu_baseline (the oracle on host cores:
decode sample, whole-plan calibration, canonical encode sample).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: replicas only (each rank runs the same workload on its own GPU; no data-path
collective); timing is the max over ranks.  ``--impl reference`` times the CPU oracle
(the plain fp64 restatement of the method) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_quantization_head_b200 import kvtc, synth  # noqa: E402

DECODE_WORKLOAD = "llama8b-32L-128k-1bpd"
ENCODE_WORKLOAD = "qwen7b-28L-128k-2bpd"

# DRAM bytes (read + write) of one decode call per layer, from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum) of the current decode kernel: layer 6 of
# the 8-layer copy of the workload read 32.40 MB against its 32.08 MB of algorithmic
# bytes (1.010x); scaled by that ratio to this workload's mean layer (the file named
# beside it).  None whenever a decode kernel has changed since the capture.
DECODE_TRAFFIC = {"llama8b-32L-128k-1bpd": (34.42e6, "profiles/decode_split_llama8b-8L-128k-1bpd_ncu.md")}
METRIC = "decode-attn effective HBM GB/s (% of peak) at 128k ctx; encode Mtok/s"


# ---------------------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu_id)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
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
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def record_external(event, stream):
    """cudaEventRecordWithFlags(..., cudaEventRecordExternal): an event that stays a timing
    node when recorded inside CUDA-graph capture."""
    from cuda.bindings import runtime as rt
    err, = rt.cudaEventRecordWithFlags(event.cuda_event, stream.cuda_stream, rt.cudaEventRecordExternal)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaEventRecordWithFlags: {err}")


def algorithmic_bytes(plan, layers, seq_len, n_seq):
    """Packed codes of every cached token plus the fp32 bases M_K, M_V, per KV head."""
    H = plan.shape["n_kv_heads"]
    per_layer = []
    for layer in layers:
        t = 0
        for h in range(H):
            for kind in (0, 1):
                info = plan.unit((layer * H + h) * 2 + kind)
                t += n_seq * seq_len * info["r"] * info["b"] // 8 + info["r"] * 128 * 4
        per_layer.append(t)
    return per_layer


# ---------------------------------------------------------------------------- our arm
def build_decode_setup(torch, w, rank, k_only=False):
    """Calibrate, allocate the cache, prefill 131071 tokens of every layer (encode path),
    and prepare the step's inputs.  Returns a dict of state."""
    t0 = time.time()
    k_cal, v_cal, q_cal = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k_cal, v_cal, q_cal, n_layers=w.n_layers, n_kv_heads=w.n_kv_heads,
                               group=w.group, bpd=w.bpd, seed=w.seed, fixed_r=w.fixed_r,
                               fixed_b=w.fixed_b, k_only=k_only).upload()
    t_cal = time.time() - t0
    H, G, L, T, B = w.n_kv_heads, w.group, w.n_layers, w.seq_len, w.batch
    pages = (T + 127) // 128
    rng = np.random.default_rng(1234 + rank)
    bt = torch.from_numpy(rng.permutation(B * pages).astype(np.int32).reshape(B, pages))
    cache = kvtc.Cache(plan, B * pages, bt)
    dev = torch.device("cuda")
    specs = {(l, h, kd): synth.unit_spec(w, l, h, kd) for l in range(L) for h in range(H) for kd in (0, 1)}
    prefix = T - 1
    for layer in range(L):
        for s in range(B):
            k, v = synth.layer_kv_torch(w, layer, prefix, dev, seq=s, specs=specs)
            try:
                kvtc.kvtc_encode_prefill(plan, cache, layer, k, v, s, 0)
            except kvtc.KvtcError:
                cu = torch.tensor([0, prefix], dtype=torch.int32, device=dev)
                pos = torch.tensor([0], dtype=torch.int32, device=dev)
                # one sequence per call: cu_seqlens / pos_start describe only sequence s
                sub = kvtc.Cache.__new__(kvtc.Cache)
                sub.__dict__.update(cache.__dict__)
                sub.desc = kvtc.CacheDesc(cache.pool.data_ptr(), cache.pages_per_unit,
                                          cache.block_table[s:s + 1].data_ptr(), 1, pages,
                                          cache.status.data_ptr())
                kvtc.kvtc_encode_append(plan, sub, layer, k, v, cu, pos)
            del k, v
    torch.cuda.synchronize()
    # step inputs: one new token per sequence and layer, and the decode queries
    dt = torch.bfloat16
    k_new = torch.empty((L, B, H, 128), dtype=dt, device=dev)
    v_new = torch.empty((L, B, H, 128), dtype=dt, device=dev)
    q = torch.empty((L, B, H * G, 128), dtype=dt, device=dev)
    for layer in range(L):
        for s in range(B):
            k1, v1 = synth.layer_kv_torch(w, layer, 1, dev, seq=10_000 + s, specs=specs)
            k_new[layer, s] = k1[0]
            v_new[layer, s] = v1[0]
            q[layer, s] = torch.from_numpy(synth.decode_queries(w, layer, s)).to(dev, dt)
    out = torch.empty((L, B, H * G, 128), dtype=dt, device=dev)
    cu = torch.arange(B + 1, dtype=torch.int32, device=dev)
    pos = torch.full((B,), prefix, dtype=torch.int32, device=dev)
    seq_lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    ws = torch.zeros(kvtc.kvtc_decode_workspace_bytes(plan, B, T), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    return dict(plan=plan, cache=cache, k_new=k_new, v_new=v_new, q=q, out=out, cu=cu, pos=pos,
                seq_lens=seq_lens, ws=ws, t_cal=t_cal, t_setup=time.time() - t0)


def decode_step(st, w, stream=None):
    """One decode step of the whole model: per layer, append the new token, then decode."""
    plan, cache = st["plan"], st["cache"]
    for layer in range(w.n_layers):
        kvtc.kvtc_encode_append(plan, cache, layer, st["k_new"][layer], st["v_new"][layer], st["cu"], st["pos"],
                                stream=stream)
        kvtc.kvtc_decode_attention(plan, cache, layer, st["q"][layer], st["seq_lens"], w.seq_len,
                                   st["out"][layer], st["ws"], stream=stream)


def kernels_per_step(plan, w):
    """Launches of the library's kernels per step: per layer the append and one split
    kernel per distinct (b_K, b_V) pair among the layer's KV heads (the merge and the
    back-projection run inside the split kernel)."""
    n = 0
    H = plan.shape["n_kv_heads"]
    for layer in range(w.n_layers):
        groups = {(plan.unit((layer * H + h) * 2)["b"], plan.unit((layer * H + h) * 2 + 1)["b"]) for h in range(H)}
        n += 1 + len(groups)
    return n


def cpu_baseline_decode(torch, st, w, budget_s=12.0):
    """The oracle (as it stands) on a bounded sample: KV heads of layer 0 over the full
    131072-token cache, fp64 d-space attention over the GPU-written pages."""
    from oracle import attention as oatt
    from oracle import codec as ocodec
    plan, cache = st["plan"], st["cache"]
    H, G, T = w.n_kv_heads, w.group, w.seq_len
    pages = (T + 127) // 128
    q = st["q"][0, 0].float().cpu().numpy().astype(np.float64)
    bt = cache.block_table.cpu().numpy()[0]
    done_bytes, t_used, heads = 0, 0.0, 0
    for h in range(H):
        uK, uV = h * 2, h * 2 + 1
        infos = [plan.unit(uK), plan.unit(uV)]
        pools = [cache.unit_pool(u).cpu().numpy() for u in (uK, uV)]
        units = [dict(M=plan.matrix(u), delta=i["delta"], b=i["b"]) for u, i in zip((uK, uV), infos)]
        t0 = time.perf_counter()
        codes = []
        for kind, (pool, info) in enumerate(zip(pools, infos)):
            pb = info["page_bytes"]
            pg = [pool[int(bt[p]) * pb:(int(bt[p]) + 1) * pb] for p in range(pages)]
            codes.append(ocodec.unpack_sequence(pg, kind, info["r"], info["b"], T))
        oatt.decode_head(q[h * G:(h + 1) * G], codes[0], codes[1], units[0], units[1], 1 / math.sqrt(128))
        t_used += time.perf_counter() - t0
        done_bytes += sum(T * i["r"] * i["b"] // 8 + i["r"] * 128 * 4 for i in infos)
        heads += 1
        if t_used >= budget_s:
            break
    return done_bytes, t_used, heads


def host_cores():
    """Host cores this process may run on (the oracle's numpy/BLAS threads use them)."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def encode_bench(torch, w, steps, warmup, rank, n_layers=None, keep=False):
    """Encode Mtok/s: every layer's K and V of 131072 tokens, resident in HBM.  With keep,
    also returns the encoded cache (plan, cache) for the decode leg over it."""
    dev = torch.device("cuda")
    if n_layers:
        w = synth.scaled(w, n_layers=n_layers)
    k_cal, v_cal, q_cal = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k_cal, v_cal, q_cal, n_layers=w.n_layers, n_kv_heads=w.n_kv_heads,
                               group=w.group, bpd=w.bpd, seed=w.seed).upload()
    T = w.seq_len
    pages = T // 128
    bt = torch.arange(pages, dtype=torch.int32).reshape(1, pages)
    cache = kvtc.Cache(plan, pages, bt)
    specs = {(l, h, kd): synth.unit_spec(w, l, h, kd) for l in range(w.n_layers) for h in range(w.n_kv_heads)
             for kd in (0, 1)}
    kv = [synth.layer_kv_torch(w, l, T, dev, specs=specs) for l in range(w.n_layers)]
    cu = torch.tensor([0, T], dtype=torch.int32, device=dev)
    pos = torch.tensor([0], dtype=torch.int32, device=dev)
    use_prefill = True
    try:
        kvtc.kvtc_encode_prefill(plan, cache, 0, kv[0][0], kv[0][1], 0, 0)
    except kvtc.KvtcError:
        use_prefill = False

    def one_pass():
        for l in range(w.n_layers):
            if use_prefill:
                kvtc.kvtc_encode_prefill(plan, cache, l, kv[l][0], kv[l][1], 0, 0)
            else:
                kvtc.kvtc_encode_append(plan, cache, l, kv[l][0], kv[l][1], cu, pos)

    for _ in range(max(1, warmup)):
        one_pass()
    torch.cuda.synchronize()
    fix = kvtc.kvtc_plan_prefill_stats(plan, reset=True) if use_prefill else (0, 0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one_pass()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    fix = kvtc.kvtc_plan_prefill_stats(plan) if use_prefill else (0, 0)
    in_bytes = w.n_layers * T * w.n_kv_heads * 128 * 2 * 2
    code_bytes = sum(T * plan.unit(u)["r"] * plan.unit(u)["b"] // 8 for u in range(plan.shape["n_units"]))
    flops = sum(2 * 128 * plan.unit(u)["r"] for u in range(plan.shape["n_units"])) * T
    hbm_peak, tf_peak, peak_kind = measured_peaks()
    gbs = (in_bytes + code_bytes) / ms / 1e6
    res = {"workload": w.name, "path": "prefill (tensor cores)" if use_prefill else "append (CUDA cores)",
           "recomputed_fraction": (fix[1] / fix[0]) if fix[0] else None,
           "ms_per_pass": round(ms, 4), "mtok_s": round(T / ms / 1e3, 3), "gb_s": round(gbs, 1),
           "bytes_per_pass": in_bytes + code_bytes, "tflop_s": round(flops / ms / 1e9, 2), "layers": w.n_layers,
           "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                        "frac": round(gbs / hbm_peak, 4), "peak_kind": peak_kind,
                        "hbm_roof_mtok_s": round(hbm_peak * 1e9 / ((in_bytes + code_bytes) / T) / 1e6, 2)}}
    del kv
    torch.cuda.empty_cache()
    if keep:
        return res, (w, plan, cache)
    return res


def graph_of(torch, stream, fn):
    """fn() captured in a CUDA graph on stream (after one eager run that warms it)."""
    with torch.cuda.stream(stream):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    torch.cuda.synchronize()
    return g


def time_graph(torch, g, stream, steps, warmup):
    """Mean ms per replay of g: warm-up replays, then steps replays bracketed by events."""
    with torch.cuda.stream(stream):
        for _ in range(max(3, warmup)):
            g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def decode_calls(st, w, stream):
    """The decode calls of every layer alone (no appends): the per-call timing graph."""
    for layer in range(w.n_layers):
        kvtc.kvtc_decode_attention(st["plan"], st["cache"], layer, st["q"][layer], st["seq_lens"], w.seq_len,
                                   st["out"][layer], st["ws"], stream=stream)


def rope_leg(torch, st, w, steps, warmup):
    """The pre-RoPE decode (keys coded before the rotary embedding; kvtc_decode_attention_rope)
    over the same cache: every layer's call in one graph, mean call time.  Its work is
    dominated by the per-block key reconstruction on the tensor cores (16 tokens x r_K x
    128, fp16 hi + lo parts of M_K), so the line also reports those MMA flops."""
    stream = torch.cuda.Stream()

    def calls():
        for layer in range(w.n_layers):
            kvtc.kvtc_decode_attention_rope(st["plan"], st["cache"], layer, st["q"][layer], st["seq_lens"], w.seq_len,
                                            st["out"][layer], st["ws"], stream=stream)
    g = graph_of(torch, stream, calls)
    ms = time_graph(torch, g, stream, steps, warmup) / w.n_layers
    del g
    plan = st["plan"]
    b = sum(algorithmic_bytes(plan, range(w.n_layers), w.seq_len, w.batch)) / w.n_layers
    H = plan.shape["n_kv_heads"]
    rec_flops = sum(2 * 2 * 16 * ((plan.unit((l * H + h) * 2)["r"] + 15) // 16) * 128
                    for l in range(w.n_layers) for h in range(H)) * w.seq_len * w.batch / w.n_layers
    hbm_peak, tf_peak, peak_kind = measured_peaks()
    return {"workload": w.name, "decode_call_ms": round(ms, 5), "gb_s": round(b / (ms * 1e-3) / 1e9, 1),
            "frac": round(b / (ms * 1e-3) / 1e9 / hbm_peak, 4), "peak": hbm_peak, "peak_kind": peak_kind,
            "reconstruction_tflop_s": round(rec_flops / (ms * 1e-3) / 1e12, 1),
            "rope_base": 500000.0, "bytes_per_call": int(b)}


def decode_leg(torch, w, steps, warmup, rank, k_only=False, setup=None):
    """Throughput of one decode step over a workload: the step graph (append + decode per
    layer) and the decode calls alone (the roofline figure: algorithmic bytes of one
    call / mean call time from a graph of the calls with no events inside)."""
    st = setup or build_decode_setup(torch, w, rank, k_only=k_only)
    plan = st["plan"]
    stream = torch.cuda.Stream()
    per_layer = algorithmic_bytes(plan, range(w.n_layers), w.seq_len, w.batch)
    step_bytes = sum(per_layer)
    g_step = graph_of(torch, stream, lambda: decode_step(st, w, stream=stream))
    g_dec = graph_of(torch, stream, lambda: decode_calls(st, w, stream))
    ms_step = time_graph(torch, g_step, stream, steps, warmup)
    ms_dec = time_graph(torch, g_dec, stream, steps, warmup) / w.n_layers
    hbm_peak, _, peak_kind = measured_peaks()
    achieved = (step_bytes / w.n_layers) / (ms_dec * 1e-3) / 1e9
    out = {"workload": w.name, "layers": w.n_layers, "batch": w.batch, "seq_len": w.seq_len, "bpd": w.bpd,
           "group": w.group, "k_only": bool(k_only), "bytes_per_step": step_bytes,
           "ms_per_step": round(ms_step, 4), "gb_s": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
           "decode_call_ms": round(ms_dec, 5), "decode_call_gb_s": round(achieved, 1),
           "frac": round(achieved / hbm_peak, 4), "peak": hbm_peak, "peak_kind": peak_kind}
    del g_step, g_dec
    return out, st


def layer32k_leg(torch, reps=30):
    """One 32k-token layer at 2 bpd (16.8 MB of codes, L2-resident unless evicted): each
    timed decode call follows a 512 MB write that evicts L2; median of reps."""
    w = synth.WORKLOADS["llama8b-layer-32k-2bpd"]
    st = build_decode_setup(torch, w, 0)
    stream = torch.cuda.Stream()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        decode_step(st, w, stream=stream)  # the newest token
        for ea, eb in evs:                 # torch creates its events lazily, on first record
            ea.record(stream)
            eb.record(stream)
    torch.cuda.synchronize()

    def call():
        kvtc.kvtc_decode_attention(st["plan"], st["cache"], 0, st["q"][0], st["seq_lens"], w.seq_len, st["out"][0],
                                   st["ws"], stream=stream)
    with torch.cuda.stream(stream):
        call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for ea, eb in evs:
            flush.fill_(1)
            record_external(ea, stream)
            call()
            record_external(eb, stream)
    with torch.cuda.stream(stream):
        g.replay()
        g.replay()
    torch.cuda.synchronize()
    ms = statistics.median(ea.elapsed_time(eb) for ea, eb in evs)
    b = algorithmic_bytes(st["plan"], [0], w.seq_len, 1)[0]
    hbm_peak, _, peak_kind = measured_peaks()
    del g, flush, st
    torch.cuda.empty_cache()
    return {"workload": w.name, "bytes_per_call": b, "decode_call_us": round(ms * 1e3, 2),
            "gb_s": round(b / (ms * 1e-3) / 1e9, 1), "frac": round(b / (ms * 1e-3) / 1e9 / hbm_peak, 4),
            "peak": hbm_peak, "peak_kind": peak_kind, "l2": "512 MB write before every timed call"}


def qwen_decode_leg(torch, enc_state, steps, warmup):
    """One decode step over the 28-layer Qwen cache the encode leg wrote (G = 7)."""
    w, plan, cache = enc_state
    dev = torch.device("cuda")
    T = w.seq_len
    q = torch.stack([torch.from_numpy(synth.decode_queries(w, l)) for l in range(w.n_layers)]).to(dev, torch.bfloat16)
    st = dict(plan=plan, cache=cache, q=q.reshape(w.n_layers, 1, w.n_q_heads, 128),
              out=torch.empty((w.n_layers, 1, w.n_q_heads, 128), dtype=torch.bfloat16, device=dev),
              seq_lens=torch.full((1,), T, dtype=torch.int32, device=dev),
              ws=torch.zeros(kvtc.kvtc_decode_workspace_bytes(plan, 1, T), dtype=torch.uint8, device=dev))
    stream = torch.cuda.Stream()
    g = graph_of(torch, stream, lambda: decode_calls(st, w, stream))
    ms = time_graph(torch, g, stream, steps, warmup)
    b = sum(algorithmic_bytes(plan, range(w.n_layers), T, 1))
    hbm_peak, _, peak_kind = measured_peaks()
    del g
    return {"workload": w.name, "group": w.group, "layers": w.n_layers, "bytes_per_step": b,
            "ms_per_step": round(ms, 4), "decode_call_ms": round(ms / w.n_layers, 5),
            "gb_s": round(b / (ms * 1e-3) / 1e9, 1), "frac": round(b / (ms * 1e-3) / 1e9 / hbm_peak, 4),
            "peak": hbm_peak, "peak_kind": peak_kind, "step": "decode calls of every layer (no append)"}


def oracle_calibrate_and_encode(budget_s=6.0):
    """The oracle timed on the host: the whole-model calibration of the 32-layer llama
    plan (eigen-decompositions, KL weights, C1 + C2, Hadamard folds), and its canonical
    fp32 encode (project, quantize) of a sample of the Qwen prefill workload (layer 0,
    every KV head, K and V), reported per whole-model token."""
    from oracle import calibration as ocal
    from oracle import codec as ocodec
    w = synth.WORKLOADS[DECODE_WORKLOAD]
    k_cal, v_cal, q_cal = synth.calibration_set(w)
    t0 = time.perf_counter()
    ocal.calibrate(k_cal, v_cal, q_cal, w.n_layers, w.n_kv_heads, bpd=w.bpd, seed=w.seed)
    t_cal = time.perf_counter() - t0
    we = synth.WORKLOADS[ENCODE_WORKLOAD]
    kc, vc, qc = synth.calibration_set(we, layers=[0])
    units = ocal.calibrate(kc, vc, qc, 1, we.n_kv_heads, bpd=we.bpd, seed=we.seed)
    n_tok, t_enc = 0, 0.0
    chunk = 512
    while t_enc < budget_s:
        for h in range(we.n_kv_heads):
            for kind in (0, 1):
                u = units[h * 2 + kind]
                x = synth.cache_tokens(we, 0, h, kind, chunk, seq=1 + n_tok // chunk)
                t0 = time.perf_counter()
                ocodec.encode_tokens(x, ocodec.to_bf16(u["M"].astype(np.float32)), u["inv_delta"], u["b"])
                t_enc += time.perf_counter() - t0
        n_tok += chunk
    units_model = we.n_layers * we.n_kv_heads * 2
    tok_s = n_tok * (2 * we.n_kv_heads) / units_model / t_enc
    return {"calibrate_s": round(t_cal, 2),
            "calibrate_sample": f"whole {w.name} plan ({w.n_layers * w.n_kv_heads * 2} units, C2 over all)",
            "encode_mtok_s": round(tok_s / 1e6, 6),
            "encode_sample": f"layer 0 of {we.name}: {n_tok} tokens x {we.n_kv_heads} KV heads x K, V "
                             f"(canonical fp32 projection + quantize), scaled to whole-model tokens"}


def max_over_ranks(torch, dist, x):
    """The largest value of x over the ranks (every rank gets it); x itself when alone.
    The reduction runs on the backend's device (CUDA for NCCL, host for gloo)."""
    if not dist:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(world, step_bytes, ms):
    """Whole-job GB/s: every rank streams step_bytes per step (replicas, weak scaling);
    the step time is the slowest rank's."""
    return world * step_bytes / (ms * 1e-3) / 1e9


def run_ours(args, torch, dist, rank, world):
    w = synth.WORKLOADS[args.workload]
    if args.layers:
        w = synth.scaled(w, n_layers=args.layers)
    if args.seq_len:
        w = synth.scaled(w, seq_len=args.seq_len)
    if args.bpd:
        w = synth.with_bpd(w, args.bpd)
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    if args.no_decode:
        return {"encode": encode_bench(torch, synth.WORKLOADS[ENCODE_WORKLOAD], max(1, min(args.steps, 5)),
                                       args.warmup, rank, args.encode_layers)}
    st = build_decode_setup(torch, w, rank, k_only=args.k_only)
    plan = st["plan"]
    stream = torch.cuda.Stream()
    L = w.n_layers
    per_layer_bytes = algorithmic_bytes(plan, range(L), w.seq_len, w.batch)
    step_bytes = sum(per_layer_bytes)

    g = graph_of(torch, stream, lambda: decode_step(st, w, stream=stream))
    # the decode calls alone (no appends, no events inside): the per-call roofline figure
    g_dec = graph_of(torch, stream, lambda: decode_calls(st, w, stream))

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            g.replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    gpu_id = torch.cuda.get_device_properties(torch.cuda.current_device()).uuid
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(f"GPU-{gpu_id}") as clk, torch.cuda.stream(stream):
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(torch, dist, e0.elapsed_time(e1) / args.steps)
    if dist:
        dist.barrier()

    dec_ms = time_graph(torch, g_dec, stream, max(10, min(args.steps, 50)), args.warmup) / L
    hbm_peak, tf_peak, peak_kind = measured_peaks()
    achieved = (step_bytes / L) / (dec_ms * 1e-3) / 1e9

    # end to end: H2D of the step's inputs from pinned memory, the graph, D2H of outputs
    q_h = st["q"].cpu().pin_memory()
    kn_h = st["k_new"].cpu().pin_memory()
    vn_h = st["v_new"].cpu().pin_memory()
    out_h = torch.empty_like(st["out"], device="cpu").pin_memory()
    h2d = q_h.numel() * 2 + kn_h.numel() * 2 + vn_h.numel() * 2
    d2h = out_h.numel() * 2
    with torch.cuda.stream(stream):
        for _ in range(3):
            st["q"].copy_(q_h, non_blocking=True)
            g.replay()
            out_h.copy_(st["out"], non_blocking=True)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for _ in range(args.steps):
            st["q"].copy_(q_h, non_blocking=True)
            st["k_new"].copy_(kn_h, non_blocking=True)
            st["v_new"].copy_(vn_h, non_blocking=True)
            g.replay()
            out_h.copy_(st["out"], non_blocking=True)
        f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(torch, dist, f0.elapsed_time(f1) / args.steps)
    del g, g_dec

    traffic, traffic_from = (None, None) if args.k_only else DECODE_TRAFFIC.get(w.name, (None, None))
    value = aggregate_value(world, step_bytes, ms)
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "layers": L, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
                   "head_dim": 128, "batch": w.batch, "seq_len": w.seq_len, "bpd": w.bpd,
                   "parallelism": f"replicas x{world}", "k_only": bool(args.k_only),
                   "step": f"per layer: append 1 token + decode attention; {L} layers in one CUDA graph",
                   "l2": f"inputs larger than L2: {step_bytes / 1e9:.3f} GB of codes+bases per step vs 126 MB",
                   "compute": "bf16 in/out; fp16 tensor-core operands (codes exact, q split hi+lo), "
                              "fp32 accumulation"},
        "pct_of_peak": round(100 * value / world / hbm_peak, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": traffic, "traffic_from": traffic_from,
                     "kernel": "decode call of one layer (all its launches)", "peak_kind": peak_kind,
                     "bytes_per_launch": step_bytes // L, "launch_ms": round(dec_ms, 5),
                     "launch_ms_from": "graph of the 32 decode calls alone (no events inside), mean per call"},
        "e2e": {"value": round(aggregate_value(world, step_bytes, e2e_ms), 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": kernels_per_step(plan, w) * args.steps,
        "clocks": clk.summary(),
        "setup_s": {"calibrate": round(st["t_cal"], 1), "total": round(st["t_setup"], 1),
                    "calib_stats": round(plan.calib_seconds()[0], 3),
                    "calib_c1_c2": round(plan.calib_seconds()[1], 4)},
    }
    if not args.no_sdpa:
        res["sdpa_context"] = sdpa_context(torch, w, dec_ms)
    if not args.no_extra and not args.k_only:
        res["prerope"] = rope_leg(torch, st, w, max(3, min(args.steps, 10)), 3)
    cpu_decode = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_decode = cpu_baseline_decode(torch, st, w, budget_s=8.0)
    del st
    torch.cuda.empty_cache()
    side_steps = max(3, min(args.steps, 20))
    if not args.no_extra:
        # the scope table's other decode workloads (each set up, timed and freed in turn)
        res["layer32k"] = layer32k_leg(torch)
        sweep = []
        for bpd in (0.5, 1.0, 2.0, 4.0):
            ws = synth.with_bpd(synth.WORKLOADS["llama8b-32L-b16x32k"], bpd)
            out, st2 = decode_leg(torch, ws, side_steps, 3, rank)
            sweep.append(out)
            del st2
            torch.cuda.empty_cache()
        res["sweep"] = sweep
        if not args.k_only:
            out, st2 = decode_leg(torch, w, side_steps, 3, rank, k_only=True)
            res["k_only"] = out
            del st2
            torch.cuda.empty_cache()
    if not args.no_encode:
        enc, enc_state = encode_bench(torch, synth.WORKLOADS[ENCODE_WORKLOAD], max(1, min(args.steps, 5)),
                                      args.warmup, rank, args.encode_layers, keep=True)
        res["encode"] = enc
        if not args.no_extra:
            res["qwen_decode"] = qwen_decode_leg(torch, enc_state, side_steps, 3)
        del enc_state
        torch.cuda.empty_cache()
    if cpu_decode is not None:
        b, t, heads = cpu_decode
        res["cpu_baseline"] = {"value": round(b / t / 1e9, 5), "unit": "GB/s", "cores": host_cores(),
                               "kind": "oracle",
                               "sample": f"{heads} KV head(s) of layer 0 (G={w.group} queries each) over the "
                                         f"{w.seq_len}-token cache: unpack + fp64 d-space attention"}
        res["cpu_baseline"].update(oracle_calibrate_and_encode())
    return res


def sdpa_context(torch, w, dec_ms, reps=20):
    """Context for the pages' speed claim against FP16 SDPA (KV-COBRA project page,
    "Efficiency"): torch's fp16 scaled_dot_product_attention for one decode query over an
    uncompressed cache of the same shape (G query heads per KV head), timed per layer.
    Not part of the product path; the cache is 2 * H_kv * T * 256 bytes > L2."""
    import torch.nn.functional as F
    T, H, Hq = w.seq_len, w.n_kv_heads, w.n_q_heads
    gen = torch.Generator(device="cuda").manual_seed(7)
    k = torch.randn((w.batch, H, T, 128), generator=gen, device="cuda", dtype=torch.float16)
    v = torch.randn((w.batch, H, T, 128), generator=gen, device="cuda", dtype=torch.float16)
    q = torch.randn((w.batch, Hq, 1, 128), generator=gen, device="cuda", dtype=torch.float16)
    for _ in range(3):
        F.scaled_dot_product_attention(q, k, v, enable_gqa=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        F.scaled_dot_product_attention(q, k, v, enable_gqa=True)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    kv_bytes = 2 * w.batch * H * T * 128 * 2
    del k, v, q
    torch.cuda.empty_cache()
    return {"fp16_sdpa_ms_per_layer": round(ms, 5), "fp16_sdpa_gb_s": round(kv_bytes / (ms * 1e-3) / 1e9, 1),
            "compressed_decode_ms_per_layer": round(dec_ms, 5), "speedup": round(ms / dec_ms, 3),
            "shape": f"batch {w.batch}, {Hq} q / {H} kv heads, {T} tokens, d 128"}


def efficiency_table(torch, reps=20):
    """The KV-COBRA project page's Efficiency table restated on this GPU: the per-layer
    attention primitive (one decode call: 32 query / 8 KV heads, d = 128, batch 1, every
    K and V head at the table's fixed (r, b)) against torch's fp16 SDPA over an
    uncompressed cache of the same shape, at 32k, 64k and 128k tokens.  Each timed call
    follows a 256 MB write that evicts L2, and both sides run from CUDA graphs with
    events around the call alone.  Returns one row per (context, r, b) with the pages'
    RTX 6000 Ada speed-up beside the measured one."""
    import torch.nn.functional as F
    pages = {(16, 2): (1.83, 1.79, 1.89), (16, 4): (1.84, 1.85, 1.88), (32, 2): (1.77, 1.82, 1.85),
             (64, 2): (1.40, 1.48, 1.49)}
    contexts = (32768, 65536, 131072)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    base = synth.WORKLOADS[DECODE_WORKLOAD]

    def graph_time(fn):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        with torch.cuda.stream(stream):
            fn()
            for ea, eb in evs:
                ea.record(stream)
                eb.record(stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for ea, eb in evs:
                flush.fill_(1)
                record_external(ea, stream)
                fn()
                record_external(eb, stream)
        with torch.cuda.stream(stream):
            g.replay()
            g.replay()
        torch.cuda.synchronize()
        t = statistics.median(ea.elapsed_time(eb) for ea, eb in evs)
        del g
        return t

    rows = []
    for ci, T in enumerate(contexts):
        gen = torch.Generator(device="cuda").manual_seed(11)
        H, Hq = base.n_kv_heads, base.n_q_heads
        kf = torch.randn((1, H, T, 128), generator=gen, device="cuda", dtype=torch.float16)
        vf = torch.randn((1, H, T, 128), generator=gen, device="cuda", dtype=torch.float16)
        qf = torch.randn((1, Hq, 1, 128), generator=gen, device="cuda", dtype=torch.float16)
        sdpa_ms = graph_time(lambda: F.scaled_dot_product_attention(qf, kf, vf, enable_gqa=True))
        del kf, vf, qf
        for (r, b), sp in pages.items():
            w = synth.scaled(base, n_layers=1, seq_len=T, fixed_r=r, fixed_b=b)
            st = build_decode_setup(torch, w, 0)
            with torch.cuda.stream(stream):
                decode_step(st, w, stream=stream)  # the newest token
            torch.cuda.synchronize()

            def call():
                kvtc.kvtc_decode_attention(st["plan"], st["cache"], 0, st["q"][0], st["seq_lens"], T, st["out"][0],
                                           st["ws"], stream=stream)
            dec_ms = graph_time(call)
            rows.append({"context": T, "r": r, "b": b, "decode_us": round(dec_ms * 1e3, 2),
                         "fp16_sdpa_us": round(sdpa_ms * 1e3, 2), "speedup": round(sdpa_ms / dec_ms, 2),
                         "pages_speedup_rtx6000ada": sp[ci]})
            del st
            torch.cuda.empty_cache()
    return rows


# ---------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The CPU oracle as it stands on a bounded sample of the decode workload: one KV head
    of the 32-layer 1-bpd model over a 131072-token cache that the oracle itself encodes
    (setup, untimed); each step is one oracle decode of that head.  The head's context is
    cut to the first T_s tokens, T_s = T * 40 / (steps + warmup) rounded to whole pages,
    when more than 40 steps are asked for, so that a long run stays within minutes."""
    from oracle import attention as oatt
    from oracle import calibration as ocal
    from oracle import codec as ocodec
    w = synth.WORKLOADS[args.workload]
    k_cal, v_cal, q_cal = synth.calibration_set(w, layers=[0])
    units = ocal.calibrate(k_cal, v_cal, q_cal, 1, w.n_kv_heads, bpd=w.bpd, seed=w.seed)
    T = w.seq_len
    uK, uV = units[0], units[1]
    codes = []
    for kind, u in ((0, uK), (1, uV)):
        x = synth.cache_tokens(w, 0, 0, kind, T)
        codes.append(ocodec.encode_tokens(x, ocodec.to_bf16(u["M"].astype(np.float32)), u["inv_delta"], u["b"]))
    pages = [ocodec.pack_sequence(c, kind, u["b"]) for kind, (c, u) in enumerate(zip(codes, (uK, uV)))]
    q = synth.decode_queries(w, 0)[:w.group].astype(np.float64)
    M = [dict(M=u["M"].astype(np.float32), delta=np.float32(u["delta"]), b=u["b"]) for u in (uK, uV)]

    n_total = args.steps + args.warmup
    Ts = T if n_total <= 40 else max(128, (T * 40 // n_total) // 128 * 128)
    n_pg = (Ts + 127) // 128

    def step():
        ck = ocodec.unpack_sequence(pages[0][:n_pg], 0, uK["r"], uK["b"], Ts)
        cv = ocodec.unpack_sequence(pages[1][:n_pg], 1, uV["r"], uV["b"], Ts)
        return oatt.decode_head(q, ck, cv, M[0], M[1], 1 / math.sqrt(128))

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    b = sum(Ts * u["r"] * u["b"] // 8 + u["r"] * 128 * 4 for u in (uK, uV))
    value = b / dt / 1e9
    cores = host_cores()
    sample = (f"1 KV head (G={w.group} queries) of layer 0 over the first {Ts} tokens of a {T}-token cache "
              "encoded by the oracle; unpack + fp64 d-space attention per step")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "seq_len": T, "sample": sample},
            "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DECODE_WORKLOAD)
    ap.add_argument("--no-encode", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="encode measurement only (profiling)")
    ap.add_argument("--encode-layers", type=int, default=0, help="limit the encode workload's layers")
    ap.add_argument("--layers", type=int, default=0, help="limit the decode workload's layers (profiling)")
    ap.add_argument("--seq-len", type=int, default=0, help="override the decode workload's context (profiling)")
    ap.add_argument("--bpd", type=float, default=0.0,
                    help="override the decode workload's budget (e.g. the 16 x 32k sweep at 0.5/1/2/4)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--k-only", action="store_true",
                    help="keys-only plan: keys coded at the budget, values stored as fp16")
    ap.add_argument("--no-sdpa", action="store_true", help="skip the fp16 SDPA context timing")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other decode workloads (32k layer, 16 x 32k budget sweep, keys-only, Qwen decode)")
    ap.add_argument("--efficiency", action="store_true",
                    help="only the project page's Efficiency table (fixed r, b vs fp16 SDPA, 32k-128k)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    import torch
    if args.efficiency:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        print(json.dumps({"efficiency_table": efficiency_table(torch)}), flush=True)
        return
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as td
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = td
    res = run_ours(args, torch, dist, rank, world)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
