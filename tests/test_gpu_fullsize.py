"""GPU parity at the workloads' full sizes, in the launch configuration bench.py times:
the whole-model plan (C1 + C2 over every layer), caches of the full context written by
the tensor-core prefill, one decode call per tested layer over all KV heads.  The oracle
checks samples it can afford one by one: whole pages of codes (byte for byte against
its canonical encode of the same tokens) and the attention outputs of sampled KV heads
(within 2e-3, the bound of test_gpu_parity.py) over the pages the GPU wrote.

Workloads: llama8b-32L-128k-1bpd (the bench's decode step), llama8b-32L-b16x32k at
0.5 / 1 / 2 / 4 bpd (16 sequences), qwen7b-28L-128k-2bpd (query groups of 7)."""

import math

import numpy as np
import pytest
import torch

from bit_quantization_head_b200 import kvtc
from bit_quantization_head_b200 import synth
from oracle import attention as oatt
from oracle import codec as ocodec
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu
TOL = 2e-3
P = 128


def _plan(w):
    k, v, q = synth.calibration_set(w)
    return kvtc.kvtc_calibrate(k, v, q, n_layers=w.n_layers, n_kv_heads=w.n_kv_heads, group=w.group,
                               bpd=w.bpd, seed=w.seed).upload()


def _encode_layers(w, plan, layers, n_seq, T, keep=(0,)):
    """Prefill every tested layer of every sequence; returns the cache and the host
    copies of K and V of the sequences in ``keep``: (layer, seq) -> (K, V) as fp32 numpy
    [T, H, d] (the bf16 values the GPU encoded)."""
    pages = (T + P - 1) // P
    bt = torch.arange(n_seq * pages, dtype=torch.int32).reshape(n_seq, pages)
    cache = kvtc.Cache(plan, n_seq * pages, bt)
    specs = {(l, h, kd): synth.unit_spec(w, l, h, kd) for l in layers for h in range(w.n_kv_heads)
             for kd in (0, 1)}
    host = {}
    for layer in layers:
        for s in range(n_seq):
            k, v = synth.layer_kv_torch(w, layer, T, torch.device("cuda"), seq=s, specs=specs)
            kvtc.kvtc_encode_prefill(plan, cache, layer, k, v, s, 0)
            if s in keep:
                host[layer, s] = (k.float().cpu().numpy(), v.float().cpu().numpy())
            del k, v
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    return cache, host


def _check_sampled_pages(plan, cache, host, layer, s, H, page_ids):
    units = gh.plan_units(plan)
    for h in range(H):
        for kind in (0, 1):
            u = (layer * H + h) * 2 + kind
            x = host[layer, s][kind]
            got = gh.gpu_pages(cache, plan, u, s, max(page_ids) + 1)
            for p in page_ids:
                codes = gh.oracle_codes(x[p * P:(p + 1) * P, h], units[u], "bf16")
                want = ocodec.pack_page(codes, kind, units[u]["b"])
                assert np.array_equal(want, got[p]), (layer, s, h, kind, p)


def _check_sampled_heads(plan, cache, layer, w, seqs, heads, T, n_seq):
    H, G = w.n_kv_heads, w.group
    q = np.stack([synth.decode_queries(w, layer, s) for s in range(n_seq)])
    got = gh.run_decode(plan, cache, layer, q, [T] * n_seq, "f32", "bf16")
    units = gh.plan_units(plan)
    n_pages = (T + P - 1) // P
    for s in seqs:
        for h in heads:
            uK, uV = (layer * H + h) * 2, (layer * H + h) * 2 + 1
            ck = ocodec.unpack_sequence(gh.gpu_pages(cache, plan, uK, s, n_pages), 0, units[uK]["r"],
                                        units[uK]["b"], T)
            cv = ocodec.unpack_sequence(gh.gpu_pages(cache, plan, uV, s, n_pages), 1, units[uV]["r"],
                                        units[uV]["b"], T)
            qh = synth.round_dtype(q[s, h * G:(h + 1) * G], "bf16").astype(np.float64)
            ref = oatt.decode_head(qh, ck, cv, units[uK], units[uV], 1 / math.sqrt(128))
            ab, rel = gh.decode_errors(got[s, h * G:(h + 1) * G], ref)
            assert ab <= TOL and rel <= TOL, (layer, s, h, ab, rel)
    assert int(cache.status.item()) == 0


def test_llama_32_layers_128k_1bpd_sampled():
    w = synth.WORKLOADS["llama8b-32L-128k-1bpd"]
    plan = _plan(w)
    T = w.seq_len
    layers = [0, 31]
    cache, host = _encode_layers(w, plan, layers, 1, T)
    for layer in layers:
        _check_sampled_pages(plan, cache, host, layer, 0, w.n_kv_heads, [0, 511, 1023])
        _check_sampled_heads(plan, cache, layer, w, [0], [0, 5], T, 1)


@pytest.mark.parametrize("bpd", [0.5, 1.0, 2.0, 4.0])
def test_llama_batch16_32k_budgets_sampled(bpd):
    w = synth.with_bpd(synth.WORKLOADS["llama8b-32L-b16x32k"], bpd)
    plan = _plan(w)
    T, n_seq = w.seq_len, w.batch
    layers = [17]
    cache, host = _encode_layers(w, plan, layers, n_seq, T, keep=(0, 15))
    for s in (0, 15):
        _check_sampled_pages(plan, cache, host, 17, s, w.n_kv_heads, [0, 255])
    _check_sampled_heads(plan, cache, 17, w, [0, 7, 15], [3], T, n_seq)


def test_qwen_28_layers_128k_2bpd_sampled():
    w = synth.WORKLOADS["qwen7b-28L-128k-2bpd"]
    plan = _plan(w)
    T = w.seq_len
    layers = [27]
    cache, host = _encode_layers(w, plan, layers, 1, T)
    _check_sampled_pages(plan, cache, host, 27, 0, w.n_kv_heads, [0, 700, 1023])
    _check_sampled_heads(plan, cache, 27, w, [0], [1, 3], T, 1)
