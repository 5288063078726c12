"""GPU parity of the pre-RoPE decode (KV-COBRA project page, Results: keys compressed
before the rotary position embedding): kvtc_decode_attention_rope against the oracle's
decode_head_prerope (reconstructed keys rotated to their positions in fp64, textbook
softmax attention), over the pages the GPU wrote.  Tolerance as the other decode tests:
max |o - o_ref| <= 2e-3 max |o_ref| per (sequence, query head) and <= 2e-3 absolute."""

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


def _oracle_rope(plan, cache, layer, q, seq_lens, H, G, base, heads=None):
    units = gh.plan_units(plan)
    out = np.zeros((len(seq_lens), H * G, 128))
    for s, T in enumerate(seq_lens):
        n_pages = (T + 127) // 128
        for h in (range(H) if heads is None else heads):
            uK, uV = (layer * H + h) * 2, (layer * H + h) * 2 + 1
            ck = ocodec.unpack_sequence(gh.gpu_pages(cache, plan, uK, s, n_pages), 0, units[uK]["r"], units[uK]["b"], T)
            cv = ocodec.unpack_sequence(gh.gpu_pages(cache, plan, uV, s, n_pages), 1, units[uV]["r"], units[uV]["b"], T)
            out[s, h * G:(h + 1) * G] = oatt.decode_head_prerope(q[s, h * G:(h + 1) * G], ck, cv, units[uK], units[uV],
                                                                 1 / math.sqrt(128), base=base)
    return out


def _run_rope(plan, cache, layer, q, seq_lens, q_dtype, out_dtype="f32", base=0.0):
    qd = gh.to_dev(q, q_dtype)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    mx = max(seq_lens + [0])
    ws = torch.zeros(max(1, kvtc.kvtc_decode_workspace_bytes(plan, len(seq_lens), mx)), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((len(seq_lens), q.shape[1], 128), dtype=torch.float32 if out_dtype == "f32" else torch.bfloat16,
                      device="cuda")
    kvtc.kvtc_decode_attention_rope(plan, cache, layer, qd, sl, mx, out, ws, rope_base=base)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rope_decode_every_code_width_ragged_sequences(dtype):
    rng = np.random.default_rng(31)
    pairs = [((16, 2), (16, 2)), ((6, 3), (18, 5)), ((126, 4), (2, 8)), ((34, 6), (20, 7)),
             ((128, 8), (96, 4)), ((64, 2), (128, 8)), ((50, 2), (34, 2)), ((32, 2), (128, 16))]
    H, G = len(pairs), 3
    plan = gh.random_plan(1, H, G, pairs, rng)
    lens = [1000, 0, 129, 2500]
    cache = gh.make_cache(plan, lens, rng)
    kv = []
    for T in lens:
        K = (rng.standard_normal((T, H, 128)) * rng.uniform(0.3, 3.0, (1, H, 1))).astype(np.float32)
        V = (rng.standard_normal((T, H, 128)) * rng.uniform(0.3, 3.0, (1, H, 1))).astype(np.float32)
        kv.append((synth.round_dtype(K, dtype), synth.round_dtype(V, dtype)))
    gh.encode_all(plan, cache, 0, kv, dtype, chunk=300)
    q = synth.round_dtype((rng.standard_normal((len(lens), H * G, 128)) * 0.5).astype(np.float32), dtype)
    ref = _oracle_rope(plan, cache, 0, q.astype(np.float64), lens, H, G, oatt.ROPE_BASE)
    got = _run_rope(plan, cache, 0, q, lens, dtype)
    ab, rel = gh.decode_errors(got, ref)
    assert ab <= TOL and rel <= TOL, (ab, rel)
    assert np.all(got[1] == 0.0)          # the empty sequence
    got16 = _run_rope(plan, cache, 0, q, lens, dtype, "bf16")
    bound = TOL * np.abs(ref).max(axis=-1, keepdims=True) + 2.0 ** -8 * np.abs(ref)
    assert np.all(np.abs(got16 - ref) <= bound + 1e-30)
    assert int(cache.status.item()) == 0


def test_rope_decode_other_base_sharp_softmax_and_eight_query_heads():
    rng = np.random.default_rng(32)
    H, G = 2, 8
    plan = gh.random_plan(1, H, G, [((32, 4), (32, 4)), ((64, 2), (48, 3))], rng)
    lens = [700, 3000]
    cache = gh.make_cache(plan, lens, rng)
    kv = [(rng.standard_normal((T, H, 128)).astype(np.float32), rng.standard_normal((T, H, 128)).astype(np.float32))
          for T in lens]
    gh.encode_all(plan, cache, 0, kv, "f32")
    q = (rng.standard_normal((2, H * G, 128)) * 2.0).astype(np.float32)
    for base in (10000.0, 500000.0):
        ref = _oracle_rope(plan, cache, 0, q.astype(np.float64), lens, H, G, base)
        got = _run_rope(plan, cache, 0, q, lens, "f32", base=base)
        ab, rel = gh.decode_errors(got, ref)
        assert ab <= TOL and rel <= TOL, (base, ab, rel)


def test_rope_decode_calibrated_llama_layer_32k():
    # the 32k Llama-shaped layer at 2 bpd (C1 + C2 widths), whole layer against the oracle
    w = synth.WORKLOADS["llama8b-layer-32k-2bpd"]
    k, v, qc = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k, v, qc, n_layers=1, n_kv_heads=w.n_kv_heads, group=w.group, bpd=w.bpd,
                               seed=w.seed).upload()
    rng = np.random.default_rng(33)
    T = w.seq_len
    cache = gh.make_cache(plan, [T], rng)
    K = np.stack([synth.cache_tokens(w, 0, h, 0, T) for h in range(w.n_kv_heads)], axis=1)
    V = np.stack([synth.cache_tokens(w, 0, h, 1, T) for h in range(w.n_kv_heads)], axis=1)
    gh.encode_all(plan, cache, 0, [(K, V)], "bf16", path="prefill")
    q = synth.decode_queries(w, 0)[None]
    ref = _oracle_rope(plan, cache, 0, q.astype(np.float64), [T], w.n_kv_heads, w.group, oatt.ROPE_BASE)
    got = _run_rope(plan, cache, 0, q, [T], "bf16")
    ab, rel = gh.decode_errors(got, ref)
    assert ab <= TOL and rel <= TOL, (ab, rel)


def test_rope_decode_128k_sampled_heads():
    # one 131072-token layer of the 32-layer 1-bpd Llama plan (positions up to 131071,
    # where the page angles need the fp64 reduction); heads 0 and 5 checked in full
    w = synth.WORKLOADS["llama8b-32L-128k-1bpd"]
    k, v, qc = synth.calibration_set(w, layers=[0])
    plan = kvtc.kvtc_calibrate(k, v, qc, n_layers=1, n_kv_heads=w.n_kv_heads, group=w.group, bpd=w.bpd,
                               seed=w.seed).upload()
    T = w.seq_len
    dev = torch.device("cuda")
    kt, vt = synth.layer_kv_torch(w, 0, T, dev)
    bt = torch.arange(T // 128, dtype=torch.int32).reshape(1, -1)
    cache = kvtc.Cache(plan, T // 128, bt)
    kvtc.kvtc_encode_prefill(plan, cache, 0, kt, vt, 0, 0)
    del kt, vt
    q = synth.decode_queries(w, 0)[None]
    got = _run_rope(plan, cache, 0, q, [T], "bf16")
    ref = _oracle_rope(plan, cache, 0, q.astype(np.float64), [T], w.n_kv_heads, w.group, oatt.ROPE_BASE,
                       heads=[0, 5])
    for h in (0, 5):
        sl = slice(h * w.group, (h + 1) * w.group)
        ab, rel = gh.decode_errors(got[:, sl], ref[:, sl])
        assert ab <= TOL and rel <= TOL, (h, ab, rel)
