"""GPU parity: the CUDA path (through the C ABI) against the oracle on the same seeded
inputs.  Codes and bit layout must be identical byte for byte; attention outputs must
agree within 2e-3 of the oracle's result, read as max |o_gpu - o_oracle| <= 2e-3 *
max |o_oracle| per (sequence, query head) output vector (and <= 2e-3 absolute).  For a
bf16 output one bf16 rounding (2^-8 relative) is added to the bound."""

import numpy as np
import pytest
import torch

from bit_quantization_head_b200 import kvtc
from bit_quantization_head_b200 import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _calibrated(w, layers=None):
    k, v, q = synth.calibration_set(w, layers)
    nl = k.shape[0]
    plan = kvtc.kvtc_calibrate(k, v, q, n_layers=nl, n_kv_heads=w.n_kv_heads, group=w.group, bpd=w.bpd,
                               seed=w.seed, fixed_r=w.fixed_r, fixed_b=w.fixed_b)
    return plan.upload()


def _kv(w, layer, T, seq=0):
    K = np.stack([synth.cache_tokens(w, layer, h, 0, T, seq) for h in range(w.n_kv_heads)], axis=1)
    V = np.stack([synth.cache_tokens(w, layer, h, 1, T, seq) for h in range(w.n_kv_heads)], axis=1)
    return K, V


def _check_decode(plan, cache, layer, q, seq_lens, H, G, q_dtype):
    ref = gh.oracle_decode(plan, cache, layer, q.astype(np.float64), seq_lens, H, G)
    got = gh.run_decode(plan, cache, layer, q, seq_lens, "f32", q_dtype)
    ab, rel = gh.decode_errors(got, ref)
    assert ab <= TOL and rel <= TOL, (ab, rel)
    got16 = gh.run_decode(plan, cache, layer, q, seq_lens, "bf16", q_dtype)
    bound = TOL * np.abs(ref).max(axis=-1, keepdims=True) + 2.0 ** -8 * np.abs(ref)
    assert np.all(np.abs(got16 - ref) <= bound + 1e-30)
    assert int(cache.status.item()) == 0
    return ab, rel


def test_head1_fp32_codes_and_attention():
    w = synth.WORKLOADS["head1-fp32-1k"]
    plan = _calibrated(w)
    rng = np.random.default_rng(0)
    cache = gh.make_cache(plan, [w.seq_len], rng)
    K, V = _kv(w, 0, w.seq_len)
    gh.encode_all(plan, cache, 0, [(K, V)], "f32")
    assert gh.check_encode(plan, cache, 0, [(K, V)], "f32", 1) == 0
    q = synth.decode_queries(w, 0)[None]
    _check_decode(plan, cache, 0, q, [w.seq_len], 1, 1, "f32")


def test_llama_layer_32k_2bpd_codes_and_attention():
    w = synth.WORKLOADS["llama8b-layer-32k-2bpd"]
    plan = _calibrated(w)
    bs = {plan.unit(u)["b"] for u in range(16)}
    assert len(bs) >= 2            # a real mix of widths from C2
    # the plan the GPU runs with is the oracle's calibration of the same inputs: identical
    # (r, b) per unit, and M within 1e-6 of the oracle's normwise
    from oracle import calibration as ocal
    k, v, q = synth.calibration_set(w)
    units = ocal.calibrate(k, v, q, 1, w.n_kv_heads, bpd=w.bpd, seed=w.seed)
    for u, ou in enumerate(units):
        info = plan.unit(u)
        assert (info["r"], info["b"]) == (ou["r"], ou["b"]), u
        assert np.abs(plan.matrix(u) - ou["M"]).max() <= 1e-6 * np.abs(ou["M"]).max(), u
    rng = np.random.default_rng(1)
    cache = gh.make_cache(plan, [w.seq_len], rng)
    K, V = _kv(w, 0, w.seq_len)
    gh.encode_all(plan, cache, 0, [(K, V)], "bf16")
    assert gh.check_encode(plan, cache, 0, [(K, V)], "bf16", 8) == 0
    q = synth.decode_queries(w, 0)[None]
    _check_decode(plan, cache, 0, q, [w.seq_len], 8, 4, "bf16")


PAIRS = [((16, 2), (16, 2)), ((6, 3), (18, 5)), ((126, 4), (2, 8)), ((10, 5), (128, 3)),
         ((34, 6), (20, 7)), ((2, 7), (64, 6)), ((128, 8), (96, 4)), ((64, 2), (128, 8)),
         ((50, 2), (34, 2))]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_every_code_width_ragged_sequences_and_chunked_appends(dtype):
    rng = np.random.default_rng(2)
    H, G = len(PAIRS), 3
    plan = gh.random_plan(1, H, G, PAIRS, rng)
    lens = [1000, 0, 129, 2500]
    cache = gh.make_cache(plan, lens, rng)
    kv = []
    for T in lens:
        K = (rng.standard_normal((T, H, 128)) * rng.uniform(0.3, 3.0, (1, H, 1))).astype(np.float32)
        V = (rng.standard_normal((T, H, 128)) * rng.uniform(0.3, 3.0, (1, H, 1))).astype(np.float32)
        kv.append((synth.round_dtype(K, dtype), synth.round_dtype(V, dtype)))
    gh.encode_all(plan, cache, 0, kv, dtype, chunk=300)
    assert gh.check_encode(plan, cache, 0, kv, dtype, H) == 0
    q = (rng.standard_normal((len(lens), H * G, 128)) * 0.5).astype(np.float32)
    q = synth.round_dtype(q, dtype)
    _check_decode(plan, cache, 0, q, lens, H, G, dtype)


@pytest.mark.parametrize("G", [2, 6])
def test_every_pair_of_key_and_value_widths(G):
    # one KV head per (b_K, b_V) pair of 2..8 (each pair is its own kernel variant; G = 2
    # runs the packed score mode, G = 6 the unpacked one), random even ranks from 2 to 128
    rng = np.random.default_rng(20 + G)
    pairs = []
    for bk in range(2, 9):
        for bv in range(2, 9):
            rk, rv = (int(x) for x in 2 * rng.integers(1, 65, 2))
            pairs.append(((rk, bk), (rv, bv)))
    H = len(pairs)
    plan = gh.random_plan(1, H, G, pairs, rng)
    lens = [700, 129]
    cache = gh.make_cache(plan, lens, rng)
    kv = [((rng.standard_normal((T, H, 128)) * 1.5).astype(np.float32),
           (rng.standard_normal((T, H, 128)) * 1.5).astype(np.float32)) for T in lens]
    gh.encode_all(plan, cache, 0, kv, "f32")
    q = (rng.standard_normal((len(lens), H * G, 128)) * 0.5).astype(np.float32)
    _check_decode(plan, cache, 0, q, lens, H, G, "f32")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_keys_only_raw_values_codes_and_attention(dtype):
    # keys-only plans: coded keys of several widths, values stored as fp16 (raw pages);
    # packed (G = 4) and unpacked (G = 6) query groups
    rng = np.random.default_rng(12)
    for G in (4, 6):
        pairs = [((16, 2), (128, 16)), ((34, 3), (128, 16)), ((64, 4), (128, 16)), ((8, 8), (128, 16))]
        H = len(pairs)
        plan = gh.random_plan(1, H, G, pairs, rng)
        lens = [777, 130, 0]
        cache = gh.make_cache(plan, lens, rng)
        kv = []
        for T in lens:
            K = (rng.standard_normal((T, H, 128)) * rng.uniform(0.3, 3.0, (1, H, 1))).astype(np.float32)
            V = (rng.standard_normal((T, H, 128)) * rng.uniform(0.3, 3.0, (1, H, 1))).astype(np.float32)
            kv.append((synth.round_dtype(K, dtype), synth.round_dtype(V, dtype)))
        gh.encode_all(plan, cache, 0, kv, dtype, chunk=200)
        assert gh.check_encode(plan, cache, 0, kv, dtype, H) == 0
        q = synth.round_dtype((rng.standard_normal((len(lens), H * G, 128)) * 0.7).astype(np.float32), dtype)
        _check_decode(plan, cache, 0, q, lens, H, G, dtype)


def test_keys_only_calibrated_llama_layer():
    w = synth.WORKLOADS["llama8b-layer-32k-2bpd"]
    k, v, q = synth.calibration_set(w)
    plan = kvtc.kvtc_calibrate(k, v, q, n_layers=1, n_kv_heads=w.n_kv_heads, group=w.group, bpd=w.bpd,
                               seed=w.seed, k_only=True).upload()
    rng = np.random.default_rng(13)
    T = 5000
    cache = gh.make_cache(plan, [T], rng)
    K, V = _kv(w, 0, T)
    gh.encode_all(plan, cache, 0, [(K, V)], "bf16")
    assert gh.check_encode(plan, cache, 0, [(K, V)], "bf16", w.n_kv_heads) == 0
    with pytest.raises(kvtc.KvtcError):   # prefill encodes compressed units only
        kvtc.kvtc_encode_prefill(plan, cache, 0, gh.to_dev(K, "bf16"), gh.to_dev(V, "bf16"), 0, 0)
    q = synth.decode_queries(w, 0)[None]
    _check_decode(plan, cache, 0, q, [T], w.n_kv_heads, w.group, "bf16")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_debug_latent_is_the_canonical_projection(dtype):
    # the fp32 latents the append quantizes, bit for bit against the oracle's canonical
    # projection; the oracle's quantizer applied to them gives the canonical codes
    from oracle import codec as ocodec
    rng = np.random.default_rng(14)
    plan = gh.random_plan(1, 2, 1, [((34, 3), (128, 16)), ((128, 8), (16, 2))], rng)
    n = 300
    x = synth.round_dtype((rng.standard_normal((n, 128)) * 2).astype(np.float32), dtype)
    for h in range(2):
        for kind in (0, 1):
            u = h * 2 + kind
            info = plan.unit(u)
            M = plan.matrix(u)
            y = torch.empty((n, info["r"]), dtype=torch.float32, device="cuda")
            kvtc.kvtc_debug_encode_latent(plan, 0, h, kind, gh.to_dev(x, dtype), y)
            torch.cuda.synchronize()
            got = y.cpu().numpy()
            if info["b"] == kvtc.RAW_BITS:
                want = x.astype(np.float32)
            else:
                Mop = ocodec.to_bf16(M) if dtype == "bf16" else M.astype(np.float32)
                want = ocodec.project_canonical(x, Mop).astype(np.float32)
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (h, kind)
            if info["b"] != kvtc.RAW_BITS:
                unit = dict(info, M=M)
                assert np.array_equal(ocodec.quantize(got, np.float32(info["inv_delta"]), info["b"]),
                                      gh.oracle_codes(x, unit, dtype))


def test_query_groups_larger_than_eight_and_peaked_attention():
    rng = np.random.default_rng(3)
    H, G = 2, 12
    plan = gh.random_plan(1, H, G, [((32, 4), (32, 4)), ((64, 2), (48, 3))], rng)
    lens = [700, 3000]
    cache = gh.make_cache(plan, lens, rng)
    kv = [(rng.standard_normal((T, H, 128)).astype(np.float32),
           rng.standard_normal((T, H, 128)).astype(np.float32)) for T in lens]
    gh.encode_all(plan, cache, 0, kv, "f32")
    assert gh.check_encode(plan, cache, 0, kv, "f32", H) == 0
    q = (rng.standard_normal((2, H * G, 128)) * 3.0).astype(np.float32)   # sharp softmax
    _check_decode(plan, cache, 0, q, lens, H, G, "f32")


@pytest.mark.parametrize("G", [6, 12])
def test_shared_merge_over_long_contexts_and_head_groups(G):
    # 33k tokens give the launch 33 splits per KV head, so the merge is shared by the last
    # CTAs of each head group (one query head each; G = 12 has groups of 8 and 4, G = 6
    # one group of 6, unpacked); the short third sequence leaves most of its splits empty
    rng = np.random.default_rng(40 + G)
    H = 2
    plan = gh.random_plan(1, H, G, [((48, 2), (40, 2)), ((96, 3), (128, 4))], rng)
    lens = [20000, 33000, 700]
    cache = gh.make_cache(plan, lens, rng)
    kv = [(rng.standard_normal((T, H, 128)).astype(np.float32),
           rng.standard_normal((T, H, 128)).astype(np.float32)) for T in lens]
    gh.encode_all(plan, cache, 0, kv, "f32", path="prefill")
    q = (rng.standard_normal((len(lens), H * G, 128)) * 1.5).astype(np.float32)
    _check_decode(plan, cache, 0, q, lens, H, G, "f32")


def test_out_of_range_pages_and_positions_set_status_bits():
    rng = np.random.default_rng(4)
    plan = gh.random_plan(1, 1, 1, [((16, 2), (16, 2))], rng)
    bt = torch.tensor([[0, 1, 99]], dtype=torch.int32)           # page 99 is outside the pool
    cache = kvtc.Cache(plan, 3, bt)
    K = rng.standard_normal((300, 1, 128)).astype(np.float32)
    gh.encode_all(plan, cache, 0, [(K, K)], "f32")
    torch.cuda.synchronize()
    assert int(cache.status.item()) & kvtc.STATUS_BAD_PAGE
    cache.status.zero_()
    # position beyond the block table: 3 pages = 384 tokens, start at 380, 10 tokens
    k = gh.to_dev(K[:10], "f32")
    kvtc.kvtc_encode_append(plan, cache, 0, k, k, torch.tensor([0, 10], dtype=torch.int32).cuda(),
                            torch.tensor([380], dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert int(cache.status.item()) & kvtc.STATUS_BAD_POS
    cache.status.zero_()
    q = rng.standard_normal((1, 1, 128)).astype(np.float32)
    out = gh.run_decode(plan, cache, 0, q, [300])
    assert int(cache.status.item()) & kvtc.STATUS_BAD_PAGE
    assert np.all(np.isfinite(out))


def test_decode_rejects_short_workspace_and_long_max_seq_len():
    rng = np.random.default_rng(5)
    plan = gh.random_plan(1, 1, 1, [((16, 2), (16, 2))], rng)
    cache = gh.make_cache(plan, [256], rng)
    q = torch.zeros((1, 1, 128), device="cuda")
    out = torch.zeros((1, 1, 128), device="cuda")
    sl = torch.tensor([256], dtype=torch.int32, device="cuda")
    ws = torch.empty(8, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvtc.KvtcError) as e:
        kvtc.kvtc_decode_attention(plan, cache, 0, q, sl, 256, out, ws)
    assert e.value.status == 5
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvtc.KvtcError) as e:
        kvtc.kvtc_decode_attention(plan, cache, 0, q, sl, 100000, out, ws)
    assert e.value.status == 1


# ---------------------------------------------------------------- tensor-core prefill
def test_prefill_tensor_core_codes_equal_canonical_codes_llama_layer():
    w = synth.WORKLOADS["llama8b-layer-32k-2bpd"]
    plan = _calibrated(w)
    rng = np.random.default_rng(6)
    T = 8192
    cache = gh.make_cache(plan, [T], rng)
    K, V = _kv(w, 0, T)
    gh.encode_all(plan, cache, 0, [(K, V)], "bf16", path="prefill")
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    assert gh.check_encode(plan, cache, 0, [(K, V)], "bf16", 8) == 0


def test_prefill_every_code_width_and_partial_last_page():
    rng = np.random.default_rng(7)
    H = len(PAIRS)
    plan = gh.random_plan(1, H, 2, PAIRS, rng)
    lens = [1000, 129, 256]
    cache = gh.make_cache(plan, lens, rng)
    kv = []
    for T in lens:
        K = (rng.standard_normal((T, H, 128)) * rng.uniform(0.3, 3.0, (1, H, 1))).astype(np.float32)
        V = (rng.standard_normal((T, H, 128)) * rng.uniform(0.3, 3.0, (1, H, 1))).astype(np.float32)
        kv.append((synth.round_dtype(K, "bf16"), synth.round_dtype(V, "bf16")))
    gh.encode_all(plan, cache, 0, kv, "bf16", path="prefill")
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    assert gh.check_encode(plan, cache, 0, kv, "bf16", H) == 0


def test_prefill_and_append_write_identical_pools_on_long_span():
    w = synth.WORKLOADS["qwen7b-28L-128k-2bpd"]
    plan = _calibrated(w, layers=[0])
    T = 32768 + 77
    dev = torch.device("cuda")
    k, v = synth.layer_kv_torch(w, 0, T, dev)
    rng = np.random.default_rng(8)
    c1 = gh.make_cache(plan, [T], rng)
    c2 = kvtc.Cache(plan, c1.pages_per_unit, c1.block_table.cpu())
    kvtc.kvtc_encode_prefill(plan, c1, 0, k, v, 0, 0)
    kvtc.kvtc_encode_append(plan, c2, 0, k, v, torch.tensor([0, T], dtype=torch.int32, device=dev),
                            torch.tensor([0], dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert int(c1.status.item()) == 0 and int(c2.status.item()) == 0
    assert torch.equal(c1.pool, c2.pool)
