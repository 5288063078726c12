"""GPU parity on the quantizer's special inputs ("How KV-COBRA Works", Inference: the
head's b*-bit uniform quantizer; canonical fp32 arithmetic with floor, NaN -> 0 and
+-Inf -> the end codes) and on the tensor-core encoder's slow paths: rows with NaN, +Inf,
-Inf, +-0 and huge finite values, latents placed exactly on quantizer thresholds (and
one ulp either side), rows of tiny values whose squared norm underflows, and a page whose
every code lies on a threshold (more flagged codes than the recompute queue holds).
Both encoders are compared byte for byte with the oracle's codes; the layer is then
decoded and checked against the oracle over the pages the GPU wrote."""

import numpy as np
import pytest
import torch

from bit_quantization_head_b200 import kvtc
from bit_quantization_head_b200 import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu
TOL = 2e-3
BF16_MAX = float(np.array([0x7F7F0000], dtype=np.uint32).view(np.float32)[0])


def _decode_matches(plan, cache, kv_lens, H, G, rng, dtype):
    q = synth.round_dtype((rng.standard_normal((len(kv_lens), H * G, 128)) * 0.5).astype(np.float32), dtype)
    ref = gh.oracle_decode(plan, cache, 0, q.astype(np.float64), kv_lens, H, G)
    got = gh.run_decode(plan, cache, 0, q, kv_lens, "f32", dtype)
    assert np.all(np.isfinite(got))
    ab, rel = gh.decode_errors(got, ref)
    assert ab <= TOL and rel <= TOL, (ab, rel)


def _special_rows(rng, T, H, big):
    """Gaussian rows with special values planted in some of them."""
    X = (rng.standard_normal((T, H, 128)) * 0.7).astype(np.float32)
    for t in range(0, T, 7):
        h = t % H
        kind = (t // 7) % 8
        if kind == 0:
            X[t, h, rng.integers(128)] = np.nan
        elif kind == 1:
            X[t, h, rng.integers(128)] = np.inf
        elif kind == 2:
            X[t, h, rng.integers(128)] = -np.inf
        elif kind == 3:
            X[t, h] = 0.0
        elif kind == 4:
            X[t, h] = -0.0
        elif kind == 5:
            X[t, h, rng.integers(128, size=3)] = big * np.array([1.0, -1.0, 1.0], np.float32)
        elif kind == 6:
            X[t, h] = np.float32(1e-30) * rng.standard_normal(128).astype(np.float32)  # ||x||^2 underflows
        else:
            X[t, h, rng.integers(128)] = -big
    return X


@pytest.mark.parametrize("dtype,path", [("bf16", "append"), ("bf16", "prefill"), ("f32", "append")])
def test_special_values_encode_bit_exact_and_decode_finite(dtype, path):
    rng = np.random.default_rng(21)
    pairs = [((16, 2), (32, 4)), ((24, 3), (16, 8)), ((64, 5), (40, 2))]
    H, G = len(pairs), 4
    plan = gh.random_plan(1, H, G, pairs, rng)
    lens = [128 * 4 + 40, 256]
    cache = gh.make_cache(plan, lens, rng)
    big = BF16_MAX if dtype == "bf16" else np.float32(3e38)
    kv = []
    for T in lens:
        K = synth.round_dtype(_special_rows(rng, T, H, big), dtype)
        V = synth.round_dtype(_special_rows(rng, T, H, big), dtype)
        kv.append((K, V))
    gh.encode_all(plan, cache, 0, kv, dtype, path=path)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    assert gh.check_encode(plan, cache, 0, kv, dtype, H) == 0
    _decode_matches(plan, cache, lens, H, G, rng, dtype)


def _threshold_plan(rng, pairs, delta):
    """Units whose M rows are distinct unit vectors (y_j = x_perm(j) exactly, in both the
    canonical chain and a bf16 tensor-core sum) with a power-of-two step, so a chosen x
    puts y * inv_delta + 2^(b-1) exactly on an integer."""
    r, b, dl, M, perms = [], [], [], [], []
    for (rk, bk), (rv, bv) in pairs:
        for rr, bb in ((rk, bk), (rv, bv)):
            perm = rng.permutation(128)[:rr]
            m = np.zeros((rr, 128), np.float32)
            m[np.arange(rr), perm] = 1.0
            r.append(rr)
            b.append(bb)
            dl.append(delta)
            M.append(m)
            perms.append(perm)
    plan = kvtc.kvtc_plan_create(1, len(pairs), 2, r, b, dl, M).upload()
    return plan, perms


def _on_thresholds(rng, T, H, plan, perms, kind, delta, every=True):
    X = (rng.standard_normal((T, H, 128)) * 0.3).astype(np.float32)
    for h in range(H):
        u = h * 2 + kind
        bb = plan.unit(u)["b"]
        for t in range(T):
            if not every and t % 3:
                continue
            k = rng.integers(-2, (1 << bb) + 3, size=len(perms[u]))   # includes the clamped ends
            x = ((k - (1 << (bb - 1))) * delta).astype(np.float32)
            if not every:   # one bf16 ulp either side of some thresholds
                nud = rng.integers(-1, 2, size=len(x)).astype(np.float32)
                x = x + nud * np.abs(x) * np.float32(2.0 ** -7)
            X[t, h, perms[u]] = x
    return synth.round_dtype(X, "bf16")


@pytest.mark.parametrize("path", ["append", "prefill"])
def test_latents_exactly_on_quantizer_thresholds(path):
    rng = np.random.default_rng(22)
    pairs = [((16, 4), (32, 2)), ((20, 3), (18, 6)), ((32, 8), (16, 5))]
    H = len(pairs)
    delta = 2.0 ** -3
    plan, perms = _threshold_plan(rng, pairs, delta)
    T = 128 * 3 + 17
    cache = gh.make_cache(plan, [T], rng)
    K = _on_thresholds(rng, T, H, plan, perms, 0, delta, every=False)
    V = _on_thresholds(rng, T, H, plan, perms, 1, delta, every=False)
    kvtc.kvtc_plan_prefill_stats(plan, reset=True)
    gh.encode_all(plan, cache, 0, [(K, V)], "bf16", path=path)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    assert gh.check_encode(plan, cache, 0, [(K, V)], "bf16", H) == 0
    if path == "prefill":
        codes, fixed = kvtc.kvtc_plan_prefill_stats(plan)
        assert codes > 0 and fixed > 0   # threshold codes went through the canonical recompute
    _decode_matches(plan, cache, [T], H, 2, rng, "bf16")


def test_prefill_queue_overflow_recomputes_the_whole_item():
    # every code of the K and V units on a threshold: 128 x (16 + 32) flagged codes per
    # page exceed the 2048-entry queue, so each item goes through the full recompute
    rng = np.random.default_rng(23)
    pairs = [((16, 4), (32, 2)), ((20, 3), (18, 6))]
    H = len(pairs)
    delta = 2.0 ** -3
    plan, perms = _threshold_plan(rng, pairs, delta)
    T = 128 * 2
    cache = gh.make_cache(plan, [T], rng)
    K = _on_thresholds(rng, T, H, plan, perms, 0, delta)
    V = _on_thresholds(rng, T, H, plan, perms, 1, delta)
    kvtc.kvtc_plan_prefill_stats(plan, reset=True)
    gh.encode_all(plan, cache, 0, [(K, V)], "bf16", path="prefill")
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    assert gh.check_encode(plan, cache, 0, [(K, V)], "bf16", H) == 0
    codes, fixed = kvtc.kvtc_plan_prefill_stats(plan)
    per_item = [128 * (pairs[h][0][0] + pairs[h][1][0]) for h in range(H)]
    assert codes == 2 * sum(per_item)
    assert fixed >= 2 * sum(per_item)   # the slow path counts every code of an overflowing item
    _decode_matches(plan, cache, [T], H, 2, rng, "bf16")


def test_tiny_rows_at_a_tiny_step_keep_canonical_codes():
    # rows whose squared norm underflows fp32 (|x| ~ 2^-108) at a step small enough that
    # their latents spread over every code: both encoders keep the canonical codes (the
    # tensor-core encoder must not take such rows for zero rows)
    rng = np.random.default_rng(24)
    r, b, dl, M = [], [], [], []
    for rr, bb in ((16, 4), (32, 2), (48, 3), (24, 6)):
        Q, _ = np.linalg.qr(rng.standard_normal((128, 128)))
        r.append(rr)
        b.append(bb)
        dl.append(2.0 ** -108 * 0.4 * 2.0 ** (4 - bb))
        M.append(Q[:rr].astype(np.float32))
    plan = kvtc.kvtc_plan_create(1, 2, 2, r, b, dl, M).upload()
    T = 256 + 64
    K = synth.round_dtype((rng.standard_normal((T, 2, 128)) * 2.0 ** -108).astype(np.float32), "bf16")
    V = synth.round_dtype((rng.standard_normal((T, 2, 128)) * 2.0 ** -108).astype(np.float32), "bf16")
    for path in ("append", "prefill"):
        cache = gh.make_cache(plan, [T], rng)
        gh.encode_all(plan, cache, 0, [(K, V)], "bf16", path=path)
        torch.cuda.synchronize()
        assert int(cache.status.item()) == 0
        assert gh.check_encode(plan, cache, 0, [(K, V)], "bf16", 2) == 0, path
    # the codes really spread: not every code sits at the centre 2^(b-1)
    units = gh.plan_units(plan)
    codes = gh.oracle_codes(K[:, 0], units[0], "bf16")
    assert len(np.unique(codes)) > 4


def test_shared_merge_wait_is_bounded_and_reports_a_timeout():
    # The last CTAs of a head group wait for the group's arrival counter to reach the
    # split count before each merges its share.  A counter that starts at -2 (a workspace
    # that was not zero-filled) never gets there: the waits must end on their own, set
    # KVTC_STATUS_TIMEOUT and leave the context usable; a zero-filled workspace then
    # gives the oracle's result again.
    rng = np.random.default_rng(31)
    H, G = 1, 4
    plan = gh.random_plan(1, H, G, [((32, 2), (32, 2))], rng)
    T = 16384                       # 128 pages: 16 splits, the shared merge is on
    cache = gh.make_cache(plan, [T], rng)
    kv = [(rng.standard_normal((T, H, 128)).astype(np.float32), rng.standard_normal((T, H, 128)).astype(np.float32))]
    gh.encode_all(plan, cache, 0, kv, "f32")
    q = (rng.standard_normal((1, H * G, 128)) * 0.5).astype(np.float32)
    qd = gh.to_dev(q, "f32")
    sl = torch.tensor([T], dtype=torch.int32, device="cuda")
    ws = torch.zeros(kvtc.kvtc_decode_workspace_bytes(plan, 1, T), dtype=torch.uint8, device="cuda")
    out = torch.zeros((1, H * G, 128), dtype=torch.float32, device="cuda")
    ws.view(torch.int32)[0] = -2
    kvtc.kvtc_decode_attention(plan, cache, 0, qd, sl, T, out, ws)
    torch.cuda.synchronize()
    assert int(cache.status.item()) & kvtc.STATUS_TIMEOUT
    cache.status.zero_()
    ws.zero_()
    kvtc.kvtc_decode_attention(plan, cache, 0, qd, sl, T, out, ws)
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    assert int(ws.view(torch.int32)[:2].abs().sum().item()) == 0   # counters re-armed
    ref = gh.oracle_decode(plan, cache, 0, q.astype(np.float64), [T], H, G)
    ab, rel = gh.decode_errors(out.cpu().numpy(), ref)
    assert ab <= TOL and rel <= TOL, (ab, rel)
