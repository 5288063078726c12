"""The allocation-free decode entry point (kvtc_decode_attention_noalloc).

Callers that cannot allocate device memory (a runtime that owns every allocation, a
plugin limited to the buffers it is given) use this call: it keeps its split-K scratch
in a fixed array inside the library.  This file runs last so that a failure here comes
after every other test has run; it also passes alone in a fresh process."""

import numpy as np
import pytest
import torch

from bit_quantization_head_b200 import kvtc
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


def _workspace_decode(plan, cache, q, sl, mx):
    ws = torch.zeros(kvtc.kvtc_decode_workspace_bytes(plan, cache.block_table.shape[0], mx), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((q.shape[0], q.shape[1], 128), dtype=torch.float32, device="cuda")
    kvtc.kvtc_decode_attention(plan, cache, 0, q, sl, mx, out, ws)
    return out


def test_noalloc_decode_matches_workspace_decode_on_two_calls_in_a_row():
    # The shared scratch keeps whatever the last call left in it.  The first call is the
    # larger one (more sequences, longer context: more partial slots and tickets), the
    # second a smaller one with another query, so a call that read partials or tickets
    # left behind by the one before would show.  Both run the same kernels with the same
    # split plan as kvtc_decode_attention on a fresh workspace, so the outputs are equal
    # bit for bit.
    rng = np.random.default_rng(11)
    H, G = 3, 4
    plan = gh.random_plan(1, H, G, [((64, 2), (64, 2)), ((18, 3), (96, 4)), ((128, 2), (32, 8))], rng)
    calls = []
    for lens in ([7000, 517, 2048], [3000, 129]):
        cache = gh.make_cache(plan, lens, rng)
        kv = [(rng.standard_normal((T, H, 128)).astype(np.float32),
               rng.standard_normal((T, H, 128)).astype(np.float32)) for T in lens]
        gh.encode_all(plan, cache, 0, kv, "f32")
        q = torch.from_numpy((rng.standard_normal((len(lens), H * G, 128)) * 0.5).astype(np.float32)).cuda()
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        calls.append((cache, q, sl, max(lens)))
    for cache, q, sl, mx in calls:
        out = torch.full((q.shape[0], H * G, 128), float("nan"), dtype=torch.float32, device="cuda")
        kvtc.kvtc_decode_attention_noalloc(plan, cache, 0, q, sl, mx, out)
        ref = _workspace_decode(plan, cache, q, sl, mx)
        torch.cuda.synchronize()
        assert torch.all(torch.isfinite(out))
        assert torch.equal(out, ref)
        assert int(cache.status.item()) == 0
    # and once more with the first call's shapes, after the smaller call
    cache, q, sl, mx = calls[0]
    out = torch.empty((q.shape[0], H * G, 128), dtype=torch.float32, device="cuda")
    kvtc.kvtc_decode_attention_noalloc(plan, cache, 0, q * 0.5, sl, mx, out)
    ref = _workspace_decode(plan, cache, q * 0.5, sl, mx)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_noalloc_decode_rejects_work_beyond_its_fixed_scratch():
    rng = np.random.default_rng(12)
    plan = gh.random_plan(1, 1, 64, [((16, 2), (16, 2))], rng)
    n_seq, T = 4, 1 << 17        # 4 x 64 query heads x 128 splits of partials exceed 16 MiB
    assert kvtc.kvtc_decode_workspace_bytes(plan, n_seq, T) > 16 << 20
    bt = torch.zeros((n_seq, T // 128), dtype=torch.int32)
    cache = kvtc.Cache(plan, 1, bt)
    q = torch.zeros((n_seq, 64, 128), device="cuda")
    out = torch.zeros((n_seq, 64, 128), device="cuda")
    sl = torch.full((n_seq,), T, dtype=torch.int32, device="cuda")
    with pytest.raises(kvtc.KvtcError) as e:
        kvtc.kvtc_decode_attention_noalloc(plan, cache, 0, q, sl, T, out)
    assert e.value.status == 5                       # ECAPACITY
