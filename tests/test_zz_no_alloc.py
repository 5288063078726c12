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
TOL = 2e-3


def test_noalloc_decode_matches_workspace_decode_on_two_calls_in_a_row():
    rng = np.random.default_rng(11)
    H, G = 3, 4
    plan = gh.random_plan(1, H, G, [((64, 2), (64, 2)), ((18, 3), (96, 4)), ((128, 2), (32, 8))], rng)
    lens = [3000, 517]
    cache = gh.make_cache(plan, lens, rng)
    kv = [(rng.standard_normal((T, H, 128)).astype(np.float32),
           rng.standard_normal((T, H, 128)).astype(np.float32)) for T in lens]
    gh.encode_all(plan, cache, 0, kv, "f32")
    q = torch.from_numpy((rng.standard_normal((2, H * G, 128)) * 0.5).astype(np.float32)).cuda()
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    mx = max(lens)
    ws = torch.empty(kvtc.kvtc_decode_workspace_bytes(plan, 2, mx), dtype=torch.uint8, device="cuda")
    ref = torch.empty((2, H * G, 128), dtype=torch.float32, device="cuda")
    kvtc.kvtc_decode_attention(plan, cache, 0, q, sl, mx, ref, ws)
    torch.cuda.synchronize()
    ref = ref.cpu().numpy()
    for _ in range(2):
        out = torch.full((2, H * G, 128), float("nan"), dtype=torch.float32, device="cuda")
        kvtc.kvtc_decode_attention_noalloc(plan, cache, 0, q, sl, mx, out)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        err = np.abs(got - ref).max(axis=-1) / np.maximum(np.abs(ref).max(axis=-1), 1e-30)
        assert np.all(np.isfinite(got))
        assert err.max() <= TOL
    assert int(cache.status.item()) == 0


def test_noalloc_decode_rejects_work_beyond_its_fixed_scratch():
    rng = np.random.default_rng(12)
    plan = gh.random_plan(1, 1, 64, [((16, 2), (16, 2))], rng)
    big = 1 << 21                                    # 2M tokens: partials exceed 16 MiB
    bt = torch.zeros((1, big // 128), dtype=torch.int32)
    cache = kvtc.Cache(plan, 1, bt)
    q = torch.zeros((1, 64, 128), device="cuda")
    out = torch.zeros((1, 64, 128), device="cuda")
    sl = torch.tensor([big], dtype=torch.int32, device="cuda")
    with pytest.raises(kvtc.KvtcError) as e:
        kvtc.kvtc_decode_attention_noalloc(plan, cache, 0, q, sl, big, out)
    assert e.value.status == 5                       # ECAPACITY
