"""kvtc_decode_step (the fused append of one token per sequence plus the decode) against
kvtc_encode_append followed by kvtc_decode_attention on the same inputs: the cache pools
must be identical byte for byte (the same canonical codes, written into the same slots)
and the attention outputs identical bit for bit (the decode then reads identical pages),
for packed and unpacked score modes, two head groups, keys-only plans, fp32 and bf16
inputs, a new token at the start, middle and end of a page, an empty sequence, and a
context long enough for the shared merge.  The attention is also checked against the
oracle over the pages the fused call wrote."""

import numpy as np
import pytest
import torch

from bit_quantization_head_b200 import kvtc
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _step_both(plan, H, G, lens, dtype, rng, raw_values=False):
    """Two caches with the same prefix (every sequence's first len - 1 tokens), then the
    new token through append + decode on one and through the fused step on the other."""
    n_seq = len(lens)
    caches = [gh.make_cache(plan, lens, np.random.default_rng(7)) for _ in range(2)]
    prefix = [(rng.standard_normal((max(T - 1, 0), H, 128)).astype(np.float32),
               rng.standard_normal((max(T - 1, 0), H, 128)).astype(np.float32)) for T in lens]
    for c in caches:
        gh.encode_all(plan, c, 0, prefix, dtype)
    knew = rng.standard_normal((n_seq, H, 128)).astype(np.float32)
    vnew = rng.standard_normal((n_seq, H, 128)).astype(np.float32)
    q = (rng.standard_normal((n_seq, H * G, 128)) * 0.7).astype(np.float32)
    mx = max(lens)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    qd = gh.to_dev(q, dtype)
    wsb = kvtc.kvtc_decode_workspace_bytes(plan, n_seq, mx)
    outs = []
    # (a) append of the non-empty sequences' new rows, then the decode
    live = [s for s in range(n_seq) if lens[s] > 0]
    # cu_seqlens over every sequence: sequence s gets one token if lens[s] > 0
    cu_all = [0]
    for s in range(n_seq):
        cu_all.append(cu_all[-1] + (1 if lens[s] > 0 else 0))
    cu = torch.tensor(cu_all, dtype=torch.int32, device="cuda")
    pos = torch.tensor([max(T - 1, 0) for T in lens], dtype=torch.int32, device="cuda")
    kv_k = gh.to_dev(knew[live], dtype) if live else None
    kv_v = gh.to_dev(vnew[live], dtype) if live else None
    if live:
        kvtc.kvtc_encode_append(plan, caches[0], 0, kv_k, kv_v, cu, pos)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    out_a = torch.full((n_seq, H * G, 128), float("nan"), dtype=torch.float32, device="cuda")
    kvtc.kvtc_decode_attention(plan, caches[0], 0, qd, sl, mx, out_a, ws)
    # (b) the fused step
    ws2 = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    out_b = torch.full((n_seq, H * G, 128), float("nan"), dtype=torch.float32, device="cuda")
    kvtc.kvtc_decode_step(plan, caches[1], 0, gh.to_dev(knew, dtype), gh.to_dev(vnew, dtype), qd, sl, mx, out_b, ws2)
    torch.cuda.synchronize()
    for c in caches:
        assert int(c.status.item()) == 0
    assert torch.equal(caches[0].pool, caches[1].pool)
    assert torch.equal(out_a, out_b)
    # and the fused call's output against the oracle over the pages it wrote
    q64 = (gh.to_dev(q, dtype).float().cpu().numpy()).astype(np.float64)
    ref = gh.oracle_decode(plan, caches[1], 0, q64, lens, H, G)
    ab, rel = gh.decode_errors(out_b.cpu().numpy(), ref)
    assert ab <= TOL and rel <= TOL, (ab, rel)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("G", [4, 12])
def test_decode_step_equals_append_then_decode(dtype, G):
    rng = np.random.default_rng(60 + G + (dtype == "bf16"))
    H = 3
    plan = gh.random_plan(1, H, G, [((16, 2), (16, 2)), ((34, 3), (18, 5)), ((128, 8), (96, 4))], rng)
    # new token at slot 0 of a page, mid page, last slot, a one-token sequence, an empty one
    lens = [129, 700, 256, 1, 0, 3000]
    _step_both(plan, H, G, lens, dtype, rng)


def test_decode_step_keys_only_and_shared_merge():
    rng = np.random.default_rng(70)
    H, G = 2, 4
    plan = gh.random_plan(1, H, G, [((32, 2), (128, kvtc.RAW_BITS)), ((64, 3), (128, kvtc.RAW_BITS))], rng)
    _step_both(plan, H, G, [20001, 640], "bf16", rng)
