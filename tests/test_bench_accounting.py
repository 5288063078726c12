"""bench.py's accounting, on the host: the algorithmic bytes the GB/s figures divide by
(packed codes of every cached token plus the fp32 bases, per KV head) and the count of
the library's kernel launches per step, for a coded and a keys-only plan."""

import numpy as np

import bench
from bit_quantization_head_b200 import kvtc
from bit_quantization_head_b200 import synth


def _plan(k_only):
    w = synth.scaled(synth.WORKLOADS["llama8b-32L-128k-1bpd"], n_layers=2, n_cal=256)
    k, v, q = synth.calibration_set(w)
    return w, kvtc.kvtc_calibrate(k, v, q, n_layers=2, n_kv_heads=8, group=4, bpd=1.0, seed=w.seed,
                                  k_only=k_only)


def test_algorithmic_bytes_count_codes_and_bases():
    for k_only in (False, True):
        w, plan = _plan(k_only)
        T, n_seq = 131072, 3
        got = bench.algorithmic_bytes(plan, range(2), T, n_seq)
        for layer in range(2):
            want = 0
            for h in range(8):
                for kind in (0, 1):
                    info = plan.unit((layer * 8 + h) * 2 + kind)
                    want += n_seq * T * info["r"] * info["b"] // 8 + info["r"] * 128 * 4
                    if k_only and kind == 1:
                        assert (info["r"], info["b"]) == (128, kvtc.RAW_BITS)   # 256 B per token
            assert got[layer] == want
        if not k_only:
            # the joint 1-bpd budget covers both layers' 32 units: at most one bit per
            # dimension of codes over the plan (a single layer may hold more)
            bases = sum(plan.unit(u)["r"] * 128 * 4 for u in range(32))
            assert sum(got) - bases <= n_seq * T * 32 * 128 // 8


def test_kernels_per_step_counts_append_and_one_split_launch_per_width_pair():
    # per layer: the append, then one decode launch per distinct (b_K, b_V) of its heads
    w, plan = _plan(False)
    w2 = synth.scaled(w, n_layers=2)
    n = bench.kernels_per_step(plan, w2)
    pairs = []
    for layer in range(2):
        pairs.append({(plan.unit((layer * 8 + h) * 2)["b"], plan.unit((layer * 8 + h) * 2 + 1)["b"])
                      for h in range(8)})
    assert n == sum(1 + len(p) for p in pairs)
    assert all(len(p) >= 1 for p in pairs)
