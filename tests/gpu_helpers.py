"""Shared helpers of the GPU parity tests: build caches, run the CUDA path through the
C ABI, and evaluate the oracle on the same inputs (and on the pages the GPU wrote)."""

import math

import numpy as np
import torch

from bit_quantization_head_b200 import kvtc
from oracle import attention as oatt
from oracle import codec as ocodec

P = 128


def plan_units(plan):
    n = plan.shape["n_units"]
    out = []
    for u in range(n):
        info = plan.unit(u)
        info["M"] = plan.matrix(u)
        out.append(info)
    return out


def make_cache(plan, seq_lens, rng, extra_pages=3):
    """A cache with a shuffled block table: sequence s owns ceil(len/128) (+1 spare) pages."""
    n_seq = len(seq_lens)
    max_pages = max(1, max((l + P - 1) // P for l in seq_lens) + 1)
    total = n_seq * max_pages + extra_pages
    perm = rng.permutation(total)[: n_seq * max_pages].reshape(n_seq, max_pages)
    bt = torch.from_numpy(perm.astype(np.int32))
    return kvtc.Cache(plan, total, bt)


def to_dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32))
    return t.to(dtype=torch.bfloat16 if dtype == "bf16" else torch.float32).cuda().contiguous()


def encode_all(plan, cache, layer, kv_per_seq, dtype, path="append", chunk=None):
    """kv_per_seq: list of (K [T, H, d], V [T, H, d]) numpy arrays; appends every sequence
    from position 0 in one call (or chunk-sized calls)."""
    n_seq = len(kv_per_seq)
    Ks = [kv[0] for kv in kv_per_seq]
    Vs = [kv[1] for kv in kv_per_seq]
    lens = [k.shape[0] for k in Ks]
    if path == "prefill":
        for s in range(n_seq):
            if lens[s] == 0:
                continue
            kvtc.kvtc_encode_prefill(plan, cache, layer, to_dev(Ks[s], dtype), to_dev(Vs[s], dtype), s, 0)
        return
    step = chunk or max(lens + [1])
    for start in range(0, max(lens + [1]), step):
        pieces_k, pieces_v, cu, pos = [], [], [0], []
        for s in range(n_seq):
            a, b = min(start, lens[s]), min(start + step, lens[s])
            pieces_k.append(Ks[s][a:b])
            pieces_v.append(Vs[s][a:b])
            cu.append(cu[-1] + (b - a))
            pos.append(a)
        if cu[-1] == 0:
            continue
        k = to_dev(np.concatenate(pieces_k), dtype)
        v = to_dev(np.concatenate(pieces_v), dtype)
        kvtc.kvtc_encode_append(plan, cache, layer, k, v, torch.tensor(cu, dtype=torch.int32).cuda(),
                                torch.tensor(pos, dtype=torch.int32).cuda())


def gpu_pages(cache, plan, unit, seq, n_pages):
    pool = cache.unit_pool(unit).cpu().numpy()
    pb = plan.unit(unit)["page_bytes"]
    bt = cache.block_table.cpu().numpy()
    return [pool[int(bt[seq, p]) * pb:(int(bt[seq, p]) + 1) * pb] for p in range(n_pages)]


def oracle_codes(x, unit, dtype):
    """Canonical codes of tokens x [T, d] for a unit dict (M fp32 from the plan)."""
    M = unit["M"]
    Mop = ocodec.to_bf16(M) if dtype == "bf16" else M.astype(np.float32)
    return ocodec.encode_tokens(np.asarray(x, np.float32), Mop, np.float32(unit["inv_delta"]), unit["b"])


def check_encode(plan, cache, layer, kv_per_seq, dtype, H):
    units = plan_units(plan)
    mism = 0
    for s, (K, V) in enumerate(kv_per_seq):
        T = K.shape[0]
        n_pages = (T + P - 1) // P
        for h in range(H):
            for kind, X in ((0, K), (1, V)):
                u = (layer * H + h) * 2 + kind
                codes = oracle_codes(X[:, h], units[u], dtype)
                want = ocodec.pack_sequence(codes, kind, units[u]["b"])
                got = gpu_pages(cache, plan, u, s, n_pages)
                for pw, pg in zip(want, got):
                    if not np.array_equal(pw, pg):
                        mism += 1
    return mism


def oracle_decode(plan, cache, layer, q, seq_lens, H, G, scale=None):
    """Oracle attention [n_seq, Hq, d] over the pages the GPU wrote."""
    units = plan_units(plan)
    d = 128
    scale = scale or 1.0 / math.sqrt(d)
    out = np.zeros((len(seq_lens), H * G, d))
    for s, T in enumerate(seq_lens):
        n_pages = (T + P - 1) // P
        for h in range(H):
            uK, uV = (layer * H + h) * 2, (layer * H + h) * 2 + 1
            ck = ocodec.unpack_sequence(gpu_pages(cache, plan, uK, s, n_pages), 0, units[uK]["r"],
                                        units[uK]["b"], T)
            cv = ocodec.unpack_sequence(gpu_pages(cache, plan, uV, s, n_pages), 1, units[uV]["r"],
                                        units[uV]["b"], T)
            out[s, h * G:(h + 1) * G] = oatt.decode_head(q[s, h * G:(h + 1) * G], ck, cv, units[uK],
                                                         units[uV], scale)
    return out


def run_decode(plan, cache, layer, q, seq_lens, out_dtype="f32", q_dtype="f32", scale=0.0):
    n_seq = len(seq_lens)
    Hq = q.shape[1]
    qd = to_dev(q, q_dtype)
    sl = torch.tensor(seq_lens, dtype=torch.int32).cuda()
    mx = max(seq_lens + [0])
    ws = torch.zeros(max(1, kvtc.kvtc_decode_workspace_bytes(plan, n_seq, mx)), dtype=torch.uint8, device="cuda")
    out = torch.empty((n_seq, Hq, 128), dtype=torch.float32 if out_dtype == "f32" else torch.bfloat16).cuda()
    kvtc.kvtc_decode_attention(plan, cache, layer, qd, sl, mx, out, ws, scale)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


def decode_errors(got, ref):
    """(max abs error, max normwise-relative error over (seq, head) output vectors)."""
    err = np.abs(got - ref)
    den = np.maximum(np.abs(ref).max(axis=-1), 1e-30)
    rel = err.max(axis=-1) / den
    live = np.abs(ref).max(axis=-1) > 0
    return float(err.max()), float(rel[live].max()) if live.any() else 0.0


def random_plan(n_layers, H, G, rb_pairs, rng):
    """A plan with given (r, b) per unit and random orthonormal projections."""
    r, b, delta, M = [], [], [], []
    for (rk, bk), (rv, bv) in rb_pairs:
        for rr, bb in ((rk, bk), (rv, bv)):
            Q, _ = np.linalg.qr(rng.standard_normal((128, 128)))
            r.append(rr)
            b.append(bb)
            if bb == kvtc.RAW_BITS:  # uncompressed value unit: identity, c = v * 2^24
                delta.append(2.0 ** -24)
                M.append(np.eye(128, dtype=np.float32))
                continue
            delta.append(float(rng.uniform(0.05, 0.3)) * 2.0 ** (2 - bb))
            M.append(Q[:rr].astype(np.float32))
    return kvtc.kvtc_plan_create(n_layers, H, G, r, b, delta, M).upload()
