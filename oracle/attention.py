"""Oracle: one decode step of attention over the compressed cache.  TEST INFRASTRUCTURE ONLY.

Source: KV-COBRA project page, "Efficiency" (the cache is stored as packed b-bit
codes; dequantisation and the inverse rotation are applied when it is read) and
"How KV-COBRA Works" (keys are rotated and truncated with H.V^T before
quantisation, so the inverse is V.H^T).

The oracle works in the ORIGINAL d-space: it dequantises every code, reconstructs
k_hat_t = M_K^T y_hat_K,t and v_hat_t = M_V^T y_hat_V,t in fp64, then applies
textbook softmax attention (two-pass, fp64).  It deliberately does not use the
latent shortcut (q moved into the key basis, values accumulated in the value basis)
that the GPU path uses, so that shortcut is checked against an independent
formulation.

Reading: the synthetic workloads have no rotary embedding, so keys are compared with
queries exactly as stored; the softmax scale is 1/sqrt(d) with d the head dimension
(not the retained rank).
"""

from __future__ import annotations

import numpy as np

from .codec import RAW_BITS, dequantize


def reconstruct(codes, M, delta, b):
    """x_hat [T, d] = dequantize(codes) @ M in fp64 (M: [r, d] as stored in the plan).
    An uncompressed unit (b = RAW_BITS, keys-only plans) is stored in d-space: x_hat is
    its fp16 values, whatever M and delta the plan carries."""
    y = dequantize(codes, delta, b)
    if b == RAW_BITS:
        return y
    return y @ np.asarray(M, dtype=np.float64)


def softmax_attention(q, K, V, scale):
    """Textbook attention for G queries over T tokens, fp64, two-pass softmax.

    q: [G, d]; K, V: [T, d].  Returns o [G, d].  For T == 0 the output is zero (the
    defined behaviour of an empty cache).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros((q.shape[0], V.shape[1]))
    s = (q @ K.T) * scale                       # [G, T]
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ V) / l


def decode_head(q, k_codes, v_codes, unit_k, unit_v, scale):
    """One KV head: G query vectors against the dequantised, reconstructed cache.

    unit_k / unit_v: dicts with keys M (r x d), delta, b.  k_codes [T, r_K],
    v_codes [T, r_V].
    """
    K = reconstruct(k_codes, unit_k["M"], unit_k["delta"], unit_k["b"])
    V = reconstruct(v_codes, unit_v["M"], unit_v["delta"], unit_v["b"])
    return softmax_attention(q, K, V, scale)


# ---------------------------------------------------------------- pre-RoPE keys
# The project page's Results caption states that keys are compressed pre-RoPE: the codes
# hold keys before the rotary position embedding, which is applied when they are read.
# The pages name no RoPE variant.  Readings: the common rotate-half form over pairs
# (i, i + d/2) with angle t * base^(-2i/d), base 500000 (the Llama-3.1 value), no
# frequency scaling; cached token t sits at position t; the query arrives already
# rotated to its own position (as a model applies RoPE to q before attention).
ROPE_BASE = 500000.0


def rope_angles(positions, d, base=ROPE_BASE):
    """Angles [n, d/2]: position * base^(-2i/d) for i < d/2, fp64."""
    pos = np.asarray(positions, dtype=np.float64)
    inv = base ** (-np.arange(0, d, 2, dtype=np.float64) / d)
    return pos[:, None] * inv[None, :]


def apply_rope(x, positions, base=ROPE_BASE):
    """Rotary embedding of rows x [n, d] at the given positions (rotate-half form):
    (x_i, x_{i+d/2}) -> (x_i cos a_i - x_{i+d/2} sin a_i, x_{i+d/2} cos a_i + x_i sin a_i)."""
    x = np.asarray(x, dtype=np.float64)
    h = x.shape[1] // 2
    a = rope_angles(positions, x.shape[1], base)
    c, s = np.cos(a), np.sin(a)
    x1, x2 = x[:, :h], x[:, h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)


def decode_head_prerope(q_rot, k_codes, v_codes, unit_k, unit_v, scale, base=ROPE_BASE):
    """One KV head with keys coded before RoPE: each reconstructed key k_hat_t is
    rotated to its position t, then scored against the already-rotated queries
    q_rot [G, d]; values as in ``decode_head``."""
    K = reconstruct(k_codes, unit_k["M"], unit_k["delta"], unit_k["b"])
    K = apply_rope(K, np.arange(K.shape[0]), base)
    V = reconstruct(v_codes, unit_v["M"], unit_v["delta"], unit_v["b"])
    return softmax_attention(q_rot, K, V, scale)


def split_merge_attention(q, K, V, scale, n_split):
    """The same attention computed over ``n_split`` contiguous token ranges with an
    online (max, sum, weighted-sum) state per range, merged by log-sum-exp.  Used
    only to pin that a split-context merge equals the two-pass result."""
    q = np.asarray(q, dtype=np.float64)
    T = K.shape[0]
    bounds = np.linspace(0, T, n_split + 1).astype(int)
    parts = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        if b <= a:
            continue
        s = (q @ K[a:b].T) * scale
        m = s.max(axis=1)
        p = np.exp(s - m[:, None])
        parts.append((m, p.sum(axis=1), p @ V[a:b]))
    M = np.max(np.stack([p[0] for p in parts]), axis=0)
    l = sum(np.exp(p[0] - M) * p[1] for p in parts)
    z = sum(np.exp(p[0] - M)[:, None] * p[2] for p in parts)
    return z / l[:, None]
