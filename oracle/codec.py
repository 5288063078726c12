"""Oracle: per-token encode and the packed page layout.  TEST INFRASTRUCTURE ONLY.

Source: KV-COBRA project page, "How KV-COBRA Works" (Inference: each key is rotated
and truncated with H.V^T and quantized with its head's b*-bit quantizer) and
"Efficiency" (the cache is stored as packed b-bit codes), and the "0 per-token
overhead" figure (only per-unit static parameters exist).

Readings taken where the page is silent:
  * Projection arithmetic is fp32 in one fixed order (the pages fix none): for each
    output coordinate j, eight interleaved chains a_e <- fma(x_k, M_jk, a_e) over
    k = e, e+8, ..., e+d-8 ascending (e = 0..7), each starting at 0, each fma rounded
    once (round to nearest even); then y_j = ((a_0 + a_1) + (a_2 + a_3)) +
    ((a_4 + a_5) + (a_6 + a_7)), each add rounded once.  Operands: the input values
    exactly as stored; M in the input's precision (bf16-rounded M for bf16 inputs,
    fp32 M for fp32 inputs).
  * Quantizer (mid-rise, 2^b levels, no zero level): t = fl32(y * inv_delta),
    u = fl32(t + 2^(b-1)), c = min(max(floor(u), 0), 2^b - 1) with fmax/fmin
    semantics (NaN -> 0, +inf -> 2^b-1, -inf -> 0).  Dequantize:
    y_hat = delta * (c - (2^b - 1) / 2).
  * Page layout (this build's specification; the page names none): see
    ``field_bit_positions``.
  * Keys-only mode (the project page's "k-only" results compress keys and keep values
    as they are): a value unit is then stored uncompressed, r = d and b = 16, each value
    rounded to fp16 (round to nearest even); ``RAW_BITS`` marks such a unit.  Its page
    layout is this build's specification too: see ``raw_word_index``.
"""

from __future__ import annotations

import numpy as np

PAGE_TOKENS = 128
KIND_K = 0
KIND_V = 1
RAW_BITS = 16  # b of an uncompressed (fp16) value unit in keys-only mode


# ---------------------------------------------------------------- fp32 arithmetic
def fmaf32(a, b, c):
    """Correctly rounded fp32 fused multiply-add, elementwise, emulated in fp64.

    a, b, c are float32 arrays.  The product a*b is exact in fp64 (24+24 bits); the
    sum p + c is formed in fp64 together with its exact rounding error e (TwoSum),
    so p + c = s + e exactly.  RN32(s + e) equals RN32(s) unless s is exactly halfway
    between two fp32 neighbours, where the sign of e decides.
    Pinned against the C library's fmaf on random and halfway-constructed inputs.
    """
    a = np.asarray(a, dtype=np.float32)
    b = np.asarray(b, dtype=np.float32)
    c = np.asarray(c, dtype=np.float32)
    p = a.astype(np.float64) * b.astype(np.float64)
    c64 = c.astype(np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        s = p + c64
        bb = s - p
        e = (p - (s - bb)) + (c64 - bb)
        r = s.astype(np.float32)
        r64 = r.astype(np.float64)
        lo = np.where(r64 <= s, r, np.nextafter(r, np.float32(-np.inf)))
        hi = np.nextafter(lo, np.float32(np.inf))
        mid = 0.5 * (lo.astype(np.float64) + hi.astype(np.float64))
        tie = (s == mid) & (e != 0) & np.isfinite(s)
        r = np.where(tie & (e > 0), hi, np.where(tie & (e < 0), lo, r))
    return r.astype(np.float32)


def to_bf16(x):
    """Round fp32 values to bf16 (round to nearest even), returned as fp32."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16) << 16
    out = out.astype(np.uint32)
    nan = np.isnan(x)
    out = np.where(nan, np.uint32(0x7FC00000), out)
    return out.view(np.float32)


def project_canonical(x, M):
    """y[n, j] = the canonical fp32 projection of x[n, :] against M[j, :] (module
    docstring: eight interleaved fma chains over k mod 8, then a fixed pairwise sum).

    x: [n, d] float32 (values exactly as the device reads them); M: [r, d] float32
    operand matrix, d a multiple of 8.  Returns [n, r] float32.  When every product
    x_k * M_jk is exact in fp32 (both operands bf16-representable) the fma reduces to
    an fp32 add of the exact product; otherwise the fp64 emulation ``fmaf32`` is used.
    """
    x = np.asarray(x, dtype=np.float32)
    M = np.asarray(M, dtype=np.float32)
    n, d = x.shape
    r = M.shape[0]
    assert d % 8 == 0
    chains = np.zeros((n, r, 8), dtype=np.float32)
    exact_products = (np.array_equal(to_bf16(x), x, equal_nan=True)
                      and np.array_equal(to_bf16(M), M))
    for k0 in range(0, d, 8):
        xk = x[:, None, k0:k0 + 8]          # [n, 1, 8]: element e feeds chain e
        mk = M[None, :, k0:k0 + 8]          # [1, r, 8]
        if exact_products:
            with np.errstate(invalid="ignore", over="ignore"):
                chains = (chains + xk * mk).astype(np.float32)
        else:
            chains = fmaf32(np.broadcast_to(xk, chains.shape), np.broadcast_to(mk, chains.shape), chains)
    a = [chains[:, :, e] for e in range(8)]
    with np.errstate(invalid="ignore", over="ignore"):
        return (((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]))).astype(np.float32)


def quantize(y, inv_delta, b):
    """b-bit mid-rise uniform quantizer in canonical fp32 (module docstring)."""
    y = np.asarray(y, dtype=np.float32)
    inv = np.float32(inv_delta)
    half = np.float32(1 << (b - 1))
    with np.errstate(invalid="ignore", over="ignore"):
        t = (y * inv).astype(np.float32)
        u = (t + half).astype(np.float32)
        f = np.floor(u)
        f = np.fmax(f, np.float32(0.0))
        f = np.fmin(f, np.float32((1 << b) - 1))
    return f.astype(np.int64)


def dequantize(c, delta, b):
    """y_hat = delta * (c - (2^b - 1)/2), fp64.  For an uncompressed unit (b = RAW_BITS)
    c holds fp16 bit patterns and y_hat is their value."""
    if b == RAW_BITS:
        return np.asarray(c, dtype=np.int64).astype(np.uint16).view(np.float16).astype(np.float64)
    return float(delta) * (np.asarray(c, dtype=np.float64) - ((1 << b) - 1) / 2.0)


# ---------------------------------------------------------------- page layout
def code_parts(b):
    """Split of a b-bit code into bit fields of width 8, 4, 2 or 1, lowest bits
    first: the binary expansion of b from its highest power (so 3 = 2+1, 5 = 4+1,
    6 = 4+2, 7 = 4+2+1).  Returns [(lo_bit, width), ...]."""
    parts = []
    lo = 0
    for w in (8, 4, 2, 1):
        if b & w:
            parts.append((lo, w))
            lo += w
    return parts


def page_bytes(r, b):
    """Bytes of one page of one unit: 128 tokens * r codes * b bits = 16*r*b."""
    return 16 * r * b


def field_bit_positions(kind, r, b):
    """Bit index (within the page) of every code bit: array [128, r, b].

    The layout (this build's specification).  A page holds 128 tokens of one unit.
    Each code is split into parts (``code_parts``); part p (width w, code bits
    [lo, lo+w)) lives in its own plane, planes stored one after another, plane p
    starting at byte 16*r*lo.  A plane is a sequence of rows of 32-bit little-endian
    words; the page bit k is bit (k mod 32) of word floor(k/32).
      K unit: row rho (0 <= rho < r/2) holds coordinates 2*rho and 2*rho+1 of all
        128 tokens and is 8*w words long.  Token t belongs to owner o = t mod 8 and
        has pair index pi = 2*(t div 16) + (t div 8) mod 2.  Owner o owns words
        [o*w, (o+1)*w) of the row; pair pi sits in word o*w + pi div (16/w), at bit
        offset (pi mod (16/w))*w; coordinate 2*rho uses that offset in the low 16
        bits of the word, coordinate 2*rho+1 the same offset + 16.
      V unit: row j (0 <= j < r) holds coordinate j of all 128 tokens and is 4*w
        words long.  Token t belongs to owner o = (t mod 8) div 2, pair index
        pi = 2*(t div 16) + (t div 8) mod 2 and half h = t mod 2.  Owner o owns
        words [o*w, (o+1)*w); the pair sits in word o*w + pi div (16/w) at bit offset
        (pi mod (16/w))*w + 16*h.
    Every plane is dense, so a page is exactly 16*r*b bytes (no per-token overhead).
    Pinned: a hand-computed example, a round trip for every (r, b), and a bijection
    check (every page bit used exactly once).
    """
    assert r % 2 == 0 and 2 <= r and 2 <= b <= 8
    t = np.arange(PAGE_TOKENS)[:, None]
    j = np.arange(r)[None, :]
    pi = 2 * (t // 16) + (t // 8) % 2
    pos = np.zeros((PAGE_TOKENS, r, b), dtype=np.int64)
    for (lo, w) in code_parts(b):
        plane_base = 128 * r * lo            # bits
        per_word = 16 // w
        if kind == KIND_K:
            rho = j // 2
            half = j % 2
            o = t % 8
            row_words = 8 * w
            word = rho * row_words + o * w + pi // per_word
        else:
            half = t % 2
            o = (t % 8) // 2
            row_words = 4 * w
            word = j * row_words + o * w + pi // per_word
        offset = (pi % per_word) * w + 16 * half
        base = plane_base + 32 * word + offset
        for k in range(w):
            pos[:, :, lo + k] = base + k
    return pos


def raw_word_index(j, k):
    """Index of the 32-bit word that holds coordinate j of tokens 2k (low half) and
    2k + 1 (high half) in an uncompressed page: row j has 64 words, and pair k sits at
    position k XOR 4 (j mod 8) of its row.  (Rows are whole coordinates, like the value
    layout of the coded pages; the XOR spreads the eight rows an MMA fragment reads
    over distinct shared-memory banks.)"""
    return j * (PAGE_TOKENS // 2) + (k ^ ((j % 8) << 2))


def pack_page_raw(vals):
    """Pack fp16 bit patterns [128, d] (tokens x coordinates) of one page into
    128 * d * 2 bytes (little-endian words, see ``raw_word_index``)."""
    vals = np.asarray(vals, dtype=np.int64)
    d = vals.shape[1]
    words = np.zeros(d * (PAGE_TOKENS // 2), dtype=np.uint32)
    for j in range(d):
        for k in range(PAGE_TOKENS // 2):
            lo = int(vals[2 * k, j]) & 0xFFFF
            hi = int(vals[2 * k + 1, j]) & 0xFFFF
            words[raw_word_index(j, k)] = lo | (hi << 16)
    return words.astype("<u4").view(np.uint8)


def unpack_page_raw(page, d):
    """Inverse of ``pack_page_raw``: bytes -> fp16 bit patterns [128, d]."""
    words = np.asarray(page, dtype=np.uint8).view("<u4")
    vals = np.zeros((PAGE_TOKENS, d), dtype=np.int64)
    for j in range(d):
        for k in range(PAGE_TOKENS // 2):
            w = int(words[raw_word_index(j, k)])
            vals[2 * k, j] = w & 0xFFFF
            vals[2 * k + 1, j] = w >> 16
    return vals


def encode_raw(x):
    """Uncompressed unit: fp16 (round to nearest even) of every value, as bit
    patterns [n, d]."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).view(np.uint16).astype(np.int64)


def pack_page(codes, kind, b):
    """Pack codes [128, r] (ints in [0, 2^b)) of one page into 16*r*b bytes."""
    if b == RAW_BITS:
        return pack_page_raw(codes)
    codes = np.asarray(codes, dtype=np.int64)
    r = codes.shape[1]
    pos = field_bit_positions(kind, r, b)
    nbits = 8 * page_bytes(r, b)
    bits = np.zeros(nbits, dtype=np.uint8)
    vals = (codes[:, :, None] >> np.arange(b)[None, None, :]) & 1
    bits[pos.reshape(-1)] = vals.reshape(-1).astype(np.uint8)
    return np.packbits(bits.reshape(-1, 8), axis=1, bitorder="little").reshape(-1)


def unpack_page(page, kind, r, b):
    """Inverse of ``pack_page``: bytes -> codes [128, r]."""
    if b == RAW_BITS:
        return unpack_page_raw(page, r)
    page = np.asarray(page, dtype=np.uint8)
    bits = np.unpackbits(page, bitorder="little")
    pos = field_bit_positions(kind, r, b)
    vals = bits[pos].astype(np.int64)
    return (vals << np.arange(b)[None, None, :]).sum(axis=2)


def encode_tokens(x, M_operand, inv_delta, b):
    """Codes of n tokens of one unit: quantize(project_canonical(x, M)); for an
    uncompressed unit (b = RAW_BITS) the fp16 bit patterns of x."""
    if b == RAW_BITS:
        return encode_raw(x)
    return quantize(project_canonical(x, M_operand), inv_delta, b)


def pack_sequence(codes, kind, b):
    """Codes [T, r] of one sequence -> list of page byte arrays (the last page padded
    with zero codes, i.e. unused slots are 0 bits)."""
    codes = np.asarray(codes, dtype=np.int64)
    T, r = codes.shape
    n_pages = (T + PAGE_TOKENS - 1) // PAGE_TOKENS
    pages = []
    for p in range(n_pages):
        blk = np.zeros((PAGE_TOKENS, r), dtype=np.int64)
        part = codes[p * PAGE_TOKENS:(p + 1) * PAGE_TOKENS]
        blk[:len(part)] = part
        pages.append(pack_page(blk, kind, b))
    return pages


def unpack_sequence(pages, kind, r, b, T):
    """List of page byte arrays -> codes [T, r]."""
    out = [unpack_page(pg, kind, r, b) for pg in pages]
    if not out:
        return np.zeros((0, r), dtype=np.int64)
    return np.concatenate(out, axis=0)[:T]
