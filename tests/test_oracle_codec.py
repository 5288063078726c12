"""Pins for oracle/codec.py and oracle/attention.py (CPU only)."""

import ctypes
import ctypes.util
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import attention as att
from oracle import calibration as cal
from oracle import codec


# ---------------------------------------------------------------- fp32 fma emulation
def _libm_fmaf():
    lib = ctypes.CDLL(ctypes.util.find_library("m") or "libm.so.6")
    f = lib.fmaf
    f.restype = ctypes.c_float
    f.argtypes = [ctypes.c_float] * 3
    return f


def test_fmaf_emulation_matches_c_library_fmaf():
    fmaf = _libm_fmaf()
    rng = np.random.default_rng(0)
    n = 20000
    a = (rng.standard_normal(n) * 10.0 ** rng.integers(-3, 3, n)).astype(np.float32)
    b = (rng.standard_normal(n) * 10.0 ** rng.integers(-3, 3, n)).astype(np.float32)
    c = (rng.standard_normal(n) * 10.0 ** rng.integers(-3, 3, n)).astype(np.float32)
    # halfway cases: c chosen so that a*b + c lands next to fp32 midpoints
    m = n // 4
    a[:m] = (1 + rng.integers(1, 2 ** 12, m) / 2 ** 12).astype(np.float32)
    b[:m] = (1 + rng.integers(1, 2 ** 12, m) / 2 ** 12).astype(np.float32)
    c[:m] = np.float32(2.0 ** 24)
    got = codec.fmaf32(a, b, c)
    ref = np.array([fmaf(float(x), float(y), float(z)) for x, y, z in zip(a, b, c)], np.float32)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def _chains_by_emulated_fma(x, M):
    """The canonical order written out with the fp64-emulated fma: chain e takes
    k = e, e+8, ... ascending; then the fixed pairwise sum."""
    n, r = x.shape[0], M.shape[0]
    a = [np.zeros((n, r), np.float32) for _ in range(8)]
    for k in range(x.shape[1]):
        e = k % 8
        a[e] = codec.fmaf32(np.broadcast_to(x[:, k:k + 1], (n, r)), np.broadcast_to(M[None, :, k], (n, r)), a[e])
    return ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]))


def test_canonical_projection_fast_path_equals_emulated_fma_on_bf16_operands():
    rng = np.random.default_rng(1)
    x = codec.to_bf16(rng.standard_normal((40, 128)).astype(np.float32))
    M = codec.to_bf16(rng.standard_normal((12, 128)).astype(np.float32) / 8)
    fast = codec.project_canonical(x, M)
    ref = _chains_by_emulated_fma(x, M)
    assert np.array_equal(fast.view(np.uint32), ref.view(np.uint32))


def test_canonical_projection_equals_exact_rational_evaluation_of_its_order():
    # Each fma and each add of the stated order evaluated exactly and rounded once to
    # fp32 with rational arithmetic: independent of numpy's float32 and of fmaf32.
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((3, 32)) * 10.0 ** rng.integers(-2, 3, (3, 32))).astype(np.float32)
    M = (rng.standard_normal((2, 32)) * 10.0 ** rng.integers(-2, 3, (2, 32))).astype(np.float32)
    got = codec.project_canonical(x, M)
    for i in range(3):
        for j in range(2):
            a = [Fraction(0)] * 8
            for k in range(32):
                a[k % 8] = _rn32(Fraction(float(x[i, k])) * Fraction(float(M[j, k])) + a[k % 8])
            s01, s23 = _rn32(a[0] + a[1]), _rn32(a[2] + a[3])
            s45, s67 = _rn32(a[4] + a[5]), _rn32(a[6] + a[7])
            y = _rn32(_rn32(s01 + s23) + _rn32(s45 + s67))
            assert Fraction(float(got[i, j])) == y


def test_canonical_projection_order_is_not_the_sequential_chain():
    # The order is part of the definition: on cancelling inputs the sequential fma
    # chain and the eight-chain order give different fp32 results.
    x = np.zeros((1, 16), np.float32)
    M = np.zeros((1, 16), np.float32)
    x[0, 0], x[0, 1], x[0, 8] = 1.0, 2.0 ** -30, -1.0
    M[0, 0] = M[0, 1] = M[0, 8] = 1.0
    y = codec.project_canonical(x, M)[0, 0]
    seq = np.float32(0.0)
    for k in range(16):
        seq = codec.fmaf32(x[0, k], M[0, k], seq)
    assert y == np.float32(2.0 ** -30) and seq == np.float32(0.0)


def test_canonical_projection_within_fp32_accumulation_bound():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((50, 128)).astype(np.float32)
    M = rng.standard_normal((20, 128)).astype(np.float32)
    y = codec.project_canonical(x, M).astype(np.float64)
    exact = x.astype(np.float64) @ M.astype(np.float64).T
    bound = 128 * 2.0 ** -24 * (np.abs(x).astype(np.float64) @ np.abs(M).astype(np.float64).T)
    assert np.all(np.abs(y - exact) <= bound)


def test_to_bf16_round_to_nearest_even():
    # bf16 keeps 7 fraction bits: the spacing above 1.0 is 2^-7.
    vals = np.array([1.0, 1.0 + 2 ** -7, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 0.0],
                    np.float32)
    out = codec.to_bf16(vals)
    # 1+2^-8 is a tie -> even (1.0); 1+3*2^-8 is a tie -> even (1+2^-6); 1+2^-9 -> 1.0
    assert list(out) == [1.0, 1.0 + 2 ** -7, 1.0, 1.0 + 2 ** -6, 1.0, -2.5, 0.0]


# ---------------------------------------------------------------- quantizer
def _rn32(fr):
    """Round a Fraction to the nearest fp32 (ties to even), as a Fraction."""
    if fr == 0:
        return Fraction(0)
    sgn = -1 if fr < 0 else 1
    a = abs(fr)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 23)
    q, rem = divmod(a, ulp)
    if rem * 2 > ulp or (rem * 2 == ulp and q % 2 == 1):
        q += 1
    return sgn * q * ulp


@pytest.mark.parametrize("b", range(2, 9))
def test_quantizer_matches_exact_rational_definition(b):
    rng = np.random.default_rng(b)
    y = (rng.standard_normal(3000) * 3).astype(np.float32)
    inv = np.float32(1 / 0.37)
    got = codec.quantize(y, inv, b)
    half = Fraction(2 ** (b - 1))
    for yi, ci in zip(y, got):
        t = _rn32(Fraction(float(yi)) * Fraction(float(inv)))
        u = _rn32(t + half)
        c = min(max(math.floor(u), 0), 2 ** b - 1)
        assert c == ci


def test_quantizer_special_values_and_range():
    y = np.array([np.nan, np.inf, -np.inf, 1e30, -1e30, 0.0, -0.0], np.float32)
    c = codec.quantize(y, np.float32(2.0), 3)
    assert list(c) == [0, 7, 0, 7, 0, 4, 4]


@pytest.mark.parametrize("b", [2, 5, 8])
def test_dequantize_returns_cell_midpoint(b):
    delta = 0.25
    rng = np.random.default_rng(b)
    lim = delta * 2 ** (b - 1)
    y = rng.uniform(-lim * 0.999, lim * 0.999, 5000).astype(np.float32)
    c = codec.quantize(y, np.float32(1 / delta), b)
    yh = codec.dequantize(c, delta, b)
    assert np.all(np.abs(yh - y) <= delta / 2 * (1 + 1e-6))


# ---------------------------------------------------------------- page layout
def test_layout_hand_computed_example():
    # K unit, r = 2, b = 2: one row of 16 words.  Token 0 (owner 0, pair 0):
    # coord 0 -> word 0 bits 0-1, coord 1 -> word 0 bits 16-17.  Token 9 (owner 1,
    # pair 1): word 1*2 + 0 = 2, offset 2 -> coord 0 at bits 2-3.
    codes = np.zeros((128, 2), np.int64)
    codes[0] = (1, 2)
    codes[9, 0] = 3
    page = codec.pack_page(codes, codec.KIND_K, 2)
    words = page.view("<u4")
    assert len(page) == 16 * 2 * 2
    assert words[0] == 0x00020001
    assert words[2] == 0x0000000C
    assert np.count_nonzero(words) == 2
    # V unit, r = 1 row would be odd; use r = 2: token 3 (owner 1, half 1, pair 0),
    # coord 1 -> row 1 starts at word 4*2 = 8; owner 1 -> word 8 + 2 = 10, bit 16.
    codes = np.zeros((128, 2), np.int64)
    codes[3, 1] = 2
    codes[24, 0] = 1          # owner 0, half 0, pair 2*1 + 1 = 3 -> word 0, offset 6
    page = codec.pack_page(codes, codec.KIND_V, 2)
    words = page.view("<u4")
    assert words[10] == 0x00020000
    assert words[0] == 0x00000040
    assert np.count_nonzero(words) == 2
    # b = 3 splits into a 2-bit plane then a 1-bit plane starting at byte 16*r*2.
    codes = np.zeros((128, 2), np.int64)
    codes[0, 0] = 5            # 0b101: low part 1 in plane 0, high bit 1 in plane 1
    page = codec.pack_page(codes, codec.KIND_K, 3)
    words = page.view("<u4")
    assert words[0] == 1
    assert words[16 * 2 * 2 // 4] == 1
    assert np.count_nonzero(words) == 2


@pytest.mark.parametrize("kind", [codec.KIND_K, codec.KIND_V])
@pytest.mark.parametrize("b", range(2, 9))
def test_layout_is_a_bijection_and_round_trips(kind, b):
    rng = np.random.default_rng(10 * b + kind)
    for r in (2, 4, 6, 10, 18, 32, 50, 64, 96, 126, 128):
        pos = codec.field_bit_positions(kind, r, b)
        nbits = 8 * codec.page_bytes(r, b)
        assert np.array_equal(np.sort(pos.reshape(-1)), np.arange(nbits))
        codes = rng.integers(0, 2 ** b, size=(128, r))
        page = codec.pack_page(codes, kind, b)
        assert page.nbytes == 16 * r * b
        assert np.array_equal(codec.unpack_page(page, kind, r, b), codes)


def test_sequence_pack_pads_with_zero_codes():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 4, size=(300, 6))
    pages = codec.pack_sequence(codes, codec.KIND_V, 2)
    assert len(pages) == 3
    full = codec.unpack_sequence(pages, codec.KIND_V, 6, 2, 384)
    assert np.array_equal(full[:300], codes)
    assert not full[300:].any()


# ---------------------------------------------------------------- attention
def _sdpa(q, K, V, scale):
    import torch
    qt = torch.from_numpy(q)[None, :, None, :]              # [1, G, 1, d]
    Kt = torch.from_numpy(K)[None, None].expand(1, q.shape[0], -1, -1)
    Vt = torch.from_numpy(V)[None, None].expand(1, q.shape[0], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    return o[0, :, 0].numpy()


def test_attention_full_rank_unquantized_equals_textbook_sdpa():
    rng = np.random.default_rng(4)
    d, T, G = 128, 700, 4
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    q = rng.standard_normal((G, d)) * 0.3
    Mk, _ = np.linalg.qr(rng.standard_normal((d, d)))
    Mv, _ = np.linalg.qr(rng.standard_normal((d, d)))
    # latents y = M x (quantisation bypassed), reconstructed by M^T in the oracle path
    o = att.softmax_attention(q, (K @ Mk.T) @ Mk, (V @ Mv.T) @ Mv, 1 / math.sqrt(d))
    ref = _sdpa(q, K, V, 1 / math.sqrt(d))
    assert np.abs(o - ref).max() < 1e-12


def test_attention_truncation_only_equals_projected_cache():
    rng = np.random.default_rng(5)
    d, T, r = 64, 300, 20
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    q = rng.standard_normal((3, d))
    w, lam, Vk, _ = cal.value_unit_weights(K)
    M = cal.folded_projection(Vk, r, cal.hadamard_signs(1, 0, r))
    P = Vk[:, :r] @ Vk[:, :r].T
    o = att.softmax_attention(q, (K @ M.T) @ M, V, 0.125)
    ref = _sdpa(q, K @ P, V, 0.125)
    assert np.abs(o - ref).max() < 1e-12


def test_split_merge_equals_two_pass():
    rng = np.random.default_rng(6)
    K = rng.standard_normal((1000, 32))
    V = rng.standard_normal((1000, 32))
    q = rng.standard_normal((5, 32)) * 2
    a = att.softmax_attention(q, K, V, 0.3)
    for n in (1, 3, 7, 64):
        assert np.abs(att.split_merge_attention(q, K, V, 0.3, n) - a).max() < 1e-13


def test_empty_cache_gives_zero_output():
    q = np.ones((2, 8))
    assert not att.softmax_attention(q, np.zeros((0, 8)), np.zeros((0, 8)), 1.0).any()


def test_decode_head_reconstructs_from_codes():
    rng = np.random.default_rng(7)
    r, d, b = 8, 16, 3
    M, _ = np.linalg.qr(rng.standard_normal((d, r)))
    M = M.T
    codes = rng.integers(0, 8, size=(50, r))
    unit = dict(M=M, delta=0.5, b=b)
    K = att.reconstruct(codes, M, 0.5, b)
    assert np.allclose(K, (0.5 * (codes - 3.5)) @ M)
    q = rng.standard_normal((2, d))
    o = att.decode_head(q, codes, codes, unit, unit, 0.25)
    assert np.allclose(o, att.softmax_attention(q, K, K, 0.25))


# ---------------------------------------------------------------- keys-only: raw pages
def test_raw_page_hand_example():
    # token 5, coordinate 9 = fp16 1.0 (0x3C00): pair k = 2, odd token -> high half of
    # word 9 * 64 + (2 XOR 4) = 582, i.e. bytes 2330..2331 = 00 3C.  Token 6,
    # coordinate 0 = fp16 -2.0 (0xC000): pair 3, low half of word 0 * 64 + 3 -> bytes
    # 12..13 = 00 C0.  Nothing else is set.
    vals = np.zeros((128, 128), dtype=np.int64)
    vals[5, 9] = 0x3C00
    vals[6, 0] = 0xC000
    page = codec.pack_page(vals, codec.KIND_V, codec.RAW_BITS)
    assert page.size == codec.page_bytes(128, codec.RAW_BITS) == 32768
    expect = np.zeros(32768, dtype=np.uint8)
    expect[2331] = 0x3C
    expect[13] = 0xC0
    assert np.array_equal(page, expect)


def test_raw_page_round_trip():
    vals = np.random.default_rng(21).integers(0, 1 << 16, size=(128, 128))
    page = codec.pack_page(vals, codec.KIND_V, codec.RAW_BITS)
    assert np.array_equal(codec.unpack_page(page, codec.KIND_V, 128, codec.RAW_BITS), vals)


def test_raw_swizzle_spreads_each_fragment_read_over_32_banks():
    # The eight coordinate rows and four token pairs one 16x16 value tile takes per
    # 32-bit load land in 32 distinct 4-byte banks, for every tile and block.
    for mt in range(8):
        for blk in range(8):
            for half in range(2):
                banks = {codec.raw_word_index(16 * mt + g + 8 * e, 8 * blk + tq + 4 * half) % 32
                         for g in range(8) for tq in range(4) for e in (0,)}
                assert len(banks) == 32


def test_encode_raw_rounds_to_nearest_even_fp16():
    # 1 + 2^-11 is halfway between 1 and 1 + 2^-10 -> 1 (even); 1 + 3 * 2^-11 is halfway
    # between 1 + 2^-10 and 1 + 2^-9 -> 1 + 2^-9 (even); 2^-25 is halfway between 0 and
    # the smallest subnormal 2^-24 -> 0; 65520 overflows to +inf.
    x = np.array([[1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2.0 ** -25, -2.0, 65520.0]], dtype=np.float32)
    got = codec.encode_raw(x)[0]
    assert list(got) == [0x3C00, 0x3C02, 0x0000, 0xC000, 0x7C00]


def test_dequantize_raw_reads_fp16_values():
    c = np.array([0x3C00, 0xC000, 0x0001, 0x7BFF])
    y = codec.dequantize(c, 2.0 ** -24, codec.RAW_BITS)
    assert list(y) == [1.0, -2.0, 2.0 ** -24, 65504.0]


def test_decode_head_with_raw_values_equals_sdpa_on_fp16_values():
    # keys-only: coded keys reconstructed by M^T, values the fp16-rounded inputs
    rng = np.random.default_rng(23)
    d, T, r, b = 128, 400, 16, 4
    Mk, _ = np.linalg.qr(rng.standard_normal((d, r)))
    Mk = Mk.T
    kc = rng.integers(0, 1 << b, size=(T, r))
    V = rng.standard_normal((T, d)).astype(np.float32) * 3
    vc = codec.encode_raw(V)
    q = rng.standard_normal((4, d))
    uk = dict(M=Mk, delta=0.2, b=b)
    uv = dict(M=np.eye(d), delta=2.0 ** -24, b=codec.RAW_BITS)
    o = att.decode_head(q, kc, vc, uk, uv, 1 / math.sqrt(d))
    Khat = (0.2 * (kc - (2 ** b - 1) / 2)) @ Mk
    ref = _sdpa(q, Khat, V.astype(np.float16).astype(np.float64), 1 / math.sqrt(d))
    assert np.abs(o - ref).max() < 1e-12


# ---------------------------------------------------------------- pre-RoPE keys
def test_rope_hand_example():
    # d = 4, base 100: angles t * 100^0 = t and t * 100^(-1/2) = t / 10.  x = e_0 at
    # position 2 -> (cos 2, 0, sin 2, 0); x = e_1 -> (0, cos 0.2, 0, sin 0.2).
    x = np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0]])
    got = att.apply_rope(x, [2, 2], base=100.0)
    want = np.array([[math.cos(2), 0, math.sin(2), 0], [0, math.cos(0.2), 0, math.sin(0.2)]])
    assert np.abs(got - want).max() < 1e-15


def test_rope_is_a_rotation_by_relative_position():
    rng = np.random.default_rng(31)
    d = 128
    q, k = rng.standard_normal((1, d)), rng.standard_normal((1, d))
    assert np.allclose(att.apply_rope(q, [0]), q, atol=0)                       # identity at 0
    for m, n in ((5, 9), (1000, 70000), (131071, 3)):
        qm, kn = att.apply_rope(q, [m]), att.apply_rope(k, [n])
        assert abs(np.linalg.norm(kn) - np.linalg.norm(k)) < 1e-12                # orthogonal
        # R(m)^T R(n) = R(n - m): the score depends on the distance only
        assert abs((qm @ kn.T).item() - (q @ att.apply_rope(k, [n - m]).T).item()) < 1e-9


def test_decode_head_prerope_equals_sdpa_on_keys_rotated_as_complex_numbers():
    # independent form of the rotation: pair (x_i, x_{i+d/2}) as x_i + j x_{i+d/2} times
    # exp(j t theta_i); full rank, quantisation bypassed through an identity basis
    rng = np.random.default_rng(32)
    d, T, G = 128, 500, 4
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    theta = att.ROPE_BASE ** (-np.arange(0, d, 2) / d)
    z = (K[:, :d // 2] + 1j * K[:, d // 2:]) * np.exp(1j * np.arange(T)[:, None] * theta[None, :])
    K_rot = np.concatenate([z.real, z.imag], axis=1)
    q_rot = rng.standard_normal((G, d)) * 0.3
    unit = dict(M=np.eye(d), delta=1.0, b=codec.RAW_BITS)
    kc = codec.encode_raw(K)           # fp16 patterns: reconstruct gives fp16(K)
    vc = codec.encode_raw(V)
    o = att.decode_head_prerope(q_rot, kc, vc, unit, unit, 1 / math.sqrt(d))
    K16 = K.astype(np.float32).astype(np.float16).astype(np.float64)
    z16 = (K16[:, :d // 2] + 1j * K16[:, d // 2:]) * np.exp(1j * np.arange(T)[:, None] * theta[None, :])
    ref = _sdpa(q_rot, np.concatenate([z16.real, z16.imag], axis=1),
                V.astype(np.float32).astype(np.float16).astype(np.float64), 1 / math.sqrt(d))
    assert np.abs(o - ref).max() < 1e-12
    assert np.abs(K_rot - att.apply_rope(K, np.arange(T))).max() < 1e-12
