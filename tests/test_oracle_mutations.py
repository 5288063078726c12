"""The oracle's pins must catch plausible mistakes.  Each test plants one mistake in an
oracle function (a dropped term, a wrong constant, a swapped index, a transposed
operand, a wrong rounding), runs the pin that guards that function, and expects it to
fail.  The mistakes live only inside these tests (monkeypatch, CPU)."""

import math

import numpy as np
import pytest

from oracle import attention as att
from oracle import calibration as cal
from oracle import codec
from tests import test_oracle_calibration as pins_cal
from tests import test_oracle_codec as pins_codec


def _fails(pin, *args):
    with pytest.raises(AssertionError):
        pin(*args)


def test_dropped_quantization_term_is_caught(monkeypatch):
    monkeypatch.setattr(cal, "q_of_b", lambda b: 0.0)
    _fails(pins_cal.test_distortion_is_truncation_plus_quantization_terms)


def test_wrong_quantization_constant_is_caught(monkeypatch):
    monkeypatch.setattr(cal, "q_of_b", lambda b: 2.0 ** (-2.0 * b) / 6.0)
    _fails(pins_cal.test_q_of_b_is_uniform_quantizer_mse_on_unit_range_exact, 3)


def test_c1_rounding_the_bit_width_up_is_caught(monkeypatch):
    def c1_ceil(w, B, d=None):
        d = len(w) if d is None else d
        best = None
        for r in range(2, d + 1, 2):
            b = min(cal.B_MAX, -(-B // r))   # ceil instead of floor
            if b < cal.B_MIN:
                continue
            key = (cal.distortion(w, r, b), r * b, r)
            if best is None or key < best[0]:
                best = (key, (r, b))
        return None if best is None else best[1]
    monkeypatch.setattr(cal, "c1", c1_ceil)
    _fails(pins_cal.test_c1_equals_brute_force_on_d8)


def test_hadamard_sign_error_is_caught(monkeypatch):
    good = cal.sylvester

    def bad(n):
        H = good(n).copy()
        if n >= 2:
            H[-1, -1] = -H[-1, -1]
        return H
    monkeypatch.setattr(cal, "sylvester", bad)
    _fails(pins_cal.test_sylvester_hadamard_orthogonality, 4)


def test_quantizer_rounding_instead_of_floor_is_caught(monkeypatch):
    def quantize_round(y, inv_delta, b):
        y = np.asarray(y, dtype=np.float32)
        t = (y * np.float32(inv_delta)).astype(np.float32)
        u = (t + np.float32(1 << (b - 1))).astype(np.float32)
        f = np.fmin(np.fmax(np.rint(u), 0), (1 << b) - 1)
        return f.astype(np.int64)
    monkeypatch.setattr(codec, "quantize", quantize_round)
    _fails(pins_codec.test_quantizer_matches_exact_rational_definition, 4)


def test_dequantize_without_centring_is_caught(monkeypatch):
    monkeypatch.setattr(codec, "dequantize", lambda c, delta, b: delta * np.asarray(c, np.float64))
    _fails(pins_codec.test_dequantize_returns_cell_midpoint, 5)


def test_transposed_operand_in_projection_is_caught(monkeypatch):
    good = codec.project_canonical

    def bad(x, M):
        M = np.array(M, copy=True)
        M[:, [0, 1]] = M[:, [1, 0]]          # two columns of M exchanged
        return good(x, M)
    monkeypatch.setattr(codec, "project_canonical", bad)
    _fails(pins_codec.test_canonical_projection_equals_exact_rational_evaluation_of_its_order)


def test_swapped_tokens_in_layout_are_caught_by_the_hand_example(monkeypatch):
    # a bijection still round-trips, so only the hand-computed example can catch it
    good = codec.field_bit_positions

    def bad(kind, r, b):
        pos = good(kind, r, b)
        return pos[np.arange(codec.PAGE_TOKENS) ^ 1]
    monkeypatch.setattr(codec, "field_bit_positions", bad)
    _fails(pins_codec.test_layout_hand_computed_example)


def test_raw_layout_without_swizzle_is_caught(monkeypatch):
    monkeypatch.setattr(codec, "raw_word_index", lambda j, k: j * (codec.PAGE_TOKENS // 2) + k)
    _fails(pins_codec.test_raw_page_hand_example)
    _fails(pins_codec.test_raw_swizzle_spreads_each_fragment_read_over_32_banks)


def test_attention_scale_error_is_caught(monkeypatch):
    good = att.softmax_attention
    monkeypatch.setattr(att, "softmax_attention", lambda q, K, V, scale: good(q, K, V, scale * math.sqrt(2)))
    _fails(pins_codec.test_attention_full_rank_unquantized_equals_textbook_sdpa)


def test_rope_without_the_cross_term_is_caught(monkeypatch):
    def bad(x, positions, base=att.ROPE_BASE):
        x = np.asarray(x, dtype=np.float64)
        h = x.shape[1] // 2
        a = att.rope_angles(positions, x.shape[1], base)
        return np.concatenate([x[:, :h] * np.cos(a), x[:, h:] * np.cos(a)], axis=1)
    monkeypatch.setattr(att, "apply_rope", bad)
    _fails(pins_codec.test_rope_hand_example)
    _fails(pins_codec.test_decode_head_prerope_equals_sdpa_on_keys_rotated_as_complex_numbers)


def test_undamped_budget_exchange_is_caught(monkeypatch):
    # the earlier step rule: budgets moved in proportion to their marginal's excess over
    # the mean (no common level); it never reaches equal marginals in five rounds
    def linear_exchange(weights, total_bits, rounds=5, damping=0.5, trace=None):
        U = len(weights)
        B = [float(total_bits) / U] * U

        def dstar(u, x):
            rb = cal.c1(weights[u], int(max(4.0, min(x, 1024.0))))
            return cal.distortion(weights[u], *rb) if rb else float(np.sum(weights[u]))
        for _ in range(rounds):
            m = [(dstar(u, B[u] - 8) - dstar(u, B[u] + 8)) / 16.0 for u in range(U)]
            mb = sum(m) / U
            B = [b * (1 + damping * (x - mb) / mb) for b, x in zip(B, m)]
            s = total_bits / sum(B)
            B = [b * s for b in B]
            if trace is not None:
                trace.append((mb, int(sum(B))))
        if trace is not None:
            trace.append((mb, int(sum(B))))
        return [cal.c1(w, int(max(4.0, min(b, 1024.0)))) for w, b in zip(weights, B)], 0.0
    monkeypatch.setattr(cal, "c2_damped", linear_exchange)
    _fails(pins_cal.test_c2_damped_equalises_marginal_distortion_in_five_rounds, 1)


def test_damped_level_step_with_the_wrong_sign_is_caught(monkeypatch):
    # the level moves away from the budget (ln mu + step instead of ln mu - step)
    good = cal.c2_damped

    def flipped(weights, total_bits, rounds=5, damping=0.7, trace=None):
        return good(weights, total_bits, rounds=rounds, damping=-damping, trace=trace)
    monkeypatch.setattr(cal, "c2_damped", flipped)
    _fails(pins_cal.test_c2_damped_equalises_marginal_distortion_in_five_rounds, 0)
