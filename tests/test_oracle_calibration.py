"""Pins for oracle/calibration.py: each check ties the oracle to something other than
itself (closed forms, identities, brute force, library routines, published test
vectors).  CPU only."""

import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import calibration as cal


# ---------------------------------------------------------------- q(b) and D(r,b)
@pytest.mark.parametrize("b", range(2, 9))
def test_q_of_b_is_uniform_quantizer_mse_on_unit_range_exact(b):
    # 2^b cells of width s = 2^-b over [0, 1), midpoint reconstruction:
    # MSE = 2^b * integral_0^s (x - s/2)^2 dx = 2^b * s^3 / 12, in exact rationals.
    s = Fraction(1, 2 ** b)
    mse = (2 ** b) * (s ** 3) / 12
    assert float(mse) == pytest.approx(cal.q_of_b(b), rel=1e-15)


@pytest.mark.parametrize("b", [2, 3, 4, 6, 8])
def test_q_of_b_matches_measured_quantization_error(b):
    rng = np.random.default_rng(b)
    x = rng.random(2_000_000)
    L = 2 ** b
    c = np.minimum(np.floor(x * L), L - 1)
    xh = (c + 0.5) / L
    err2 = (x - xh) ** 2
    mse = err2.mean()
    se = err2.std() / math.sqrt(len(x))
    assert abs(mse - cal.q_of_b(b)) < 4 * se


def _random_head(rng, d, n, g=2, alpha=1.0):
    U, _ = np.linalg.qr(rng.standard_normal((d, d)))
    lam = np.arange(1, d + 1) ** (-alpha)
    k = (rng.standard_normal((n, d)) * np.sqrt(lam)) @ U.T
    sq = np.exp(rng.standard_normal(d))
    q = ((rng.standard_normal((g, n, d)) * np.sqrt(sq)) @ U.T)
    return k, q


def test_eigensolver_reconstructs_and_is_orthonormal():
    rng = np.random.default_rng(0)
    k, _ = _random_head(rng, 32, 300)
    C = cal.second_moment(k)
    lam, V = cal.eig_desc(C)
    assert np.all(np.diff(lam) <= 0)
    assert np.abs(V @ np.diag(lam) @ V.T - C).max() <= 1e-12 * np.abs(C).max()
    assert np.abs(V.T @ V - np.eye(32)).max() <= 1e-12
    for i in range(32):
        j = np.argmax(np.abs(V[:, i]))
        assert V[j, i] > 0


@pytest.mark.parametrize("r", [2, 6, 10, 16])
def test_truncation_term_equals_query_weighted_error_trace_identity(r):
    # (1/(N*M)) sum_{n,m} (q_m . (k_n - P_r k_n))^2 == sum_{i not kept} w_i exactly,
    # because the eigenvectors diagonalise the keys' second moment.
    rng = np.random.default_rng(r)
    k, q = _random_head(rng, 16, 200, g=3)
    w, lam, V, order = cal.key_unit_weights(k, q)
    P = V[:, :r] @ V[:, :r].T
    e = k - k @ P.T
    qq = q.reshape(-1, 16)
    measured = np.mean((qq @ e.T) ** 2)
    assert measured == pytest.approx(w[r:].sum(), rel=1e-10, abs=1e-14)
    # and w_i really is sigma^2_Q,i * lambda_i in that order
    sq = np.mean((qq @ V) ** 2, axis=0)
    assert np.allclose(w, sq * lam, rtol=1e-12)
    assert np.all(np.diff(w) <= 0)


@pytest.mark.parametrize("r", [2, 8, 14])
def test_truncation_term_equals_eckart_young_error_for_mse_weights(r):
    rng = np.random.default_rng(100 + r)
    v, _ = _random_head(rng, 16, 300)
    w, lam, V, _ = cal.value_unit_weights(v)
    P = V[:, :r] @ V[:, :r].T
    err = np.sum((v - v @ P) ** 2) / v.shape[0]
    assert err == pytest.approx(w[r:].sum(), rel=1e-10)


def test_distortion_is_truncation_plus_quantization_terms():
    w = np.array([5.0, 3.0, 1.0, 0.5, 0.25, 0.125])
    assert cal.distortion(w, 2, 3) == pytest.approx(1.875 + (8.0 * 2 ** -6 / 12))
    assert cal.distortion(w, 6, 2) == pytest.approx(w.sum() * 2 ** -4 / 12)


# ---------------------------------------------------------------- C1
def _brute_c1(w, B):
    best = None
    for r in range(2, len(w) + 1, 2):
        for b in range(2, 9):
            if r * b > B:
                continue
            D = cal.distortion(w, r, b)
            if best is None or D < best[0] - 1e-15:
                best = (D, r, b)
    return best


def test_c1_equals_brute_force_on_d8():
    rng = np.random.default_rng(7)
    for trial in range(60):
        w = np.sort(rng.exponential(size=8) ** (1 + trial % 3))[::-1]
        for B in range(4, 65):
            got = cal.c1(w, B)
            ref = _brute_c1(w, B)
            assert got is not None
            assert got[0] * got[1] <= B
            assert cal.distortion(w, *got) == pytest.approx(ref[0], rel=1e-13, abs=1e-16)


def test_c1_infeasible_below_four_bits_and_stationary():
    w = np.sort(np.random.default_rng(1).random(16))[::-1]
    assert cal.c1(w, 3) is None
    for B in (8, 20, 40, 90):
        r, b = cal.c1(w, B)
        D0 = cal.distortion(w, r, b)
        for r2 in (r - 2, r + 2):       # the discrete marginal statement of C1
            if 2 <= r2 <= 16 and min(8, B // r2) >= 2:
                assert D0 <= cal.distortion(w, r2, min(8, B // r2)) + 1e-15


# ---------------------------------------------------------------- C2
def _brute_c2(ws, total):
    tabs = []
    for w in ws:
        tabs.append([(r * b, cal.distortion(w, r, b)) for r in range(2, len(w) + 1, 2)
                     for b in range(2, 9)])
    best = math.inf
    for combo in itertools.product(*tabs):
        bits = sum(c[0] for c in combo)
        if bits <= total:
            best = min(best, sum(c[1] for c in combo))
    return best


def _units(rng, n, d=8):
    return [np.sort(rng.exponential(size=d) ** rng.uniform(0.5, 3))[::-1] for _ in range(n)]


def test_c2_lagrangian_picks_are_exactly_optimal_for_their_own_budget():
    rng = np.random.default_rng(3)
    for _ in range(6):
        ws = _units(rng, 3)
        tabs = [cal.candidate_table(w) for w in ws]
        for mu in (0.0, 1e-4, 1e-3, 1e-2, 0.05, 0.3):
            picks = [int(np.argmin(t[2] + mu * t[0] * t[1])) for t in tabs]
            bits = sum(int(t[0][i] * t[1][i]) for t, i in zip(tabs, picks))
            D = sum(float(t[2][i]) for t, i in zip(tabs, picks))
            assert D == pytest.approx(_brute_c2(ws, bits), rel=1e-12, abs=1e-15)


def test_c2_budget_bound_and_brute_force_gap():
    rng = np.random.default_rng(4)
    for n in (2, 3):
        for _ in range(4):
            ws = _units(rng, n)
            for total in (4 * n, 10 * n, 24 * n, 40 * n):
                out, mu = cal.c2(ws, total)
                bits = sum(r * b for r, b in out)
                D = sum(cal.distortion(w, r, b) for w, (r, b) in zip(ws, out))
                opt = _brute_c2(ws, total)
                assert bits <= total
                assert D >= opt - 1e-12
                # never worse than the exactly-optimal Lagrangian point it started from
                tabs = [cal.candidate_table(w) for w in ws]
                lag = sum(float(t[2][np.argmin(t[2] + mu * (t[0] * t[1]))]) for t in tabs)
                assert D <= lag + 1e-12


def test_c2_equal_marginal_distortion_at_multiplier():
    # At mu*, every unit's Lagrangian pick is bracketed by marginal slopes: any cheaper
    # candidate saves at most mu* per bit, any costlier one gains at most mu* per bit.
    rng = np.random.default_rng(5)
    ws = _units(rng, 12, d=16)
    out, mu = cal.c2(ws, 12 * 16 * 1)
    assert mu > 0
    for w in ws:
        r, b, D = cal.candidate_table(w)
        i = int(np.argmin(D + mu * (r * b)))
        bits = r * b
        up = bits > bits[i]
        dn = bits < bits[i]
        if up.any():
            assert np.max((D[i] - D[up]) / (bits[up] - bits[i])) <= mu * (1 + 1e-9)
        if dn.any():
            assert np.min((D[dn] - D[i]) / (bits[i] - bits[dn])) >= mu * (1 - 1e-9)


def test_c2_rejects_budget_below_four_bits_per_unit():
    ws = _units(np.random.default_rng(6), 3)
    with pytest.raises(ValueError):
        cal.c2(ws, 11)


# ---------------------------------------------------------------- Hadamard, signs
def test_splitmix64_published_test_vectors():
    # splitmix64 from state 0: the first three outputs as published with the generator.
    assert cal.splitmix64_at(0, 0) == 0xE220A8397B1DCDAF
    assert cal.splitmix64_at(0, 1) == 0x6E789E6AA1B965F4
    assert cal.splitmix64_at(0, 2) == 0x06C45D188009454F


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64, 128])
def test_sylvester_hadamard_orthogonality(n):
    H = cal.sylvester(n)
    assert np.array_equal(H @ H.T, n * np.eye(n))
    assert set(np.unique(H)) <= {-1.0, 1.0}


@pytest.mark.parametrize("r", [2, 6, 10, 48, 64, 126, 128])
def test_block_hadamard_and_folded_projection_orthonormal(r):
    H = cal.block_hadamard(r)
    assert np.abs(H @ H.T - np.eye(r)).max() < 1e-14
    rng = np.random.default_rng(r)
    V, _ = np.linalg.qr(rng.standard_normal((128, 128)))
    M = cal.folded_projection(V, r, cal.hadamard_signs(11, 3, r))
    assert np.abs(M @ M.T - np.eye(r)).max() < 1e-13


@pytest.mark.parametrize("r", [4, 16, 32])
def test_hadamard_equalises_retained_variances(r):
    # For power-of-two r the rotated coordinates' calibration second moments all equal
    # the mean retained eigenvalue (coordinates in the eigenbasis are uncorrelated).
    rng = np.random.default_rng(r)
    k, _ = _random_head(rng, 64, 500, alpha=1.5)
    w, lam, V, _ = cal.value_unit_weights(k)
    M = cal.folded_projection(V, r, cal.hadamard_signs(5, 0, r))
    y = k @ M.T
    assert np.allclose(np.mean(y ** 2, axis=0), lam[:r].mean(), rtol=1e-10)


def test_signs_are_plus_minus_one_and_seeded():
    a = cal.hadamard_signs(1, 7, 128)
    assert set(np.unique(a)) == {-1.0, 1.0}
    assert np.array_equal(a, cal.hadamard_signs(1, 7, 128))
    assert not np.array_equal(a, cal.hadamard_signs(1, 8, 128))


# ---------------------------------------------------------------- Gaussian step g(b)
def test_gaussian_step_one_bit_closed_form():
    # Two levels at +-step/2: MSE = 1 - step*sqrt(2/pi) + step^2/4, minimum at
    # step = 2*sqrt(2/pi).
    assert cal.gaussian_step(1) == pytest.approx(2 * math.sqrt(2 / math.pi), abs=1e-12)


@pytest.mark.parametrize("b", range(2, 9))
def test_gaussian_step_matches_independent_scipy_solve(b):
    from scipy import integrate, optimize, stats

    L = 2 ** b

    def mse(step):
        tot = 0.0
        for k in range(L):
            lo = -np.inf if k == 0 else (k - L / 2) * step
            hi = np.inf if k == L - 1 else (k + 1 - L / 2) * step
            c = (k - (L - 1) / 2) * step
            tot += integrate.quad(lambda x: (x - c) ** 2 * stats.norm.pdf(x), lo, hi,
                                  epsabs=1e-14, epsrel=1e-12)[0]
        return tot

    g = cal.gaussian_step(b)
    ref = optimize.minimize_scalar(mse, bounds=(0.5 * g, 1.5 * g), method="bounded",
                                   options={"xatol": 1e-10}).x
    assert g == pytest.approx(ref, rel=2e-5)
    assert cal.gaussian_uniform_mse(g, b) == pytest.approx(mse(g), rel=1e-8)


@pytest.mark.parametrize("b", [2, 4])
def test_gaussian_mse_closed_form_matches_sampling(b):
    rng = np.random.default_rng(b)
    x = rng.standard_normal(2_000_000)
    step = cal.gaussian_step(b)
    L = 2 ** b
    c = np.clip(np.floor(x / step + L / 2), 0, L - 1)
    xh = (c - (L - 1) / 2) * step
    e2 = (x - xh) ** 2
    assert abs(e2.mean() - cal.gaussian_uniform_mse(step, b)) < 4 * e2.std() / math.sqrt(len(x))


# ---------------------------------------------------------------- whole calibration
def test_calibrate_small_model_meets_budget_and_is_deterministic():
    rng = np.random.default_rng(9)
    L, H, G, N, d = 2, 2, 2, 96, 16
    k = rng.standard_normal((L, H, N, d)) * np.linspace(2, 0.1, d)
    v = rng.standard_normal((L, H, N, d)) * np.linspace(1, 0.2, d)
    q = rng.standard_normal((L, H, G, N, d))
    units = cal.calibrate(k, v, q, L, H, bpd=1.0, seed=3)
    assert len(units) == 2 * L * H
    assert sum(u["r"] * u["b"] for u in units) <= 1.0 * d * len(units)
    for u in units:
        assert u["r"] % 2 == 0 and 2 <= u["b"] <= 8
        assert np.abs(u["M"] @ u["M"].T - np.eye(u["r"])).max() < 1e-12
        assert u["delta"] == pytest.approx(cal.gaussian_step(u["b"]) * math.sqrt(np.mean(u["lam"][:u["r"]])))
    again = cal.calibrate(k, v, q, L, H, bpd=1.0, seed=3)
    for a, b in zip(units, again):
        assert (a["r"], a["b"]) == (b["r"], b["b"])
        assert np.array_equal(a["M"], b["M"])


# ---------------------------------------------------------------- C2, damped form
def _random_pool(seed, n=12):
    rng = np.random.default_rng(seed)
    return [np.sort(rng.exponential(1.0, 128) * np.arange(1, 129) ** -rng.uniform(0.5, 2.0))[::-1]
            for _ in range(n)]


_QWEN_WEIGHTS = []


def _qwen_pool():
    # the 224 units (28 layers x 4 KV heads x K, V) of the Qwen2.5-7B-shaped workload
    if not _QWEN_WEIGHTS:
        from bit_quantization_head_b200 import synth
        w = synth.WORKLOADS["qwen7b-28L-128k-2bpd"]
        k, v, q = synth.calibration_set(w)
        for layer in range(w.n_layers):
            for h in range(w.n_kv_heads):
                _QWEN_WEIGHTS.append(cal.key_unit_weights(k[layer, h], q[layer, h])[0])
                _QWEN_WEIGHTS.append(cal.value_unit_weights(v[layer, h])[0])
    return _QWEN_WEIGHTS


def _marginal_interval(w, bits):
    """(left, right) slopes of the unit's hull at a corner budget: the distortion saved
    per bit by the last bits spent and by the next ones; None off the hull."""
    r, b, D = cal.candidate_table(w)
    h = cal.hull_points(r * b, D)
    xs = [p[0] for p in h]
    if bits not in xs:
        return None
    k = xs.index(bits)
    left = (h[k - 1][1] - h[k][1]) / (h[k][0] - h[k - 1][0]) if k > 0 else math.inf
    right = (h[k][1] - h[k + 1][1]) / (h[k + 1][0] - h[k][0]) if k + 1 < len(h) else 0.0
    return left, right


def test_hull_points_are_the_convex_corners_of_c1s_distortion_curve():
    # every hull corner is a candidate, D strictly falls, slopes strictly fall, and C1's
    # distortion at any budget lies on or above the hull (brute force over budgets)
    w = _random_pool(7, 1)[0][:16].copy()
    r, b, D = cal.candidate_table(w)
    h = cal.hull_points(r * b, D)
    assert h[0][0] == 4
    sl = [(h[i][1] - h[i + 1][1]) / (h[i + 1][0] - h[i][0]) for i in range(len(h) - 1)]
    assert all(h[i + 1][1] < h[i][1] for i in range(len(h) - 1))
    assert all(sl[i + 1] < sl[i] for i in range(len(sl) - 1))
    for B in range(4, 8 * 16 + 1):
        r1, b1 = cal.c1(w, B)
        Dstar = cal.distortion(w, r1, b1)
        k = max(i for i in range(len(h)) if h[i][0] <= B)
        if k + 1 < len(h):
            t = (B - h[k][0]) / (h[k + 1][0] - h[k][0])
            Dh = h[k][1] + t * (h[k + 1][1] - h[k][1])
        else:
            Dh = h[k][1]
        assert Dstar >= Dh - 1e-12
        if B == h[k][0]:
            assert Dstar == pytest.approx(h[k][1], rel=1e-12)


def test_c2_damped_keeps_identical_units_at_equal_budgets():
    w = np.sort(np.random.default_rng(3).exponential(1.0, 128))[::-1]
    picks, _ = cal.c2_damped([w] * 6, 6 * 96)
    assert len(set(picks)) == 1 and picks[0][0] * picks[0][1] <= 96


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_c2_damped_fits_the_budget_and_lies_between_optimum_and_equal_split(seed):
    ws = _random_pool(seed)
    total = 12 * 128
    picks, _ = cal.c2_damped(ws, total)
    assert sum(r * b for r, b in picks) <= total
    D = sum(cal.distortion(w, r, b) for w, (r, b) in zip(ws, picks))
    lag, _ = cal.c2(ws, total)
    D_opt = sum(cal.distortion(w, r, b) for w, (r, b) in zip(ws, lag))
    D_eq = sum(cal.distortion(w, *cal.c1(w, total // 12)) for w in ws)
    assert D_opt <= D <= D_eq


def _check_damped_equalises(ws, total):
    """"C2, across heads": after the five damped rounds the marginal distortions are
    equal (water-filling) -- the level's picks spend the budget to within 2 %, every
    final pick is a corner of its unit's hull, one common level brackets every unit's
    marginal interval to within 5 % (max right slope <= 1.05 x min left slope), and the
    total distortion is within 2 % of the Lagrangian solver's exact water-filling."""
    trace = []
    picks, mu = cal.c2_damped(ws, total, trace=trace)
    assert len(trace) == 6
    assert abs(trace[-1][1] - total) <= 0.02 * total
    assert sum(r * b for r, b in picks) <= total
    iv = [_marginal_interval(w, r * b) for w, (r, b) in zip(ws, picks)]
    assert all(x is not None for x in iv)
    assert max(x[1] for x in iv) <= 1.05 * min(x[0] for x in iv)
    lag, _ = cal.c2(ws, total)
    D = sum(cal.distortion(w, r, b) for w, (r, b) in zip(ws, picks))
    D_lag = sum(cal.distortion(w, r, b) for w, (r, b) in zip(ws, lag))
    assert D <= 1.02 * D_lag


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_c2_damped_equalises_marginal_distortion_in_five_rounds(seed):
    _check_damped_equalises(_random_pool(seed), 12 * 128)


def test_c2_damped_equalises_marginal_distortion_on_the_qwen_plan():
    ws = _qwen_pool()
    _check_damped_equalises(ws, 2 * 128 * len(ws))


def test_c2_damped_moves_budget_toward_the_larger_marginal():
    # two units, one with ten times the weight: it must end with more bits
    w = np.sort(np.random.default_rng(4).exponential(1.0, 128))[::-1]
    picks, _ = cal.c2_damped([w, 10.0 * w], 2 * 128)
    assert picks[1][0] * picks[1][1] > picks[0][0] * picks[0][1]


# ---------------------------------------------------------------- keys-only mode
def test_calibrate_keys_only_stores_values_raw_and_spends_the_budget_on_keys():
    rng = np.random.default_rng(19)
    L, H, G, N, d = 1, 2, 2, 96, 8
    k = rng.standard_normal((L, H, N, d)) * np.linspace(2, 0.1, d)
    v = rng.standard_normal((L, H, N, d)) * np.linspace(1, 0.2, d)
    q = rng.standard_normal((L, H, G, N, d))
    bpd = 2.0
    units = cal.calibrate(k, v, q, L, H, bpd=bpd, seed=3, k_only=True)
    keys = [u for u in units if u["kind"] == cal.KIND_K]
    vals = [u for u in units if u["kind"] == cal.KIND_V]
    for u in vals:
        assert (u["r"], u["b"], u["D"]) == (d, 16, 0.0)
        assert np.array_equal(u["M"], np.eye(d)) and u["delta"] == 2.0 ** -24
    total = int(round(bpd * d * len(keys)))
    bits = sum(u["r"] * u["b"] for u in keys)
    D = sum(u["D"] for u in keys)
    assert bits <= total
    # the key picks are within the brute-force optimum over the two key units' (r, b)
    # pairs at that budget and no worse than the Lagrangian point they started from
    ws = [u["w"] for u in keys]
    assert D >= _brute_c2(ws, total) - 1e-12
    tabs = [cal.candidate_table(w) for w in ws]
    mu = keys[0]["mu"]
    lag = sum(float(t[2][np.argmin(t[2] + mu * (t[0] * t[1]))]) for t in tabs)
    assert D <= lag + 1e-12
    # with fixed (r, b) the keys take it and the values stay raw
    fixed = cal.calibrate(k, v, q, L, H, bpd=bpd, seed=3, fixed_r=4, fixed_b=3, k_only=True)
    assert [(u["r"], u["b"]) for u in fixed] == [(4, 3), (d, 16), (4, 3), (d, 16)]
