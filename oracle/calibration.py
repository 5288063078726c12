"""Oracle: calibration and bit/rank allocation (fp64, numpy).  TEST INFRASTRUCTURE ONLY.

Source: KV-COBRA project page ("KV-COBRA: KV Cache Compression via Co-Optimized
Bit-Rank Allocation"), sections "How KV-COBRA Works" (distortion model, calibration,
inference), "C1, per head", "C2, across heads", "Hadamard rotation" and
"Attention-KL reordering"; joint K+V allocation from the KV-COBRA abstract.

Readings taken where the page is silent:
  * the "SVD of prefill keys" is the eigen-decomposition of the uncentered second
    moment C = X^T X / N (its eigenvectors are the right singular vectors of X);
  * for a value unit the weights are the eigenvalues (MSE weights), since the page
    gives attention-KL weights for keys only;
  * sigma^2_Q,i is the mean of (q . v_i)^2 over all calibration queries of the
    query heads that share the KV head;
  * "b ~ B/r" is floor(B/r), clipped to at most 8, and a rank r is feasible only if
    floor(B/r) >= 2, so r*b <= B always;
  * C2 is solved in Lagrangian form (each unit minimises D + mu*r*b; mu is bisected
    so the pool meets its budget) plus a greedy spend of the leftover bits; each
    unit's final (r, b) is C1 at the budget C2 gave it; the pages' damped five-round
    form iterates the same common level mu with damped Newton steps (``c2_damped``);
  * the Walsh-Hadamard of a non-power-of-two order r is block diagonal (normalised
    Sylvester blocks from the binary expansion of r, largest first);
  * one uniform quantizer per unit, step = g(b) * sqrt(mean retained eigenvalue),
    g(b) the MSE-optimal step of a 2^b-level mid-rise uniform quantizer on N(0,1).
"""

from __future__ import annotations

import math

import numpy as np

from .codec import RAW_BITS

B_MIN = 2
B_MAX = 8
KIND_K = 0
KIND_V = 1


# ---------------------------------------------------------------- distortion model
def q_of_b(b):
    """Quantisation-loss model q(b) = 2^(-2b) / 12 ("How KV-COBRA Works").

    Pinned: equals the MSE of a 2^b-level uniform quantizer over a unit range on
    uniform data (tests/test_oracle_calibration.py, sampled and exact-integral).
    """
    return 2.0 ** (-2.0 * b) / 12.0


def distortion(w, r, b):
    """Per-head distortion D(r,b) = sum_{i>r} w_i + q(b) * sum_{i<=r} w_i.

    ``w`` is already sorted in the order the basis is truncated (descending weight).
    ("How KV-COBRA Works", the displayed equation.)  Pinned: the truncation term is
    the measured truncation error (Eckart-Young / trace identity) and q(b) is pinned
    separately.
    """
    w = np.asarray(w, dtype=np.float64)
    return float(w[r:].sum() + q_of_b(b) * w[:r].sum())


# ---------------------------------------------------------------- eigenbasis
def eig_desc(C):
    """Eigenvalues (descending) and eigenvectors (columns) of a symmetric matrix.

    Sign convention: the largest-magnitude component of each eigenvector is positive
    (ties: lowest index).  Library routine: numpy.linalg.eigh.  Pinned by
    reconstruction and orthonormality.
    """
    C = np.asarray(C, dtype=np.float64)
    lam, V = np.linalg.eigh(C)
    lam = lam[::-1].copy()
    V = V[:, ::-1].copy()
    for i in range(V.shape[1]):
        k = int(np.argmax(np.abs(V[:, i])))
        if V[k, i] < 0:
            V[:, i] = -V[:, i]
    return lam, V


def second_moment(X):
    """C = X^T X / N in fp64 (the uncentered calibration second moment)."""
    X = np.asarray(X, dtype=np.float64)
    return X.T @ X / X.shape[0]


def key_unit_weights(k_cal, q_cal):
    """Attention-KL weights of a key unit ("Attention-KL reordering").

    k_cal: [N, d] calibration keys of one KV head.  q_cal: [G, N_q, d] calibration
    queries of the G query heads that read this KV head.
    Returns (w, lam, V, order): w_i = sigma^2_Q,i * sigma^2_K,i in the sorted order,
    lam the eigenvalues in that order, V the eigenvectors in that order (columns),
    order the permutation applied to the descending-eigenvalue basis.
    sigma^2_K,i is the i-th eigenvalue; sigma^2_Q,i the mean squared projection of
    the queries on eigenvector i.  Sort: descending w, stable on eigen index.
    """
    lam, V = eig_desc(second_moment(k_cal))
    q = np.asarray(q_cal, dtype=np.float64).reshape(-1, V.shape[0])
    sq = np.mean((q @ V) ** 2, axis=0)
    w_raw = sq * lam
    order = np.argsort(-w_raw, kind="stable")
    return w_raw[order], lam[order], V[:, order], order


def value_unit_weights(v_cal):
    """MSE weights of a value unit: w_i = lambda_i (the page's KV-COBRA_MSE weight,
    applied to values; reading documented in the module docstring)."""
    lam, V = eig_desc(second_moment(v_cal))
    order = np.argsort(-lam, kind="stable")
    return lam[order], lam[order], V[:, order], order


def mse_unit_weights(x_cal):
    """KV-COBRA_MSE weights for any unit ("Attention-KL reordering": w_i = lambda_i)."""
    return value_unit_weights(x_cal)


# ---------------------------------------------------------------- C1
def c1(w, B, d=None):
    """C1, per head ("C1, per head"): for head budget B bits per token, enumerate the
    even ranks r, set b = min(8, floor(B / r)), keep the feasible pair (b >= 2) with
    the smallest D; ties go to the smaller r*b, then the smaller r.  Returns (r, b)
    or None when no rank is feasible (B < 4).
    Pinned: brute-force enumeration over all (r, b) with r*b <= B on d = 8.
    """
    d = len(w) if d is None else d
    best = None
    for r in range(2, d + 1, 2):
        b = min(B_MAX, B // r)
        if b < B_MIN:
            continue
        D = distortion(w, r, b)
        key = (D, r * b, r)
        if best is None or key < best[0]:
            best = (key, (r, b))
    return None if best is None else best[1]


# ---------------------------------------------------------------- C2
def candidate_table(w, d=None):
    """All (r, b) with r even in [2, d] and b in [2, 8], with their D(r, b), ordered
    by (r*b, r) so that a first-occurrence argmin breaks ties toward fewer bits and
    then the smaller rank.  Returns arrays (r, b, D)."""
    d = len(w) if d is None else d
    rows = [(r, b) for r in range(2, d + 1, 2) for b in range(B_MIN, B_MAX + 1)]
    rows.sort(key=lambda rb: (rb[0] * rb[1], rb[0]))
    r = np.array([x[0] for x in rows])
    b = np.array([x[1] for x in rows])
    D = np.array([distortion(w, int(ri), int(bi)) for ri, bi in rows])
    return r, b, D


def c2(weights, total_bits, iters=200):
    """C2, across heads ("C2, across heads"), solved in Lagrangian form.

    weights: list of per-unit sorted weight vectors (the pool: every unit of the
    model, K and V together).  total_bits: the pool's budget in bits per token.
    For a multiplier mu >= 0 each unit picks argmin D_u(r,b) + mu*r*b (ties: fewer
    bits, then smaller r); mu is bisected (fp64, ``iters`` steps) for the smallest
    value whose picks fit the budget.  The leftover bits are then spent greedily:
    repeatedly take the single upgrade (another (r,b) of some unit with more bits
    and lower D that still fits) with the largest distortion drop per bit (ties:
    lowest unit index, then fewer bits, then smaller r).  Each unit's budget is the
    bits of its final pick, and its (r, b) is C1 at that budget.
    Returns (list of (r, b), mu).  Raises ValueError if even 4 bits per unit exceed
    the budget.
    Pinned: equal-marginal (KKT) check at the solution and brute force over all
    combinations for 2-3 units with d = 8.
    """
    tabs = [candidate_table(w) for w in weights]
    U = len(tabs)
    if 4 * U > total_bits:
        raise ValueError("budget below 4 bits per unit")
    R = np.stack([t[0] for t in tabs])
    Bq = np.stack([t[1] for t in tabs])
    D = np.stack([t[2] for t in tabs])
    bits = R * Bq

    def pick(mu):
        return np.argmin(D + mu * bits, axis=1)

    def bits_at(mu):
        return int(bits[np.arange(U), pick(mu)].sum())

    lo, hi = 0.0, 1.0
    while bits_at(hi) > total_bits:
        hi *= 2.0
        if hi > 1e300:
            raise ValueError("no multiplier meets the budget")
    if bits_at(lo) <= total_bits:
        hi = lo
    else:
        for _ in range(iters):
            mid = 0.5 * (lo + hi)
            if bits_at(mid) <= total_bits:
                hi = mid
            else:
                lo = mid
    sel = pick(hi)
    rows = np.arange(U)
    left = total_bits - int(bits[rows, sel].sum())
    while True:
        b0 = bits[rows, sel][:, None]
        D0 = D[rows, sel][:, None]
        extra = bits - b0
        ok = (extra > 0) & (extra <= left) & (D < D0)
        if not ok.any():
            break
        gain = np.where(ok, (D0 - D) / np.where(ok, extra, 1), -np.inf)
        flat = int(np.argmax(gain))          # first occurrence: lowest unit, fewest bits
        u, c = divmod(flat, bits.shape[1])
        left -= int(extra[u, c])
        sel[u] = c
    out = []
    for u, w in enumerate(weights):
        out.append(c1(w, int(bits[u, sel[u]])))
    return out, hi


def hull_points(bits, D):
    """Lower convex hull of one unit's candidate points (bits, D) given in (bits, r)
    order: the corners of C1's distortion-versus-budget curve B -> min{D(r, b) : r*b <= B}
    that a marginal exchange of budget can reach.  Returns a list of (x, y) with x
    increasing and y strictly decreasing."""
    stair = []
    for x, y in zip(bits, D):
        x, y = int(x), float(y)
        if stair and y >= stair[-1][1]:
            continue
        if stair and stair[-1][0] == x:
            stair.pop()
        stair.append((x, y))
    hull = []
    for x, y in stair:
        while len(hull) >= 2:
            (xa, ya), (xb, yb) = hull[-2], hull[-1]
            if (yb - ya) * (x - xa) >= (y - ya) * (xb - xa):  # b on or above segment a -> (x, y)
                hull.pop()
            else:
                break
        hull.append((x, y))
    return hull


def hull_marginal(hull, B):
    """Marginal distortion of a unit at budget B (bits per token) on its hull: the
    distortion saved per extra bit, i.e. the slope of the hull segment that holds B; at
    a corner the mean of the two adjacent slopes; 0 past the last corner."""
    n = len(hull)
    k = 0
    while k + 1 < n and hull[k + 1][0] <= B:
        k += 1
    if k + 1 >= n:
        return 0.0
    right = (hull[k][1] - hull[k + 1][1]) / (hull[k + 1][0] - hull[k][0])
    if B == hull[k][0] and k > 0:
        left = (hull[k - 1][1] - hull[k][1]) / (hull[k][0] - hull[k - 1][0])
        return 0.5 * (left + right)
    return right


def c2_damped(weights, total_bits, rounds=5, damping=0.7, trace=None):
    """C2, across heads, in the pages' iterative form ("C2, across heads": with C1 as
    the oracle, budget moves between heads until their marginal distortions equalize,
    the water-filling condition; a damped update converges in five rounds).

    Reading (the pages give no step rule): the water-filling condition is a common
    level mu of marginal distortion per bit.  At a level mu every unit holds the budget
    at which its marginal distortion falls to mu, i.e. the pick argmin D + mu * r*b on
    the corners of C1's distortion-versus-budget curve (ties: fewer bits, then smaller
    r), so the marginals are equal by construction and only the level has to be found.
      * Level 0: the mean, over units, of the hull marginal distortion at the equal
        split total_bits / U (``hull_marginal``).
      * Each round: S = the bits the picks at mu spend and R = the sum of their ranks;
        a damped Newton step in log mu,
            ln mu <- ln mu - damping * 2 ln 2 * (total_bits - S) / R,
        where R / (2 ln 2) is the high-rate model's -dS/d ln mu (D ~ 2^(-2B/r) for a
        unit of rank r).
      * After ``rounds`` rounds the picks at the final level are made to fit: while
        over budget, the downgrade to a cheaper candidate with the smallest distortion
        increase per bit saved; then the leftover bits go greedily to the upgrade with
        the largest drop per bit (as in ``c2``).  Each unit's (r, b) is C1 at the bits
        of its pick.
    log and exp are the C library's (math.log / math.exp); every other step is +, -,
    *, / or a comparison, so a C++ restatement reproduces the picks.
    Returns (list of (r, b), final mu).  ``trace``, if a list, receives (mu, S) per round
    and once more for the final level.  Raises ValueError if even 4 bits per unit exceed
    the budget.
    Pinned: after five rounds the picks spend the budget to within 1 % and every unit's
    marginal interval on its hull brackets the common level; the final total D is
    within 2 % of the Lagrangian solver's; identical units stay equal.
    """
    tabs = [candidate_table(w) for w in weights]
    U = len(tabs)
    if 4 * U > total_bits:
        raise ValueError("budget below 4 bits per unit")
    R = np.stack([t[0] for t in tabs])
    Bq = np.stack([t[1] for t in tabs])
    D = np.stack([t[2] for t in tabs])
    bits = R * Bq
    rows = np.arange(U)

    def pick(mu):
        return np.argmin(D + mu * bits, axis=1)

    B0 = float(total_bits) / U
    msum = 0.0
    for u in range(U):
        msum += hull_marginal(hull_points(bits[u], D[u]), B0)
    mbar = msum / U
    if mbar > 0.0:
        lmu = math.log(mbar)
        for _ in range(rounds):
            sel = pick(math.exp(lmu))
            S = 0
            rsum = 0
            for u in range(U):
                S += int(bits[u, sel[u]])
                rsum += int(R[u, sel[u]])
            if trace is not None:
                trace.append((math.exp(lmu), S))
            lmu = lmu - damping * (2.0 * math.log(2.0)) * float(total_bits - S) / float(rsum)
        mu = math.exp(lmu)
    else:
        mu = 0.0
    sel = pick(mu)
    used = int(bits[rows, sel].sum())
    if trace is not None:
        trace.append((mu, used))
    while used > total_bits:  # over budget: cheapest downgrade per bit saved
        b0 = bits[rows, sel][:, None]
        D0 = D[rows, sel][:, None]
        saved = b0 - bits
        ok = saved > 0
        cost = np.where(ok, (D - D0) / np.where(ok, saved, 1), np.inf)
        flat = int(np.argmin(cost))
        u, c = divmod(flat, bits.shape[1])
        used -= int(saved[u, c])
        sel[u] = c
    left = total_bits - used
    while True:  # leftover: best drop per bit that fits
        b0 = bits[rows, sel][:, None]
        D0 = D[rows, sel][:, None]
        extra = bits - b0
        ok = (extra > 0) & (extra <= left) & (D < D0)
        if not ok.any():
            break
        gain = np.where(ok, (D0 - D) / np.where(ok, extra, 1), -np.inf)
        flat = int(np.argmax(gain))
        u, c = divmod(flat, bits.shape[1])
        left -= int(extra[u, c])
        sel[u] = c
    return [c1(w, int(bits[u, sel[u]])) for u, w in enumerate(weights)], mu


# ---------------------------------------------------------------- Hadamard + signs
_GAMMA = 0x9E3779B97F4A7C15
_MASK64 = (1 << 64) - 1


def splitmix64_at(seed, n):
    """Output n (n >= 0) of the splitmix64 generator (Steele, Lea & Flood 2014, as
    published by Vigna) started from state ``seed``: the finaliser applied to
    seed + (n + 1) * 0x9E3779B97F4A7C15 (mod 2^64)."""
    z = (seed + (n + 1) * _GAMMA) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def unit_index(layer, head, kind, n_kv_heads):
    """Flat unit index: ((layer * H_kv) + head) * 2 + kind (kind 0 = K, 1 = V)."""
    return (layer * n_kv_heads + head) * 2 + kind


def hadamard_signs(seed, unit, r):
    """The fixed random sign flip of one unit ("Hadamard rotation"): eps_i = +1 if
    the top bit of splitmix64 output (unit * 256 + i) is 0, else -1."""
    return np.array([1.0 if (splitmix64_at(seed, unit * 256 + i) >> 63) == 0 else -1.0
                     for i in range(r)], dtype=np.float64)


def sylvester(n):
    """Sylvester Hadamard matrix of order n (a power of two): H_1 = [1],
    H_2n = [[H, H], [H, -H]].  Pinned: H H^T = n I."""
    assert n >= 1 and (n & (n - 1)) == 0
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def block_hadamard(r):
    """Orthonormal Walsh-Hadamard of order r: block diagonal of (1/sqrt(n)) H_n for
    the powers of two n in r's binary expansion, largest first."""
    H = np.zeros((r, r))
    off = 0
    for bit in reversed(range(r.bit_length())):
        n = 1 << bit
        if r & n:
            H[off:off + n, off:off + n] = sylvester(n) / math.sqrt(n)
            off += n
    return H


def folded_projection(V_sorted, r, signs):
    """M = H_r diag(eps) V_r^T (r x d): rotate-and-truncate with the random-sign
    Walsh-Hadamard folded into the basis ("Hadamard rotation"; "Inference": H.V^T).
    Pinned: M M^T = I_r; equal second moments of the rotated coordinates for
    power-of-two r."""
    return block_hadamard(r) @ np.diag(signs) @ V_sorted[:, :r].T


# ---------------------------------------------------------------- quantizer step
def _phi(x):
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi) if math.isfinite(x) else 0.0


def _Phi(x):
    if x == math.inf:
        return 1.0
    if x == -math.inf:
        return 0.0
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def _cell_mse(a, b, c):
    """Integral over [a, b) of (x - c)^2 phi(x) dx, closed form."""
    ta = a * _phi(a) if math.isfinite(a) else 0.0
    tb = b * _phi(b) if math.isfinite(b) else 0.0
    return ((1.0 + c * c) * (_Phi(b) - _Phi(a)) + ta - tb
            - 2.0 * c * (_phi(a) - _phi(b)))


def gaussian_uniform_mse(step, b):
    """MSE of the 2^b-level mid-rise uniform quantizer of step ``step`` on N(0,1):
    thresholds (k - 2^(b-1)) * step for k = 1..2^b-1, reconstruction at the cell
    midpoints, outer cells unbounded."""
    L = 1 << b
    total = 0.0
    for k in range(L):
        lo = -math.inf if k == 0 else (k - L / 2) * step
        hi = math.inf if k == L - 1 else (k + 1 - L / 2) * step
        total += _cell_mse(lo, hi, (k - (L - 1) / 2.0) * step)
    return total


def gaussian_mse_slope(step, b):
    """d MSE / d step of ``gaussian_uniform_mse``, closed form.  The thresholds move
    with the step but sit midway between neighbouring reconstruction points, so
    their boundary terms cancel; what is left is
    -2 * sum_k c_k * integral_cell_k (x - c_k*step) phi(x) dx, with c_k = k - (L-1)/2."""
    L = 1 << b
    total = 0.0
    for k in range(L):
        lo = -math.inf if k == 0 else (k - L / 2) * step
        hi = math.inf if k == L - 1 else (k + 1 - L / 2) * step
        ck = k - (L - 1) / 2.0
        total += ck * (_phi(lo) - _phi(hi) - ck * step * (_Phi(hi) - _Phi(lo)))
    return -2.0 * total


def gaussian_step(b, lo=1e-3, hi=4.0, iters=200):
    """g(b): the step minimising ``gaussian_uniform_mse``, as the root of its slope
    (bisection in fp64; the slope is negative below the optimum and positive above).
    Pinned: the two-level closed form (b = 1: 2*sqrt(2/pi)) and an independent
    scipy quad + minimize_scalar solve for b = 2..8."""
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if gaussian_mse_slope(mid, b) < 0.0:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


# ---------------------------------------------------------------- whole calibration
def calibrate(k_cal, v_cal, q_cal, n_layers, n_kv_heads, bpd, seed, *,
              weight_mode="kl", fixed_r=0, fixed_b=0, c2_iters=200, c2_mode="lagrange",
              k_only=False):
    """Calibrate every unit (layer, KV head, K|V) and allocate (r, b).

    k_cal, v_cal: [L, H_kv, N, d]; q_cal: [L, H_kv, G, N, d] (float arrays).
    bpd: joint bits per dimension over K and V (ignored with fixed_r/fixed_b).
    Returns a list of unit dicts in flat unit order (see ``unit_index``) with keys
    layer, head, kind, r, b, w, lam, V (sorted basis), M (fp64, r x d), sigma,
    delta, inv_delta (fp32 of 1/delta), D.

    k_only (the project page's "k-only" setting: keys compressed, values kept): the
    allocation runs over the key units alone with bpd * d bits per key unit and token;
    every value unit is stored uncompressed, r = d, b = RAW_BITS (fp16 values),
    M = identity, delta = 2^-24 (an fp16 value v read as the integer code v * 2^24,
    with no centring), D = 0.
    """
    d = k_cal.shape[-1]
    units = []
    for layer in range(n_layers):
        for head in range(n_kv_heads):
            for kind in (KIND_K, KIND_V):
                if kind == KIND_K:
                    if weight_mode == "kl":
                        w, lam, V, order = key_unit_weights(k_cal[layer, head], q_cal[layer, head])
                    else:
                        w, lam, V, order = mse_unit_weights(k_cal[layer, head])
                else:
                    w, lam, V, order = value_unit_weights(v_cal[layer, head])
                units.append(dict(layer=layer, head=head, kind=kind, w=w, lam=lam, V=V,
                                  order=order))
    pool = [i for i, u in enumerate(units) if not (k_only and u["kind"] == KIND_V)]
    if fixed_r and fixed_b:
        rb_pool = [(fixed_r, fixed_b)] * len(pool)
        mu = None
    else:
        total = int(round(bpd * d * len(pool)))
        weights = [units[i]["w"] for i in pool]
        if c2_mode == "damped":
            rb_pool, mu = c2_damped(weights, total)
        else:
            rb_pool, mu = c2(weights, total, iters=c2_iters)
    rb = [(d, RAW_BITS)] * len(units)
    for i, x in zip(pool, rb_pool):
        rb[i] = x
    steps = {b: gaussian_step(b) for b in range(B_MIN, B_MAX + 1)}
    for idx, (u, (r, b)) in enumerate(zip(units, rb)):
        if b == RAW_BITS:
            u.update(r=d, b=b, signs=np.ones(d), M=np.eye(d), sigma=0.0, delta=2.0 ** -24,
                     inv_delta=np.float32(2.0 ** 24), D=0.0, mu=mu)
            continue
        signs = hadamard_signs(seed, idx, r)
        M = folded_projection(u["V"], r, signs)
        sigma = math.sqrt(float(np.mean(u["lam"][:r])))
        delta = steps[b] * sigma
        u.update(r=r, b=b, signs=signs, M=M, sigma=sigma, delta=delta,
                 inv_delta=np.float32(1.0 / delta), D=distortion(u["w"], r, b), mu=mu)
    return units
