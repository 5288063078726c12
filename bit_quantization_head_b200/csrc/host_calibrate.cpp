// kvtc_calibrate: per-unit eigenbasis, attention-KL weights, C1 + C2 allocation, folded
// random-sign Walsh-Hadamard projection and Gaussian quantizer step.
//
// Source: KV-COBRA project page, "How KV-COBRA Works" (distortion D(r,b), calibration),
// "C1, per head", "C2, across heads", "Hadamard rotation", "Attention-KL reordering";
// joint K+V pool per the KV-COBRA abstract.  The eigen-solver here is Householder
// tridiagonalisation plus implicit QR with a Wilkinson shift, with cyclic Jacobi as a
// fallback (both written here, independent of the LAPACK routine the oracle uses), run on
// host threads over units.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstring>
#include <memory>
#include <thread>
#include <utility>
#include <vector>

#include "kvtc_internal.h"

namespace kvtc {
namespace {

// ------------------------------------------------------------------ eigen-solver
// Cyclic Jacobi on a symmetric n x n matrix A (row-major, destroyed).  On return lam
// holds the eigenvalues in descending order and V (row-major, column i = eigenvector
// i) the eigenvectors, each with its largest-magnitude component positive (ties: the
// lowest index).
void jacobi_eig(std::vector<double>& A, int n, std::vector<double>& lam, std::vector<double>& V) {
  V.assign(static_cast<size_t>(n) * n, 0.0);
  for (int i = 0; i < n; ++i) V[i * n + i] = 1.0;
  double fro = 0.0;
  for (double x : A) fro += x * x;
  fro = std::sqrt(fro);
  for (int sweep = 0; sweep < 60; ++sweep) {
    double off = 0.0;
    for (int p = 0; p < n; ++p)
      for (int q = p + 1; q < n; ++q) off += A[p * n + q] * A[p * n + q];
    if (std::sqrt(2.0 * off) <= 1e-17 * fro || off == 0.0) break;
    for (int p = 0; p < n - 1; ++p) {
      for (int q = p + 1; q < n; ++q) {
        double apq = A[p * n + q];
        if (apq == 0.0) continue;
        double app = A[p * n + p], aqq = A[q * n + q];
        double theta = (aqq - app) / (2.0 * apq);
        double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        // A <- J^T A J with J the rotation in the (p, q) plane.
        for (int k = 0; k < n; ++k) {
          double akp = A[k * n + p], akq = A[k * n + q];
          A[k * n + p] = c * akp - s * akq;
          A[k * n + q] = s * akp + c * akq;
        }
        for (int k = 0; k < n; ++k) {
          double apk = A[p * n + k], aqk = A[q * n + k];
          A[p * n + k] = c * apk - s * aqk;
          A[q * n + k] = s * apk + c * aqk;
        }
        A[p * n + q] = A[q * n + p] = 0.0;
        for (int k = 0; k < n; ++k) {
          double vkp = V[k * n + p], vkq = V[k * n + q];
          V[k * n + p] = c * vkp - s * vkq;
          V[k * n + q] = s * vkp + c * vkq;
        }
      }
    }
  }
  std::vector<int> idx(n);
  for (int i = 0; i < n; ++i) idx[i] = i;
  std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return A[a * n + a] > A[b * n + b]; });
  lam.resize(n);
  std::vector<double> W(static_cast<size_t>(n) * n);
  for (int j = 0; j < n; ++j) {
    int src = idx[j];
    lam[j] = A[src * n + src];
    int kmax = 0;
    for (int k = 1; k < n; ++k)
      if (std::fabs(V[k * n + src]) > std::fabs(V[kmax * n + src])) kmax = k;
    double sgn = V[kmax * n + src] < 0 ? -1.0 : 1.0;
    for (int k = 0; k < n; ++k) W[k * n + j] = sgn * V[k * n + src];
  }
  V.swap(W);
}

// Householder tridiagonalisation followed by implicit symmetric QR steps with a Wilkinson
// shift (the textbook method for dense symmetric matrices).  A (row-major, symmetric,
// destroyed) -> eigenvalues (diagonal of the converged T) and eigenvectors (columns of
// the accumulated orthogonal Q), in the same order and sign convention as jacobi_eig.
// Returns false if the QR iteration does not converge within its step limit.
bool tridiag_qr_eig(std::vector<double>& A, int n, std::vector<double>& lam, std::vector<double>& V) {
  auto at = [&](int i, int j) -> double& { return A[static_cast<size_t>(i) * n + j]; };
  std::vector<double> Q(static_cast<size_t>(n) * n, 0.0);
  for (int i = 0; i < n; ++i) Q[static_cast<size_t>(i) * n + i] = 1.0;
  auto q = [&](int i, int j) -> double& { return Q[static_cast<size_t>(i) * n + j]; };
  // ---- A = Q T Q^T with T tridiagonal: reflection H_k = I - beta v v^T zeroes column k
  // below its subdiagonal; the trailing block becomes H A22 H = A22 - v w^T - w v^T with
  // p = beta A22 v, w = p - (beta / 2)(v^T p) v.
  std::vector<double> v(n), p(n), w(n);
  for (int k = 0; k + 2 < n; ++k) {
    double sigma = 0.0;
    for (int i = k + 1; i < n; ++i) sigma += at(i, k) * at(i, k);
    if (sigma == 0.0) continue;
    const double x0 = at(k + 1, k);
    const double alpha = x0 > 0.0 ? -std::sqrt(sigma) : std::sqrt(sigma);
    for (int i = k + 1; i < n; ++i) v[i] = at(i, k);
    v[k + 1] -= alpha;
    const double vtv = sigma - 2.0 * alpha * x0 + alpha * alpha;
    if (!(vtv > 0.0)) continue;
    const double beta = 2.0 / vtv;
    double vp = 0.0;
    for (int i = k + 1; i < n; ++i) {
      double acc = 0.0;
      for (int j = k + 1; j < n; ++j) acc += at(i, j) * v[j];
      p[i] = beta * acc;
      vp += v[i] * p[i];
    }
    const double K = 0.5 * beta * vp;
    for (int i = k + 1; i < n; ++i) w[i] = p[i] - K * v[i];
    for (int i = k + 1; i < n; ++i)
      for (int j = k + 1; j < n; ++j) at(i, j) -= v[i] * w[j] + w[i] * v[j];
    at(k + 1, k) = at(k, k + 1) = alpha;
    for (int i = k + 2; i < n; ++i) at(i, k) = at(k, i) = 0.0;
    for (int r = 0; r < n; ++r) {  // Q <- Q H_k
      double t = 0.0;
      for (int i = k + 1; i < n; ++i) t += q(r, i) * v[i];
      t *= beta;
      for (int i = k + 1; i < n; ++i) q(r, i) -= t * v[i];
    }
  }
  // ---- implicit QR on the unreduced blocks of T, deflating from the bottom.  A plane
  // rotation J on (k, k+1) (c, s with J^T [x; z] = [r; 0]) is applied as T <- J^T T J on
  // the band window rows/columns k-1 .. k+2 and accumulated as Q <- Q J.
  const double eps = std::ldexp(1.0, -52);
  auto rotate = [&](int k, double c, double s) {
    const int lo = std::max(0, k - 1), hi = std::min(n - 1, k + 2);
    for (int i = lo; i <= hi; ++i) {  // columns k, k+1
      const double a = at(i, k), b = at(i, k + 1);
      at(i, k) = c * a - s * b;
      at(i, k + 1) = s * a + c * b;
    }
    for (int j = lo; j <= hi; ++j) {  // rows k, k+1
      const double a = at(k, j), b = at(k + 1, j);
      at(k, j) = c * a - s * b;
      at(k + 1, j) = s * a + c * b;
    }
    for (int r = 0; r < n; ++r) {
      const double a = q(r, k), b = q(r, k + 1);
      q(r, k) = c * a - s * b;
      q(r, k + 1) = s * a + c * b;
    }
  };
  int steps = 0;
  for (;;) {
    for (int i = 0; i + 1 < n; ++i)
      if (std::fabs(at(i + 1, i)) <= eps * (std::fabs(at(i, i)) + std::fabs(at(i + 1, i + 1))))
        at(i + 1, i) = at(i, i + 1) = 0.0;
    int hi = n - 1;
    while (hi > 0 && at(hi, hi - 1) == 0.0) --hi;
    if (hi == 0) break;
    int lo = hi - 1;
    while (lo > 0 && at(lo, lo - 1) != 0.0) --lo;
    if (++steps > 60 * n) return false;
    // Wilkinson shift: the eigenvalue of the trailing 2x2 block nearer to its last entry
    const double a = at(hi - 1, hi - 1), b = at(hi, hi - 1), cc = at(hi, hi);
    const double t = 0.5 * (a - cc);
    const double mu = cc - b * b / (t + std::copysign(std::hypot(t, b), t == 0.0 ? 1.0 : t));
    double x = at(lo, lo) - mu, z = at(lo + 1, lo);
    for (int k = lo; k < hi; ++k) {
      const double r = std::hypot(x, z);
      const double c = r == 0.0 ? 1.0 : x / r, s = r == 0.0 ? 0.0 : -z / r;
      rotate(k, c, s);
      if (k + 1 < hi) {
        x = at(k + 1, k);
        z = at(k + 2, k);
      }
    }
  }
  // ---- order and signs as jacobi_eig
  std::vector<int> idx(n);
  for (int i = 0; i < n; ++i) idx[i] = i;
  std::stable_sort(idx.begin(), idx.end(), [&](int x1, int x2) { return at(x1, x1) > at(x2, x2); });
  lam.resize(n);
  V.assign(static_cast<size_t>(n) * n, 0.0);
  for (int j = 0; j < n; ++j) {
    const int src = idx[j];
    lam[j] = at(src, src);
    int kmax = 0;
    for (int k = 1; k < n; ++k)
      if (std::fabs(q(k, src)) > std::fabs(q(kmax, src))) kmax = k;
    const double sgn = q(kmax, src) < 0 ? -1.0 : 1.0;
    for (int k = 0; k < n; ++k) V[static_cast<size_t>(k) * n + j] = sgn * q(k, src);
  }
  return true;
}

// ------------------------------------------------------------------ model pieces
double q_of_b(int b) { return std::ldexp(1.0, -2 * b) / 12.0; }

// D(r,b) = sum_{i>r} w_i + q(b) sum_{i<=r} w_i (w sorted descending).
double distortion(const std::vector<double>& w, int r, int b) {
  double tail = 0.0, head = 0.0;
  for (int i = r; i < static_cast<int>(w.size()); ++i) tail += w[i];
  for (int i = 0; i < r; ++i) head += w[i];
  return tail + q_of_b(b) * head;
}

// C1: b = min(8, floor(B/r)), feasible iff b >= 2; min D, ties -> fewer bits, smaller r.
bool c1(const std::vector<double>& w, int B, int& r_out, int& b_out) {
  bool found = false;
  double bestD = 0.0;
  int bestBits = 0, bestR = 0, bestB = 0;
  int d = static_cast<int>(w.size());
  for (int r = 2; r <= d; r += 2) {
    int b = std::min(8, B / r);
    if (b < 2) continue;
    double D = distortion(w, r, b);
    bool better = !found || D < bestD || (D == bestD && (r * b < bestBits || (r * b == bestBits && r < bestR)));
    if (better) {
      found = true;
      bestD = D;
      bestBits = r * b;
      bestR = r;
      bestB = b;
    }
  }
  r_out = bestR;
  b_out = bestB;
  return found;
}

struct Cand {
  int r, b, bits;
};

// Candidates (r even in [2,d], b in [2,8]) ordered by (bits, r).
std::vector<Cand> candidates(int d) {
  std::vector<Cand> c;
  for (int r = 2; r <= d; r += 2)
    for (int b = 2; b <= 8; ++b) c.push_back({r, b, r * b});
  std::stable_sort(c.begin(), c.end(), [](const Cand& x, const Cand& y) {
    return x.bits != y.bits ? x.bits < y.bits : x.r < y.r;
  });
  return c;
}

// Lower convex hull of one unit's candidate points (bits, D), given in (bits, r) order:
// the corners of C1's distortion-versus-budget curve.  x increasing, y strictly falling.
std::vector<std::pair<int, double>> hull_points(const std::vector<Cand>& cand, const double* D) {
  std::vector<std::pair<int, double>> stair, hull;
  for (size_t c = 0; c < cand.size(); ++c) {
    const int x = cand[c].bits;
    const double y = D[c];
    if (!stair.empty() && y >= stair.back().second) continue;
    if (!stair.empty() && stair.back().first == x) stair.pop_back();
    stair.emplace_back(x, y);
  }
  for (const auto& p : stair) {
    while (hull.size() >= 2) {
      const auto& a = hull[hull.size() - 2];
      const auto& b = hull.back();
      // b on or above the segment a -> p
      if ((b.second - a.second) * static_cast<double>(p.first - a.first) >=
          (p.second - a.second) * static_cast<double>(b.first - a.first))
        hull.pop_back();
      else
        break;
    }
    hull.push_back(p);
  }
  return hull;
}

// Distortion saved per extra bit at budget B on a unit's hull: the slope of the segment
// holding B, the mean of the two adjacent slopes at a corner, 0 past the last corner.
double hull_marginal(const std::vector<std::pair<int, double>>& h, double B) {
  const size_t n = h.size();
  size_t k = 0;
  while (k + 1 < n && static_cast<double>(h[k + 1].first) <= B) ++k;
  if (k + 1 >= n) return 0.0;
  const double right = (h[k].second - h[k + 1].second) / static_cast<double>(h[k + 1].first - h[k].first);
  if (B == static_cast<double>(h[k].first) && k > 0) {
    const double left = (h[k - 1].second - h[k].second) / static_cast<double>(h[k].first - h[k - 1].first);
    return 0.5 * (left + right);
  }
  return right;
}

// C2 in the pages' iterative form ("C2, across heads": with C1 as the oracle, budget moves
// between heads until their marginal distortions equalize, the water-filling condition; a
// damped update converges in five rounds).  The water-filling condition is a common level
// mu of marginal distortion per bit: at a level every unit holds the corner of C1's
// distortion-versus-budget curve where its marginal falls to mu (argmin D + mu * bits,
// ties to fewer bits, then smaller r), so only the level is iterated.  Level 0: the mean
// hull marginal at the equal split.  Each round, with S the bits and R the summed ranks of
// the picks: ln mu <- ln mu - 0.7 * 2 ln 2 * (total - S) / R (a damped Newton step; R / 2 ln 2
// is the high-rate model's -dS/d ln mu).  After five rounds the picks at the final level
// are fitted: while over budget, the downgrade with the smallest distortion increase per
// bit saved; then the leftover bits go to the upgrade with the largest drop per bit.  Each
// unit gets C1 at its pick's bits.  Same operations and order as the oracle.
bool c2_damped(const std::vector<std::vector<double>>& ws, long long total_bits, std::vector<int>& r_out,
               std::vector<int>& b_out, double& mu_out) {
  const int U = static_cast<int>(ws.size());
  const int d = static_cast<int>(ws[0].size());
  const std::vector<Cand> cand = candidates(d);
  const int n = static_cast<int>(cand.size());
  const int rounds = 5;
  const double damping = 0.7;
  std::vector<double> D(static_cast<size_t>(U) * n);
  for (int u = 0; u < U; ++u)
    for (int c = 0; c < n; ++c) D[static_cast<size_t>(u) * n + c] = distortion(ws[u], cand[c].r, cand[c].b);
  auto pick = [&](int u, double mu) {
    int best = 0;
    double bv = D[static_cast<size_t>(u) * n] + mu * static_cast<double>(cand[0].bits);
    for (int c = 1; c < n; ++c) {
      const double v = D[static_cast<size_t>(u) * n + c] + mu * static_cast<double>(cand[c].bits);
      if (v < bv) {
        bv = v;
        best = c;
      }
    }
    return best;
  };
  const double B0 = static_cast<double>(total_bits) / U;
  double msum = 0.0;
  for (int u = 0; u < U; ++u) msum += hull_marginal(hull_points(cand, &D[static_cast<size_t>(u) * n]), B0);
  const double mbar = msum / U;
  double mu = 0.0;
  if (mbar > 0.0) {
    double lmu = std::log(mbar);
    for (int round = 0; round < rounds; ++round) {
      const double m = std::exp(lmu);
      long long S = 0, rsum = 0;
      for (int u = 0; u < U; ++u) {
        const int c = pick(u, m);
        S += cand[c].bits;
        rsum += cand[c].r;
      }
      lmu = lmu - damping * (2.0 * std::log(2.0)) * static_cast<double>(total_bits - S) / static_cast<double>(rsum);
    }
    mu = std::exp(lmu);
  }
  std::vector<int> sel(U);
  long long used = 0;
  for (int u = 0; u < U; ++u) {
    sel[u] = pick(u, mu);
    used += cand[sel[u]].bits;
  }
  while (used > total_bits) {  // over budget: the cheapest downgrade per bit saved
    int bu = -1, bc = -1;
    double bcost = 0.0;
    for (int u = 0; u < U; ++u) {
      const int b0 = cand[sel[u]].bits;
      const double D0 = D[static_cast<size_t>(u) * n + sel[u]];
      for (int c = 0; c < n; ++c) {
        const int saved = b0 - cand[c].bits;
        if (saved <= 0) continue;
        const double cost = (D[static_cast<size_t>(u) * n + c] - D0) / saved;
        if (bu < 0 || cost < bcost) {
          bu = u;
          bc = c;
          bcost = cost;
        }
      }
    }
    if (bu < 0) return false;
    used -= cand[sel[bu]].bits - cand[bc].bits;
    sel[bu] = bc;
  }
  long long left = total_bits - used;
  for (;;) {  // leftover: the best drop per bit that fits
    int bu = -1, bc = -1;
    double bg = 0.0;
    for (int u = 0; u < U; ++u) {
      const int b0 = cand[sel[u]].bits;
      const double D0 = D[static_cast<size_t>(u) * n + sel[u]];
      for (int c = 0; c < n; ++c) {
        const int extra = cand[c].bits - b0;
        const double Dc = D[static_cast<size_t>(u) * n + c];
        if (extra <= 0 || extra > left || !(Dc < D0)) continue;
        const double g = (D0 - Dc) / extra;
        if (bu < 0 || g > bg) {
          bu = u;
          bc = c;
          bg = g;
        }
      }
    }
    if (bu < 0) break;
    left -= cand[bc].bits - cand[sel[bu]].bits;
    sel[bu] = bc;
  }
  r_out.assign(U, 0);
  b_out.assign(U, 0);
  for (int u = 0; u < U; ++u)
    if (!c1(ws[u], cand[sel[u]].bits, r_out[u], b_out[u])) return false;
  mu_out = mu;
  return true;
}

// C2 in Lagrangian form: bisect mu so that sum_u bits(argmin D_u + mu*bits) fits the
// budget, spend the leftover greedily on the best distortion drop per bit, and give each
// unit C1 at its resulting budget.
bool c2(const std::vector<std::vector<double>>& ws, long long total_bits, std::vector<int>& r_out,
        std::vector<int>& b_out, double& mu_out) {
  const int U = static_cast<int>(ws.size());
  const int d = static_cast<int>(ws[0].size());
  const std::vector<Cand> cand = candidates(d);
  const int n = static_cast<int>(cand.size());
  std::vector<double> D(static_cast<size_t>(U) * n);
  for (int u = 0; u < U; ++u)
    for (int c = 0; c < n; ++c) D[static_cast<size_t>(u) * n + c] = distortion(ws[u], cand[c].r, cand[c].b);
  auto pick = [&](int u, double mu) {
    int best = 0;
    double bv = D[static_cast<size_t>(u) * n] + mu * static_cast<double>(cand[0].bits);
    for (int c = 1; c < n; ++c) {
      double v = D[static_cast<size_t>(u) * n + c] + mu * static_cast<double>(cand[c].bits);
      if (v < bv) {
        bv = v;
        best = c;
      }
    }
    return best;
  };
  auto bits_at = [&](double mu) {
    long long t = 0;
    for (int u = 0; u < U; ++u) t += cand[pick(u, mu)].bits;
    return t;
  };
  double lo = 0.0, hi = 1.0;
  while (bits_at(hi) > total_bits) {
    hi *= 2.0;
    if (hi > 1e300) return false;
  }
  if (bits_at(lo) <= total_bits) {
    hi = lo;
  } else {
    for (int it = 0; it < 200; ++it) {
      double mid = 0.5 * (lo + hi);
      if (bits_at(mid) <= total_bits)
        hi = mid;
      else
        lo = mid;
    }
  }
  std::vector<int> sel(U);
  long long used = 0;
  for (int u = 0; u < U; ++u) {
    sel[u] = pick(u, hi);
    used += cand[sel[u]].bits;
  }
  long long left = total_bits - used;
  for (;;) {
    int bu = -1, bc = -1;
    double bg = 0.0;
    for (int u = 0; u < U; ++u) {
      const int b0 = cand[sel[u]].bits;
      const double D0 = D[static_cast<size_t>(u) * n + sel[u]];
      for (int c = 0; c < n; ++c) {
        const int extra = cand[c].bits - b0;
        const double Dc = D[static_cast<size_t>(u) * n + c];
        if (extra <= 0 || extra > left || !(Dc < D0)) continue;
        const double g = (D0 - Dc) / extra;
        if (bu < 0 || g > bg) {
          bu = u;
          bc = c;
          bg = g;
        }
      }
    }
    if (bu < 0) break;
    left -= cand[bc].bits - cand[sel[bu]].bits;
    sel[bu] = bc;
  }
  r_out.resize(U);
  b_out.resize(U);
  for (int u = 0; u < U; ++u)
    if (!c1(ws[u], cand[sel[u]].bits, r_out[u], b_out[u])) return false;
  mu_out = hi;
  return true;
}

// ------------------------------------------------------------------ quantizer step
double phi(double x) { return std::isfinite(x) ? std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI) : 0.0; }
double Phi(double x) {
  if (x == INFINITY) return 1.0;
  if (x == -INFINITY) return 0.0;
  return 0.5 * std::erfc(-x / std::sqrt(2.0));
}

// Slope of the MSE of the 2^b-level mid-rise uniform quantizer on N(0,1) w.r.t. its step.
double mse_slope(double step, int b) {
  const int L = 1 << b;
  double t = 0.0;
  for (int k = 0; k < L; ++k) {
    double lo = k == 0 ? -INFINITY : (k - L / 2.0) * step;
    double hi = k == L - 1 ? INFINITY : (k + 1 - L / 2.0) * step;
    double ck = k - (L - 1) / 2.0;
    t += ck * (phi(lo) - phi(hi) - ck * step * (Phi(hi) - Phi(lo)));
  }
  return -2.0 * t;
}

// g(b): root of the slope by bisection.
double gaussian_step(int b) {
  double lo = 1e-3, hi = 4.0;
  for (int it = 0; it < 200; ++it) {
    double mid = 0.5 * (lo + hi);
    if (mse_slope(mid, b) < 0.0)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

// ------------------------------------------------------------------ Hadamard
uint64_t splitmix64_at(uint64_t seed, uint64_t n) {
  uint64_t z = seed + (n + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// y = H_r x in place for the orthonormal block Walsh-Hadamard of order r: diagonal
// blocks of the powers of two of r's binary expansion, largest first; a block of order n
// is the Sylvester matrix (entry sign (-1)^popcount(i & j), H_2n = [[H_n, H_n],
// [H_n, -H_n]], applied as butterflies) times 1/sqrt(n).
void block_hadamard_apply(int r, double* x) {
  int off = 0;
  for (int bit = 30; bit >= 0; --bit) {
    const int n = 1 << bit;
    if (!(r & n)) continue;
    double* y = x + off;
    for (int len = 1; len < n; len <<= 1)
      for (int i = 0; i < n; i += 2 * len)
        for (int j = i; j < i + len; ++j) {
          const double a = y[j], c = y[j + len];
          y[j] = a + c;
          y[j + len] = a - c;
        }
    const double s = 1.0 / std::sqrt(static_cast<double>(n));
    for (int j = 0; j < n; ++j) y[j] *= s;
    off += n;
  }
}

struct UnitWork {
  std::vector<double> w, lam, Vs;  // Vs: d x d row-major, column i = i-th sorted vector
};

}  // namespace
}  // namespace kvtc

using namespace kvtc;

extern "C" kvtc_status kvtc_calibrate(const kvtc_calib_desc* desc, const float* k_cal, const float* v_cal,
                                      const float* q_cal, kvtc_plan** out) {
  if (!desc || !k_cal || !v_cal || !out) return fail(KVTC_EINVAL, "null argument");
  *out = nullptr;
  const int L = desc->n_layers, H = desc->n_kv_heads, G = desc->group, d = desc->head_dim, N = desc->n_cal;
  if (L < 1 || H < 1 || G < 1 || N < 2) return fail(KVTC_EINVAL, "bad calibration shape");
  if (d != kD) return fail(KVTC_EINVAL, "head_dim must be 128");
  const bool kl = desc->weight_mode == KVTC_WEIGHTS_KL;
  if (!kl && desc->weight_mode != KVTC_WEIGHTS_MSE) return fail(KVTC_EINVAL, "bad weight_mode");
  if (kl && !q_cal) return fail(KVTC_EINVAL, "KL weights need calibration queries");
  const bool fixed = desc->fixed_r > 0 || desc->fixed_b > 0;
  if (fixed && (desc->fixed_r < 2 || desc->fixed_r > d || (desc->fixed_r & 1) || desc->fixed_b < 2 ||
                desc->fixed_b > 8))
    return fail(KVTC_EINVAL, "fixed_r must be even in [2,128] and fixed_b in [2,8]");
  const int U = 2 * L * H;
  using clock = std::chrono::steady_clock;
  const auto t0 = clock::now();
  if (!fixed && !(desc->bpd > 0.0)) return fail(KVTC_EINVAL, "bpd must be > 0");

  std::vector<UnitWork> work(U);
  std::atomic<int> next(0);
  auto worker = [&]() {
    std::vector<double> C(static_cast<size_t>(d) * d), lam, V;
    for (;;) {
      int u = next.fetch_add(1);
      if (u >= U) break;
      const int kind = u & 1, head = (u >> 1) % H, layer = (u >> 1) / H;
      const float* X = (kind == 0 ? k_cal : v_cal) + (static_cast<size_t>(layer) * H + head) * N * d;
      std::fill(C.begin(), C.end(), 0.0);
      for (int t = 0; t < N; ++t) {
        const float* x = X + static_cast<size_t>(t) * d;
        for (int i = 0; i < d; ++i) {
          const double xi = x[i];
          double* row = &C[static_cast<size_t>(i) * d];
          for (int j = i; j < d; ++j) row[j] += xi * static_cast<double>(x[j]);
        }
      }
      for (int i = 0; i < d; ++i)
        for (int j = i; j < d; ++j) {
          C[i * d + j] /= N;
          C[j * d + i] = C[i * d + j];
        }
      std::vector<double> C0 = C;
      if (!tridiag_qr_eig(C, d, lam, V)) jacobi_eig(C0, d, lam, V);
      std::vector<double> wraw(lam);
      if (kind == 0 && kl) {
        const float* Q = q_cal + (static_cast<size_t>(layer) * H + head) * G * N * d;
        std::vector<double> sq(d, 0.0), proj(d);
        const size_t nq = static_cast<size_t>(G) * N;
        for (size_t t = 0; t < nq; ++t) {
          const float* q = Q + t * d;
          std::fill(proj.begin(), proj.end(), 0.0);
          for (int k = 0; k < d; ++k) {
            const double qk = q[k];
            const double* vr = &V[static_cast<size_t>(k) * d];
            for (int i = 0; i < d; ++i) proj[i] += qk * vr[i];
          }
          for (int i = 0; i < d; ++i) sq[i] += proj[i] * proj[i];
        }
        for (int i = 0; i < d; ++i) wraw[i] = (sq[i] / nq) * lam[i];
      }
      std::vector<int> ord(d);
      for (int i = 0; i < d; ++i) ord[i] = i;
      std::stable_sort(ord.begin(), ord.end(), [&](int a, int b) { return wraw[a] > wraw[b]; });
      UnitWork& wk = work[u];
      wk.w.resize(d);
      wk.lam.resize(d);
      wk.Vs.resize(static_cast<size_t>(d) * d);
      for (int i = 0; i < d; ++i) {
        wk.w[i] = wraw[ord[i]];
        wk.lam[i] = lam[ord[i]];
        for (int k = 0; k < d; ++k) wk.Vs[static_cast<size_t>(k) * d + i] = V[static_cast<size_t>(k) * d + ord[i]];
      }
    }
  };
  unsigned nth = std::max(1u, std::min(std::thread::hardware_concurrency(), 64u));
  nth = std::min<unsigned>(nth, static_cast<unsigned>(U));
  {
    std::vector<std::thread> pool;
    for (unsigned i = 1; i < nth; ++i) pool.emplace_back(worker);
    worker();
    for (auto& t : pool) t.join();
  }
  const auto t1 = clock::now();

  std::vector<int> R(U), B(U);
  double mu = 0.0;
  if (desc->c2_mode != KVTC_C2_LAGRANGE && desc->c2_mode != KVTC_C2_DAMPED)
    return fail(KVTC_EINVAL, "c2_mode must be KVTC_C2_LAGRANGE or KVTC_C2_DAMPED");
  // The allocation pool: every unit, or the key units alone in keys-only mode (value
  // units are then stored uncompressed: r = d, b = kRawBits).
  if (desc->k_only != 0 && desc->k_only != 1) return fail(KVTC_EINVAL, "k_only must be 0 or 1");
  std::vector<int> pool;
  for (int u = 0; u < U; ++u)
    if (!(desc->k_only && (u & 1))) pool.push_back(u);
  const int P = static_cast<int>(pool.size());
  std::vector<int> Rp(P), Bp(P);
  if (fixed) {
    std::fill(Rp.begin(), Rp.end(), desc->fixed_r);
    std::fill(Bp.begin(), Bp.end(), desc->fixed_b);
  } else {
    const long long total = std::llround(desc->bpd * d * P);
    if (4ll * P > total) return fail(KVTC_EINFEASIBLE, "budget below 4 bits per unit");
    std::vector<std::vector<double>> ws(P);
    for (int i = 0; i < P; ++i) ws[i] = work[pool[i]].w;
    if (desc->c2_mode == KVTC_C2_DAMPED) {
      if (!c2_damped(ws, total, Rp, Bp, mu)) return fail(KVTC_EINFEASIBLE, "no allocation meets the budget");
    } else if (!c2(ws, total, Rp, Bp, mu)) {
      return fail(KVTC_EINFEASIBLE, "no allocation meets the budget");
    }
  }
  std::fill(R.begin(), R.end(), d);
  std::fill(B.begin(), B.end(), kRawBits);
  for (int i = 0; i < P; ++i) {
    R[pool[i]] = Rp[i];
    B[pool[i]] = Bp[i];
  }
  const auto t2 = clock::now();

  std::unique_ptr<kvtc_plan> p(new (std::nothrow) kvtc_plan());
  if (!p) return fail(KVTC_ENOMEM, "out of host memory");
  p->L = L;
  p->H = H;
  p->G = G;
  p->d = d;
  p->U = U;
  p->mu = mu;
  p->t_stats = std::chrono::duration<double>(t1 - t0).count();
  p->t_alloc = std::chrono::duration<double>(t2 - t1).count();
  double gstep[9] = {0};
  for (int b = 2; b <= 8; ++b) gstep[b] = gaussian_step(b);
  for (int u = 0; u < U; ++u) {
    const int r = R[u], b = B[u];
    const UnitWork& wk = work[u];
    if (b == kRawBits) {  // uncompressed value unit: identity basis, c = v * 2^24
      std::vector<float> M(static_cast<size_t>(d) * d, 0.0f);
      for (int i = 0; i < d; ++i) M[static_cast<size_t>(i) * d + i] = 1.0f;
      p->r.push_back(d);
      p->b.push_back(b);
      p->delta.push_back(std::ldexp(1.0, -24));
      p->inv_delta.push_back(std::ldexp(1.0f, 24));
      p->sigma.push_back(0.0);
      p->D.push_back(0.0);
      p->M.push_back(std::move(M));
      p->w.push_back(wk.w);
      p->lam.push_back(wk.lam);
      continue;
    }
    double mean = 0.0;
    for (int i = 0; i < r; ++i) mean += wk.lam[i];
    mean /= r;
    const double sigma = std::sqrt(mean);
    const double delta = gstep[b] * sigma;
    std::vector<double> eps(r);
    for (int i = 0; i < r; ++i) eps[i] = (splitmix64_at(desc->seed, static_cast<uint64_t>(u) * 256 + i) >> 63) ? -1.0 : 1.0;
    // M = H_r diag(eps) V_r^T, one column k at a time: the transform of eps .* V_r[k, :]
    std::vector<float> M(static_cast<size_t>(r) * d);
    std::vector<double> col(r);
    for (int k = 0; k < d; ++k) {
      for (int j = 0; j < r; ++j) col[j] = eps[j] * wk.Vs[static_cast<size_t>(k) * d + j];
      block_hadamard_apply(r, col.data());
      for (int i = 0; i < r; ++i) M[static_cast<size_t>(i) * d + k] = static_cast<float>(col[i]);
    }
    p->r.push_back(r);
    p->b.push_back(b);
    p->delta.push_back(delta);
    p->inv_delta.push_back(static_cast<float>(1.0 / delta));
    p->sigma.push_back(sigma);
    p->D.push_back(distortion(wk.w, r, b));
    p->M.push_back(std::move(M));
    p->w.push_back(wk.w);
    p->lam.push_back(wk.lam);
  }
  *out = p.release();
  return KVTC_OK;
}
