"""Seeded synthetic workloads (inputs only: this module holds none of the codec's
arithmetic).  Both the CUDA path's tests/bench and the CPU oracle take their inputs
from here, as arrays.

Recipe, per unit (layer, KV head, kind K|V):
  lambda_i = i^(-alpha), i = 1..d;  U Haar-orthogonal (QR of a Gaussian matrix, with
  the sign of R's diagonal folded into Q);  a token is x = (z * sqrt(lambda)) U^T with
  z ~ N(0, I_d), after which n_out distinct channels (chosen uniformly) are scaled x10.
  alpha and n_out are either fixed (the 1-head parity workload: alpha 1.5, 2 outlier
  channels) or drawn per unit: alpha ~ U[0.5, 2.0], n_out ~ U{1..4}.
Queries of query head g reading KV head h: q = (sigma_Q * z) U_K^T, with U_K the key
  unit's rotation and sigma^2_Q,i ~ LogNormal(0, 1) drawn per query head (the 1-head
  workload uses sigma^2_Q = 1).
Calibration: 512 tokens per unit and 512 queries per query head.  Cache tokens and
the decode query are fresh draws.  bf16 workloads draw in fp32 and round to bf16.

Every draw has its own stream: numpy SeedSequence([seed, layer, head, kind, purpose,
extra]).  Large caches are drawn on the device with a torch.Generator seeded from the
same tuple (different numbers from the numpy stream, same distribution); the oracle
then receives the device's bytes.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

D_HEAD = 128
PURPOSE_SPEC, PURPOSE_CAL, PURPOSE_CACHE, PURPOSE_QSPEC, PURPOSE_QCAL, PURPOSE_QDEC = range(6)


@dataclass(frozen=True)
class Workload:
    """A synthetic workload: model shape, cache shape and budget."""
    name: str
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    seq_len: int
    batch: int
    bpd: float
    dtype: str                  # "f32" or "bf16"
    seed: int
    fixed_r: int = 0
    fixed_b: int = 0
    alpha: float | None = None  # fixed spectral exponent, else U[0.5, 2]
    n_out: int | None = None    # fixed outlier count, else U{1..4}
    unit_query_var: bool = False
    n_cal: int = 512
    head_dim: int = D_HEAD

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


# The five workloads.  Sizes follow the Llama-3.1-8B / Qwen2.5-7B attention shapes.
WORKLOADS = {
    "head1-fp32-1k": Workload("head1-fp32-1k", 1, 1, 1, 1024, 1, 0.5, "f32", 1,
                              fixed_r=16, fixed_b=4, alpha=1.5, n_out=2, unit_query_var=True),
    "llama8b-layer-32k-2bpd": Workload("llama8b-layer-32k-2bpd", 1, 32, 8, 32768, 1, 2.0, "bf16", 2),
    "llama8b-32L-128k-1bpd": Workload("llama8b-32L-128k-1bpd", 32, 32, 8, 131072, 1, 1.0, "bf16", 3),
    "llama8b-32L-b16x32k": Workload("llama8b-32L-b16x32k", 32, 32, 8, 32768, 16, 1.0, "bf16", 4),
    "qwen7b-28L-128k-2bpd": Workload("qwen7b-28L-128k-2bpd", 28, 28, 4, 131072, 1, 2.0, "bf16", 5),
}


def with_bpd(w: Workload, bpd: float) -> Workload:
    """The same workload (same seeded spectra) at another budget."""
    from dataclasses import replace
    return replace(w, bpd=bpd, name=f"{w.name.split('@')[0]}@{bpd:g}bpd")


def scaled(w: Workload, **kw) -> Workload:
    """A smaller copy of a workload (tests at reduced sizes keep its spectra)."""
    from dataclasses import replace
    return replace(w, **kw)


def rng_for(seed, layer, head, kind, purpose, extra=0):
    return np.random.default_rng(np.random.SeedSequence([seed, layer, head, kind, purpose, extra]))


def seed_int(seed, layer, head, kind, purpose, extra=0):
    ss = np.random.SeedSequence([seed, layer, head, kind, purpose, extra])
    return int(ss.generate_state(1, np.uint64)[0] & np.uint64((1 << 63) - 1))


def haar_orthogonal(rng, d):
    Z = rng.standard_normal((d, d))
    Q, R = np.linalg.qr(Z)
    return Q * np.sign(np.diag(R))[None, :]


@dataclass
class UnitSpec:
    alpha: float
    channels: np.ndarray
    U: np.ndarray
    lam: np.ndarray = field(repr=False)


def unit_spec(w: Workload, layer: int, head: int, kind: int) -> UnitSpec:
    rng = rng_for(w.seed, layer, head, kind, PURPOSE_SPEC)
    d = w.head_dim
    alpha = w.alpha if w.alpha is not None else float(rng.uniform(0.5, 2.0))
    n_out = w.n_out if w.n_out is not None else int(rng.integers(1, 5))
    channels = np.sort(rng.choice(d, size=n_out, replace=False))
    U = haar_orthogonal(rng, d)
    lam = np.arange(1, d + 1, dtype=np.float64) ** (-alpha)
    return UnitSpec(alpha, channels, U, lam)


def draw_tokens(spec: UnitSpec, n: int, rng) -> np.ndarray:
    d = spec.U.shape[0]
    z = rng.standard_normal((n, d))
    x = (z * np.sqrt(spec.lam)[None, :]) @ spec.U.T
    x[:, spec.channels] *= 10.0
    return x.astype(np.float32)


def query_var(w: Workload, layer: int, qhead: int) -> np.ndarray:
    if w.unit_query_var:
        return np.ones(w.head_dim)
    rng = rng_for(w.seed, layer, qhead, 0, PURPOSE_QSPEC)
    return np.exp(rng.standard_normal(w.head_dim))


def draw_queries(kspec: UnitSpec, sigma2: np.ndarray, n: int, rng) -> np.ndarray:
    z = rng.standard_normal((n, kspec.U.shape[0]))
    return ((z * np.sqrt(sigma2)[None, :]) @ kspec.U.T).astype(np.float32)


def round_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Store in the workload's dtype (bf16 values returned as exactly-representable
    fp32 via round-to-nearest-even)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    u = x.view(np.uint32).astype(np.uint64)
    out = (((u + (((u >> 16) & 1) + 0x7FFF)) >> 16) << 16).astype(np.uint32)
    return out.view(np.float32)


def calibration_set(w: Workload, layers=None):
    """k_cal, v_cal [L, H_kv, n_cal, d] and q_cal [L, H_kv, G, n_cal, d] (fp32 arrays
    holding values of the workload dtype)."""
    layers = range(w.n_layers) if layers is None else layers
    L = len(list(layers))
    H, G, N, d = w.n_kv_heads, w.group, w.n_cal, w.head_dim
    k = np.zeros((L, H, N, d), np.float32)
    v = np.zeros((L, H, N, d), np.float32)
    q = np.zeros((L, H, G, N, d), np.float32)
    for li, layer in enumerate(layers):
        for h in range(H):
            ks = unit_spec(w, layer, h, 0)
            vs = unit_spec(w, layer, h, 1)
            k[li, h] = round_dtype(draw_tokens(ks, N, rng_for(w.seed, layer, h, 0, PURPOSE_CAL)), w.dtype)
            v[li, h] = round_dtype(draw_tokens(vs, N, rng_for(w.seed, layer, h, 1, PURPOSE_CAL)), w.dtype)
            for g in range(G):
                qh = h * G + g
                q[li, h, g] = round_dtype(draw_queries(
                    ks, query_var(w, layer, qh), N, rng_for(w.seed, layer, qh, 0, PURPOSE_QCAL)), w.dtype)
    return k, v, q


def cache_tokens(w: Workload, layer: int, head: int, kind: int, n: int, seq: int = 0) -> np.ndarray:
    """n cache tokens of one unit of sequence ``seq`` (numpy; small workloads)."""
    spec = unit_spec(w, layer, head, kind)
    return round_dtype(draw_tokens(spec, n, rng_for(w.seed, layer, head, kind, PURPOSE_CACHE, seq)), w.dtype)


def decode_queries(w: Workload, layer: int, seq: int = 0) -> np.ndarray:
    """The decode-step queries [H_q, d] of one sequence."""
    out = np.zeros((w.n_q_heads, w.head_dim), np.float32)
    for qh in range(w.n_q_heads):
        ks = unit_spec(w, layer, qh // w.group, 0)
        out[qh] = draw_queries(ks, query_var(w, layer, qh), 1,
                               rng_for(w.seed, layer, qh, 0, PURPOSE_QDEC, seq))[0]
    return round_dtype(out, w.dtype)


def layer_kv_torch(w: Workload, layer: int, n: int, device, seq: int = 0, specs=None):
    """Cache K and V of one layer as torch tensors [n, H_kv, d] in the workload dtype,
    drawn on ``device`` (for caches too large for host memory)."""
    import torch
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    out = []
    for kind in (0, 1):
        t = torch.empty((n, w.n_kv_heads, w.head_dim), dtype=dt, device=device)
        for h in range(w.n_kv_heads):
            spec = specs[(layer, h, kind)] if specs else unit_spec(w, layer, h, kind)
            g = torch.Generator(device=device)
            g.manual_seed(seed_int(w.seed, layer, h, kind, PURPOSE_CACHE, seq))
            z = torch.randn((n, w.head_dim), generator=g, device=device, dtype=torch.float32)
            x = (z * torch.from_numpy(np.sqrt(spec.lam)).float().to(device)) @ \
                torch.from_numpy(spec.U.T.copy()).float().to(device)
            x[:, torch.from_numpy(spec.channels).to(device)] *= 10.0
            t[:, h] = x.to(dt)
        out.append(t)
    return out[0], out[1]
