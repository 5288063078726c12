"""ctypes binding of libkvtc (include/kvtc.h): the same entry points, argument
marshalling only.  Every step of the encode/decode path runs in the library's CUDA
kernels; calibration runs in its C++ host code.  There is no Python or CPU fallback:
if libkvtc.so is missing, ``lib()`` raises.

Host arrays are numpy; device buffers are torch CUDA tensors (torch provides device
memory and streams only).
"""
from __future__ import annotations

import ctypes as C
import os
import re

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvtc.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "kvtc.h")

KVTC_F32, KVTC_BF16 = 0, 1
KIND_K, KIND_V = 0, 1
WEIGHTS_KL, WEIGHTS_MSE = 0, 1
C2_LAGRANGE, C2_DAMPED = 0, 1
RAW_BITS = 16  # b of an uncompressed value unit (keys-only plans)
STATUS_BAD_PAGE, STATUS_BAD_POS, STATUS_TIMEOUT = 1, 2, 4
PAGE_TOKENS = 128
HEAD_DIM = 128
STATUS_NAMES = {0: "OK", 1: "EINVAL", 2: "ENOMEM", 3: "ECUDA", 4: "EINFEASIBLE", 5: "ECAPACITY",
                6: "EVERSION", 7: "EIO", 8: "ESTATE"}


class KvtcError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"kvtc {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class CalibDesc(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("n_kv_heads", C.c_int), ("group", C.c_int), ("head_dim", C.c_int),
                ("n_cal", C.c_int), ("bpd", C.c_double), ("weight_mode", C.c_int), ("fixed_r", C.c_int),
                ("fixed_b", C.c_int), ("seed", C.c_uint64), ("c2_mode", C.c_int),
                ("k_only", C.c_int)]


class UnitInfo(C.Structure):
    _fields_ = [("layer", C.c_int), ("head", C.c_int), ("kind", C.c_int), ("r", C.c_int), ("b", C.c_int),
                ("delta", C.c_double), ("inv_delta", C.c_float), ("sigma", C.c_double),
                ("distortion", C.c_double), ("page_bytes", C.c_uint64)]


class CacheDesc(C.Structure):
    _fields_ = [("pool", C.c_void_p), ("pages_per_unit", C.c_uint64), ("block_table", C.c_void_p),
                ("n_seq", C.c_int), ("max_pages", C.c_int), ("status", C.c_void_p)]


_lib = None
_P = C.c_void_p


def lib():
    """Load libkvtc.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m bit_quantization_head_b200.build`")
    L = C.CDLL(LIB_PATH)
    st = C.c_int
    sig = {
        "kvtc_last_error": (C.c_char_p, []),
        "kvtc_version": (C.c_int, []),
        "kvtc_calibrate": (st, [C.POINTER(CalibDesc), _P, _P, _P, C.POINTER(_P)]),
        "kvtc_plan_create": (st, [C.c_int, C.c_int, C.c_int, C.c_int, _P, _P, _P, _P, C.POINTER(_P)]),
        "kvtc_plan_destroy": (None, [_P]),
        "kvtc_plan_shape": (st, [_P, _P, _P, _P, _P, _P]),
        "kvtc_plan_unit": (st, [_P, C.c_int, C.POINTER(UnitInfo)]),
        "kvtc_plan_matrix": (st, [_P, C.c_int, _P]),
        "kvtc_plan_weights": (st, [_P, C.c_int, _P, _P]),
        "kvtc_plan_budget": (st, [_P, C.POINTER(C.c_double), C.POINTER(C.c_uint64)]),
        "kvtc_plan_calib_seconds": (st, [_P, C.POINTER(C.c_double), C.POINTER(C.c_double)]),
        "kvtc_plan_save": (st, [_P, C.c_char_p]),
        "kvtc_plan_load": (st, [C.c_char_p, C.POINTER(_P)]),
        "kvtc_plan_upload": (st, [_P, _P]),
        "kvtc_cache_bytes": (C.c_uint64, [_P, C.c_uint64]),
        "kvtc_unit_pool_offset": (C.c_uint64, [_P, C.c_int, C.c_uint64]),
        "kvtc_encode_append": (st, [_P, C.POINTER(CacheDesc), C.c_int, _P, _P, C.c_int, _P, _P, C.c_int, _P]),
        "kvtc_encode_prefill": (st, [_P, C.POINTER(CacheDesc), C.c_int, _P, _P, C.c_int, C.c_int, C.c_int, _P]),
        "kvtc_plan_prefill_stats": (st, [_P, C.POINTER(C.c_uint64), C.POINTER(C.c_uint64), C.c_int]),
        "kvtc_debug_encode_latent": (st, [_P, C.c_int, C.c_int, C.c_int, _P, C.c_int, C.c_int, _P, _P]),
        "kvtc_decode_workspace_bytes": (C.c_uint64, [_P, C.c_int, C.c_int]),
        "kvtc_decode_attention": (st, [_P, C.POINTER(CacheDesc), C.c_int, _P, C.c_int, _P, C.c_int, C.c_float,
                                       _P, C.c_int, _P, C.c_uint64, _P]),
        "kvtc_decode_attention_noalloc": (st, [_P, C.POINTER(CacheDesc), C.c_int, _P, C.c_int, _P, C.c_int,
                                               C.c_float, _P, C.c_int, _P]),
        "kvtc_decode_attention_rope": (st, [_P, C.POINTER(CacheDesc), C.c_int, _P, C.c_int, _P, C.c_int, C.c_float,
                                            C.c_double, _P, C.c_int, _P, C.c_uint64, _P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def header_entry_points():
    """Names of the functions include/kvtc.h declares."""
    txt = open(HEADER_PATH).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(kvtc_[a-z0-9_]+)\s*\(", txt)))


def _check(status):
    if status != 0:
        raise KvtcError(status, lib().kvtc_last_error().decode())


def _host_ptr(a, dtype):
    assert isinstance(a, np.ndarray) and a.dtype == dtype and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_P)


def _dev_ptr(t):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "device buffers must be contiguous CUDA tensors"
    return _P(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return _P(torch.cuda.current_stream().cuda_stream)
    return _P(stream.cuda_stream if hasattr(stream, "cuda_stream") else stream)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return KVTC_BF16
    if t.dtype == torch.float32:
        return KVTC_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


class Plan:
    """Owner of a kvtc_plan*."""

    def __init__(self, handle):
        self._h = _P(handle) if not isinstance(handle, C.c_void_p) else handle

    def __del__(self):
        try:
            if self._h and self._h.value:
                lib().kvtc_plan_destroy(self._h)
                self._h = _P(None)
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    @property
    def shape(self):
        v = [C.c_int() for _ in range(5)]
        _check(lib().kvtc_plan_shape(self._h, *[C.byref(x) for x in v]))
        return dict(n_layers=v[0].value, n_kv_heads=v[1].value, group=v[2].value, head_dim=v[3].value,
                    n_units=v[4].value)

    def unit(self, u):
        info = UnitInfo()
        _check(lib().kvtc_plan_unit(self._h, u, C.byref(info)))
        return {f: getattr(info, f) for f, _ in UnitInfo._fields_}

    def matrix(self, u):
        r = self.unit(u)["r"]
        out = np.zeros((r, HEAD_DIM), np.float32)
        _check(lib().kvtc_plan_matrix(self._h, u, _host_ptr(out, np.float32)))
        return out

    def weights(self, u):
        w = np.zeros(HEAD_DIM)
        lam = np.zeros(HEAD_DIM)
        _check(lib().kvtc_plan_weights(self._h, u, _host_ptr(w, np.float64), _host_ptr(lam, np.float64)))
        return w, lam

    def budget(self):
        mu, bits = C.c_double(), C.c_uint64()
        _check(lib().kvtc_plan_budget(self._h, C.byref(mu), C.byref(bits)))
        return mu.value, bits.value

    def calib_seconds(self):
        """(statistics and eigen step, C1 + C2 allocation) seconds of kvtc_calibrate."""
        a, b = C.c_double(), C.c_double()
        _check(lib().kvtc_plan_calib_seconds(self._h, C.byref(a), C.byref(b)))
        return a.value, b.value

    def save(self, path):
        _check(lib().kvtc_plan_save(self._h, str(path).encode()))

    def upload(self, stream=None):
        _check(lib().kvtc_plan_upload(self._h, _stream(stream)))
        return self


def kvtc_calibrate(k_cal, v_cal, q_cal, *, n_layers, n_kv_heads, group, bpd=1.0, seed=0,
                   weight_mode=WEIGHTS_KL, fixed_r=0, fixed_b=0, c2_mode=C2_LAGRANGE, k_only=False):
    """Host arrays: k_cal, v_cal fp32 [L][H][N][d]; q_cal fp32 [L][H][G][N][d] (or None).
    k_only: keys-only plan (value units uncompressed, b = RAW_BITS)."""
    k_cal = np.ascontiguousarray(k_cal, np.float32)
    v_cal = np.ascontiguousarray(v_cal, np.float32)
    qp = None
    if q_cal is not None:
        q_cal = np.ascontiguousarray(q_cal, np.float32)
        qp = _host_ptr(q_cal, np.float32)
    d = CalibDesc(n_layers, n_kv_heads, group, k_cal.shape[-1], k_cal.shape[-2], float(bpd), weight_mode,
                  fixed_r, fixed_b, seed, c2_mode, 1 if k_only else 0)
    out = _P()
    _check(lib().kvtc_calibrate(C.byref(d), _host_ptr(k_cal, np.float32), _host_ptr(v_cal, np.float32), qp,
                                C.byref(out)))
    return Plan(out)


def kvtc_plan_create(n_layers, n_kv_heads, group, r, b, delta, M_list, head_dim=HEAD_DIM):
    r = np.ascontiguousarray(r, np.int32)
    b = np.ascontiguousarray(b, np.int32)
    delta = np.ascontiguousarray(delta, np.float64)
    M = np.ascontiguousarray(np.concatenate([np.asarray(m, np.float32).reshape(-1) for m in M_list]), np.float32)
    out = _P()
    _check(lib().kvtc_plan_create(n_layers, n_kv_heads, group, head_dim, _host_ptr(r, np.int32),
                                  _host_ptr(b, np.int32), _host_ptr(delta, np.float64),
                                  _host_ptr(M, np.float32), C.byref(out)))
    return Plan(out)


def kvtc_plan_load(path):
    out = _P()
    _check(lib().kvtc_plan_load(str(path).encode(), C.byref(out)))
    return Plan(out)


def kvtc_cache_bytes(plan, pages_per_unit):
    return int(lib().kvtc_cache_bytes(plan.handle, pages_per_unit))


def kvtc_unit_pool_offset(plan, unit, pages_per_unit):
    return int(lib().kvtc_unit_pool_offset(plan.handle, unit, pages_per_unit))


class Cache:
    """Caller-owned paged code cache: pool, block table and status word (torch CUDA
    tensors), described to the library as a kvtc_cache."""

    def __init__(self, plan, pages_per_unit, block_table, device="cuda"):
        import torch
        self.plan = plan
        self.pages_per_unit = int(pages_per_unit)
        nbytes = kvtc_cache_bytes(plan, self.pages_per_unit)
        self.pool = torch.zeros(max(16, nbytes), dtype=torch.uint8, device=device)
        self.block_table = block_table.to(device=device, dtype=torch.int32).contiguous()
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.desc = CacheDesc(self.pool.data_ptr(), self.pages_per_unit, self.block_table.data_ptr(),
                              self.block_table.shape[0], self.block_table.shape[1], self.status.data_ptr())

    def unit_pool(self, unit):
        """The bytes of one unit's pool (a view of the pool tensor)."""
        off = kvtc_unit_pool_offset(self.plan, unit, self.pages_per_unit)
        pb = self.plan.unit(unit)["page_bytes"]
        return self.pool[off:off + pb * self.pages_per_unit]


def kvtc_encode_append(plan, cache, layer, k, v, cu_seqlens, pos_start, stream=None):
    _check(lib().kvtc_encode_append(plan.handle, C.byref(cache.desc), layer, _dev_ptr(k), _dev_ptr(v),
                                    _dtype_code(k), _dev_ptr(cu_seqlens), _dev_ptr(pos_start), k.shape[0],
                                    _stream(stream)))


def kvtc_encode_prefill(plan, cache, layer, k, v, seq, pos_start, stream=None):
    _check(lib().kvtc_encode_prefill(plan.handle, C.byref(cache.desc), layer, _dev_ptr(k), _dev_ptr(v), seq,
                                     pos_start, k.shape[0], _stream(stream)))


def kvtc_debug_encode_latent(plan, layer, head, kind, x, y_out, stream=None):
    """Test-only: fp32 latents [n, r] of rows x [n, d] of one unit (the append's order)."""
    _check(lib().kvtc_debug_encode_latent(plan.handle, layer, head, kind, _dev_ptr(x), _dtype_code(x), x.shape[0],
                                          _dev_ptr(y_out), _stream(stream)))


def kvtc_plan_prefill_stats(plan, reset=False):
    """(codes produced, codes recomputed in canonical order) by kvtc_encode_prefill."""
    a, b = C.c_uint64(), C.c_uint64()
    _check(lib().kvtc_plan_prefill_stats(plan.handle, C.byref(a), C.byref(b), int(reset)))
    return a.value, b.value


def kvtc_decode_workspace_bytes(plan, n_seq, max_seq_len):
    return int(lib().kvtc_decode_workspace_bytes(plan.handle, n_seq, max_seq_len))


def kvtc_decode_attention(plan, cache, layer, q, seq_lens, max_seq_len, out, workspace, scale=0.0,
                          stream=None):
    _check(lib().kvtc_decode_attention(plan.handle, C.byref(cache.desc), layer, _dev_ptr(q), _dtype_code(q),
                                       _dev_ptr(seq_lens), max_seq_len, scale, _dev_ptr(out), _dtype_code(out),
                                       _dev_ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream)))


def kvtc_decode_attention_noalloc(plan, cache, layer, q, seq_lens, max_seq_len, out, scale=0.0, stream=None):
    """Decode attention using the library's own fixed scratch array (no workspace
    argument), for callers that cannot allocate device memory."""
    _check(lib().kvtc_decode_attention_noalloc(plan.handle, C.byref(cache.desc), layer, _dev_ptr(q),
                                               _dtype_code(q), _dev_ptr(seq_lens), max_seq_len, scale,
                                               _dev_ptr(out), _dtype_code(out), _stream(stream)))


def kvtc_decode_attention_rope(plan, cache, layer, q, seq_lens, max_seq_len, out, workspace, scale=0.0,
                               rope_base=0.0, stream=None):
    """Decode attention for keys coded before the rotary embedding (q already rotated)."""
    _check(lib().kvtc_decode_attention_rope(plan.handle, C.byref(cache.desc), layer, _dev_ptr(q), _dtype_code(q),
                                            _dev_ptr(seq_lens), max_seq_len, scale, float(rope_base), _dev_ptr(out),
                                            _dtype_code(out), _dev_ptr(workspace),
                                            workspace.numel() * workspace.element_size(), _stream(stream)))
