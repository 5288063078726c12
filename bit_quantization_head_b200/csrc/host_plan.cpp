// Host side of libkvtc: errors, plan objects, accessors, save/load, device upload and
// cache sizing.  Calibration is in host_calibrate.cpp; kernels in *.cu.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <memory>
#include <string>

#include "kvtc_internal.h"

namespace kvtc {

static thread_local std::string g_error;

kvtc_status fail(kvtc_status s, const std::string& msg) {
  g_error = msg;
  return s;
}

kvtc_status cuda_fail(int err, const char* what) {
  g_error = std::string(what) + ": " + cudaGetErrorString(static_cast<cudaError_t>(err));
  return KVTC_ECUDA;
}

kvtc_status check_uploaded(const kvtc_plan* plan) {
  if (!plan) return fail(KVTC_EINVAL, "plan is NULL");
  if (!plan->d_units) return fail(KVTC_ESTATE, "plan not uploaded (call kvtc_plan_upload)");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != plan->device) return fail(KVTC_ESTATE, "plan uploaded to another device");
  return KVTC_OK;
}

static uint16_t bf16_bits(float x) {
  uint32_t u;
  std::memcpy(&u, &x, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
  uint32_t rounding = ((u >> 16) & 1u) + 0x7FFFu;
  return static_cast<uint16_t>((u + rounding) >> 16);
}

// fp16 bits of x, round to nearest even (subnormals kept, overflow to infinity).
static uint16_t fp16_bits(float x) {
  uint32_t u;
  std::memcpy(&u, &x, 4);
  const uint32_t sign = (u >> 16) & 0x8000u;
  const uint32_t ax = u & 0x7FFFFFFFu;
  if (ax >= 0x7F800000u) return static_cast<uint16_t>(sign | 0x7C00u | (ax > 0x7F800000u ? 0x200u : 0u));
  if (ax >= 0x477FF000u) return static_cast<uint16_t>(sign | 0x7C00u);  // rounds past 65504
  if (ax < 0x33000001u) return static_cast<uint16_t>(sign);              // below half the least subnormal
  int e = static_cast<int>(ax >> 23) - 127;
  uint32_t m = (ax & 0x7FFFFFu) | 0x800000u;                             // 24-bit significand
  // value = m * 2^(e - 23); fp16 keeps 11 bits for normals (e >= -14), fewer below
  const int shift = e >= -14 ? 13 : 13 + (-14 - e);
  const uint32_t q = m >> shift, rem = m & ((1u << shift) - 1u), half = 1u << (shift - 1);
  uint32_t r = q + ((rem > half || (rem == half && (q & 1u))) ? 1u : 0u);
  if (e >= -14) {
    // r holds 11 significant bits (or 2^11 after rounding up)
    uint32_t exp = static_cast<uint32_t>(e + 15);
    if (r == 0x800u) {
      r = 0x400u;
      ++exp;
    }
    if (exp >= 31) return static_cast<uint16_t>(sign | 0x7C00u);
    return static_cast<uint16_t>(sign | (exp << 10) | (r & 0x3FFu));
  }
  return static_cast<uint16_t>(sign | r);  // subnormal (r == 0x400 is the least normal)
}

static float fp16_value(uint16_t h) {
  const uint32_t sign = (h & 0x8000u) ? 1u : 0u;
  const int exp = (h >> 10) & 31;
  const int man = h & 0x3FF;
  float v = exp == 0 ? std::ldexp(static_cast<float>(man), -24) : std::ldexp(static_cast<float>(man | 0x400), exp - 25);
  return sign ? -v : v;
}

static void free_device(kvtc_plan* p) {
  if (p->d_units) cudaFree(p->d_units);
  if (p->d_M) cudaFree(p->d_M);
  if (p->d_Mbf) cudaFree(p->d_Mbf);
  if (p->d_Mfrag) cudaFree(p->d_Mfrag);
  if (p->d_Mrec) cudaFree(p->d_Mrec);
  if (p->d_stats) cudaFree(p->d_stats);
  p->d_stats = nullptr;
  p->d_units = nullptr;
  p->d_M = nullptr;
  p->d_Mbf = nullptr;
  p->d_Mfrag = nullptr;
  p->d_Mrec = nullptr;
  p->device = -1;
  p->h_units.clear();
  p->dec_groups.clear();
}

}  // namespace kvtc

using namespace kvtc;

extern "C" {

const char* kvtc_last_error(void) { return kvtc::g_error.c_str(); }

int kvtc_version(void) { return KVTC_VERSION; }

kvtc_status kvtc_plan_create(int n_layers, int n_kv_heads, int group, int head_dim, const int* r,
                             const int* b, const double* delta, const float* M, kvtc_plan** out) {
  if (!out || !r || !b || !delta || !M) return fail(KVTC_EINVAL, "null argument");
  *out = nullptr;
  if (n_layers < 1 || n_kv_heads < 1 || group < 1) return fail(KVTC_EINVAL, "bad model shape");
  if (head_dim != kD) return fail(KVTC_EINVAL, "head_dim must be 128");
  std::unique_ptr<kvtc_plan> p(new (std::nothrow) kvtc_plan());
  if (!p) return fail(KVTC_ENOMEM, "out of host memory");
  p->L = n_layers;
  p->H = n_kv_heads;
  p->G = group;
  p->d = head_dim;
  p->U = 2 * n_layers * n_kv_heads;
  size_t off = 0;
  for (int u = 0; u < p->U; ++u) {
    if (!valid_rb(r[u], b[u], u & 1))
      return fail(KVTC_EINVAL, "r must be even in [2,128] and b in [2,8] (or a raw value unit: r = 128, b = 16)");
    if (!(delta[u] > 0.0) || !std::isfinite(delta[u])) return fail(KVTC_EINVAL, "delta must be > 0");
    p->r.push_back(r[u]);
    p->b.push_back(b[u]);
    p->delta.push_back(delta[u]);
    p->inv_delta.push_back(static_cast<float>(1.0 / delta[u]));
    p->sigma.push_back(0.0);
    p->D.push_back(0.0);
    p->M.emplace_back(M + off, M + off + static_cast<size_t>(r[u]) * kD);
    off += static_cast<size_t>(r[u]) * kD;
  }
  *out = p.release();
  return KVTC_OK;
}

void kvtc_plan_destroy(kvtc_plan* plan) {
  if (!plan) return;
  free_device(plan);
  delete plan;
}

kvtc_status kvtc_plan_shape(const kvtc_plan* plan, int* n_layers, int* n_kv_heads, int* group,
                            int* head_dim, int* n_units) {
  if (!plan) return fail(KVTC_EINVAL, "plan is NULL");
  if (n_layers) *n_layers = plan->L;
  if (n_kv_heads) *n_kv_heads = plan->H;
  if (group) *group = plan->G;
  if (head_dim) *head_dim = plan->d;
  if (n_units) *n_units = plan->U;
  return KVTC_OK;
}

kvtc_status kvtc_plan_unit(const kvtc_plan* plan, int unit, kvtc_unit_info* out) {
  if (!plan || !out) return fail(KVTC_EINVAL, "null argument");
  if (unit < 0 || unit >= plan->U) return fail(KVTC_EINVAL, "unit out of range");
  out->kind = unit & 1;
  out->head = (unit >> 1) % plan->H;
  out->layer = (unit >> 1) / plan->H;
  out->r = plan->r[unit];
  out->b = plan->b[unit];
  out->delta = plan->delta[unit];
  out->inv_delta = plan->inv_delta[unit];
  out->sigma = plan->sigma[unit];
  out->distortion = plan->D[unit];
  out->page_bytes = 16ull * plan->r[unit] * plan->b[unit];
  return KVTC_OK;
}

kvtc_status kvtc_plan_matrix(const kvtc_plan* plan, int unit, float* M_out) {
  if (!plan || !M_out) return fail(KVTC_EINVAL, "null argument");
  if (unit < 0 || unit >= plan->U) return fail(KVTC_EINVAL, "unit out of range");
  std::memcpy(M_out, plan->M[unit].data(), plan->M[unit].size() * sizeof(float));
  return KVTC_OK;
}

kvtc_status kvtc_plan_weights(const kvtc_plan* plan, int unit, double* w_out, double* lam_out) {
  if (!plan) return fail(KVTC_EINVAL, "plan is NULL");
  if (unit < 0 || unit >= plan->U) return fail(KVTC_EINVAL, "unit out of range");
  if (plan->w.empty()) return fail(KVTC_EINVAL, "plan has no calibration weights");
  if (w_out) std::memcpy(w_out, plan->w[unit].data(), plan->d * sizeof(double));
  if (lam_out) std::memcpy(lam_out, plan->lam[unit].data(), plan->d * sizeof(double));
  return KVTC_OK;
}

kvtc_status kvtc_plan_budget(const kvtc_plan* plan, double* mu, uint64_t* total_bits) {
  if (!plan) return fail(KVTC_EINVAL, "plan is NULL");
  if (mu) *mu = plan->mu;
  if (total_bits) {
    uint64_t t = 0;
    for (int u = 0; u < plan->U; ++u) t += static_cast<uint64_t>(plan->r[u]) * plan->b[u];
    *total_bits = t;
  }
  return KVTC_OK;
}

extern "C" kvtc_status kvtc_plan_calib_seconds(const kvtc_plan* plan, double* stats_s, double* alloc_s) {
  if (!plan) return fail(KVTC_EINVAL, "plan is NULL");
  if (stats_s) *stats_s = plan->t_stats;
  if (alloc_s) *alloc_s = plan->t_alloc;
  return KVTC_OK;
}

// File format (little-endian): "KVTCPLAN", u32 version, i32 L, H, G, d, U, f64 mu,
// u32 has_weights; per unit: i32 r, i32 b, f64 delta, f32 inv_delta, f64 sigma, f64 D,
// f32 M[r*d], then (if has_weights) f64 w[d], f64 lam[d].
kvtc_status kvtc_plan_save(const kvtc_plan* plan, const char* path) {
  if (!plan || !path) return fail(KVTC_EINVAL, "null argument");
  FILE* f = std::fopen(path, "wb");
  if (!f) return fail(KVTC_EIO, std::string("cannot open ") + path);
  bool ok = true;
  auto put = [&](const void* p, size_t n) { ok = ok && std::fwrite(p, 1, n, f) == n; };
  const char magic[8] = {'K', 'V', 'T', 'C', 'P', 'L', 'A', 'N'};
  uint32_t ver = KVTC_VERSION;
  uint32_t hw = plan->w.empty() ? 0u : 1u;
  put(magic, 8);
  put(&ver, 4);
  put(&plan->L, 4);
  put(&plan->H, 4);
  put(&plan->G, 4);
  put(&plan->d, 4);
  put(&plan->U, 4);
  put(&plan->mu, 8);
  put(&hw, 4);
  for (int u = 0; u < plan->U; ++u) {
    put(&plan->r[u], 4);
    put(&plan->b[u], 4);
    put(&plan->delta[u], 8);
    put(&plan->inv_delta[u], 4);
    put(&plan->sigma[u], 8);
    put(&plan->D[u], 8);
    put(plan->M[u].data(), plan->M[u].size() * 4);
    if (hw) {
      put(plan->w[u].data(), plan->d * 8);
      put(plan->lam[u].data(), plan->d * 8);
    }
  }
  ok = (std::fclose(f) == 0) && ok;
  return ok ? KVTC_OK : fail(KVTC_EIO, std::string("write failed: ") + path);
}

kvtc_status kvtc_plan_load(const char* path, kvtc_plan** out) {
  if (!path || !out) return fail(KVTC_EINVAL, "null argument");
  *out = nullptr;
  FILE* f = std::fopen(path, "rb");
  if (!f) return fail(KVTC_EIO, std::string("cannot open ") + path);
  std::unique_ptr<FILE, int (*)(FILE*)> guard(f, std::fclose);
  bool ok = true;
  auto get = [&](void* p, size_t n) { ok = ok && std::fread(p, 1, n, f) == n; };
  char magic[8];
  uint32_t ver = 0, hw = 0;
  std::unique_ptr<kvtc_plan> p(new (std::nothrow) kvtc_plan());
  if (!p) return fail(KVTC_ENOMEM, "out of host memory");
  get(magic, 8);
  if (!ok || std::memcmp(magic, "KVTCPLAN", 8) != 0) return fail(KVTC_EIO, "not a plan file");
  get(&ver, 4);
  if (!ok) return fail(KVTC_EIO, "truncated plan file");
  if (ver != KVTC_VERSION) return fail(KVTC_EVERSION, "plan file version mismatch");
  get(&p->L, 4);
  get(&p->H, 4);
  get(&p->G, 4);
  get(&p->d, 4);
  get(&p->U, 4);
  get(&p->mu, 8);
  get(&hw, 4);
  if (!ok || p->d != kD || p->L < 1 || p->H < 1 || p->G < 1 || p->U != 2 * p->L * p->H)
    return fail(KVTC_EIO, "corrupt plan header");
  for (int u = 0; u < p->U && ok; ++u) {
    int r = 0, b = 0;
    double delta = 0, sigma = 0, D = 0;
    float inv = 0;
    get(&r, 4);
    get(&b, 4);
    get(&delta, 8);
    get(&inv, 4);
    get(&sigma, 8);
    get(&D, 8);
    if (!ok || !valid_rb(r, b, static_cast<int>(p->r.size()) & 1)) return fail(KVTC_EIO, "corrupt unit");
    p->r.push_back(r);
    p->b.push_back(b);
    p->delta.push_back(delta);
    p->inv_delta.push_back(inv);
    p->sigma.push_back(sigma);
    p->D.push_back(D);
    p->M.emplace_back(static_cast<size_t>(r) * kD);
    get(p->M.back().data(), static_cast<size_t>(r) * kD * 4);
    if (hw) {
      p->w.emplace_back(kD);
      p->lam.emplace_back(kD);
      get(p->w.back().data(), kD * 8);
      get(p->lam.back().data(), kD * 8);
    }
  }
  if (!ok) return fail(KVTC_EIO, "truncated plan file");
  *out = p.release();
  return KVTC_OK;
}

kvtc_status kvtc_plan_upload(kvtc_plan* plan, void* stream) {
  if (!plan) return fail(KVTC_EINVAL, "plan is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  free_device(plan);
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  size_t total = 0;
  for (int u = 0; u < plan->U; ++u) total += plan->M[u].size();
  std::vector<float> hM;
  std::vector<uint16_t> hMbf;
  hM.reserve(total);
  hMbf.reserve(total);
  for (int u = 0; u < plan->U; ++u)
    for (float x : plan->M[u]) {
      hM.push_back(x);
      hMbf.push_back(bf16_bits(x));
    }
  // fp16 hi/lo A fragments of every M (m16n8k16 layout: lane (g, t) holds rows g, g + 8
  // and columns 2t, 2t + 1, 2t + 8, 2t + 9 of a 16 x 16 tile)
  std::vector<uint32_t> hFrag;
  std::vector<size_t> frag_off(plan->U);
  for (int u = 0; u < plan->U; ++u) {
    frag_off[u] = hFrag.size();
    const int r = plan->r[u], nmt = (r + 15) / 16;
    const std::vector<float>& Mu = plan->M[u];
    auto part = [&](int row, int col, int p) -> uint32_t {
      if (row >= r) return 0u;
      const float x = Mu[static_cast<size_t>(row) * kD + col];
      const uint16_t hi = fp16_bits(x);
      return p == 0 ? hi : fp16_bits(x - fp16_value(hi));
    };
    for (int mt = 0; mt < nmt; ++mt)
      for (int ks = 0; ks < 8; ++ks)
        for (int p = 0; p < 2; ++p)
          for (int lane = 0; lane < 32; ++lane) {
            const int g = lane >> 2, t = lane & 3;
            const int r0 = 16 * mt + g, c0 = 16 * ks + 2 * t;
            const int rows[4] = {r0, r0 + 8, r0, r0 + 8};
            const int cols[4] = {c0, c0, c0 + 8, c0 + 8};
            for (int i = 0; i < 4; ++i)
              hFrag.push_back(part(rows[i], cols[i], p) | (part(rows[i], cols[i] + 1, p) << 16));
          }
  }
  // key units: M^T in B-fragment order for the reconstruction K-hat = C M (lane (g, t) of
  // n-tile nt, k-step ks: b0 = M[16ks + 2t .. + 1][8nt + g], b1 = M[16ks + 8 + 2t .. + 1][8nt + g]),
  // hi and lo parts, followed by the fp32 column sums of M
  std::vector<uint32_t> hRec;
  std::vector<size_t> rec_off(plan->U, 0);
  for (int u = 0; u < plan->U; u += 2) {
    rec_off[u] = hRec.size();
    const int r = plan->r[u], nks = (r + 15) / 16;
    const std::vector<float>& Mu = plan->M[u];
    auto el = [&](int row, int col, int p) -> uint32_t {
      if (row >= r) return 0u;
      const float x = Mu[static_cast<size_t>(row) * kD + col];
      const uint16_t hi = fp16_bits(x);
      return p == 0 ? hi : fp16_bits(x - fp16_value(hi));
    };
    for (int ks = 0; ks < nks; ++ks)
      for (int nt = 0; nt < 16; ++nt)
        for (int lane = 0; lane < 32; ++lane) {
          const int g = lane >> 2, t = lane & 3;
          const int col = 8 * nt + g, r0 = 16 * ks + 2 * t;
          for (int p = 0; p < 2; ++p) {
            hRec.push_back(el(r0, col, p) | (el(r0 + 1, col, p) << 16));
            hRec.push_back(el(r0 + 8, col, p) | (el(r0 + 9, col, p) << 16));
          }
        }
    for (int col = 0; col < kD; ++col) {
      double cs = 0.0;
      for (int row = 0; row < r; ++row) cs += Mu[static_cast<size_t>(row) * kD + col];
      const float f = static_cast<float>(cs);
      uint32_t bits;
      std::memcpy(&bits, &f, 4);
      hRec.push_back(bits);
    }
  }
  if ((e = cudaMalloc(&plan->d_M, total * sizeof(float))) != cudaSuccess ||
      (e = cudaMalloc(&plan->d_Mrec, std::max<size_t>(1, hRec.size()) * sizeof(uint32_t))) != cudaSuccess ||
      (e = cudaMalloc(&plan->d_Mbf, total * sizeof(uint16_t))) != cudaSuccess ||
      (e = cudaMalloc(&plan->d_Mfrag, std::max<size_t>(1, hFrag.size()) * sizeof(uint32_t))) != cudaSuccess ||
      (e = cudaMalloc(&plan->d_units, plan->U * sizeof(UnitDesc))) != cudaSuccess ||
      (e = cudaMalloc(&plan->d_stats, 2 * sizeof(uint64_t))) != cudaSuccess ||
      (e = cudaMemsetAsync(plan->d_stats, 0, 2 * sizeof(uint64_t), st)) != cudaSuccess) {
    free_device(plan);
    return cuda_fail(e, "cudaMalloc (plan upload)");
  }
  plan->h_units.resize(plan->U);
  size_t off = 0;
  uint64_t prefix = 0;
  for (int u = 0; u < plan->U; ++u) {
    UnitDesc& ud = plan->h_units[u];
    ud.r = plan->r[u];
    ud.b = plan->b[u];
    ud.delta = static_cast<float>(plan->delta[u]);
    ud.inv_delta = plan->inv_delta[u];
    ud.page_bytes = 16ull * ud.r * ud.b;
    ud.prefix = prefix;
    ud.M = plan->d_M + off;
    ud.Mbf = plan->d_Mbf + off;
    ud.Mfrag = plan->d_Mfrag + frag_off[u];
    if (u % 2 == 0) {
      ud.Mrec = plan->d_Mrec + rec_off[u];
      ud.Msum = reinterpret_cast<const float*>(plan->d_Mrec + rec_off[u] + static_cast<size_t>((ud.r + 15) / 16) * 16 * 32 * 4);
    } else {
      ud.Mrec = nullptr;
      ud.Msum = nullptr;
    }
    double mn = 0.0;
    for (int i = 0; i < ud.r; ++i) {
      double ss = 0.0;
      for (int k = 0; k < kD; ++k) {
        const uint32_t bits = static_cast<uint32_t>(hMbf[off + static_cast<size_t>(i) * kD + k]) << 16;
        float x;
        std::memcpy(&x, &bits, 4);
        ss += static_cast<double>(x) * x;
      }
      mn = std::max(mn, std::sqrt(ss));
    }
    ud.mnorm = static_cast<float>(mn * (1.0 + 1e-6));
    prefix += ud.page_bytes;
    off += plan->M[u].size();
  }
  if ((e = cudaMemcpyAsync(plan->d_M, hM.data(), total * sizeof(float), cudaMemcpyHostToDevice, st)) !=
          cudaSuccess ||
      (e = cudaMemcpyAsync(plan->d_Mbf, hMbf.data(), total * sizeof(uint16_t), cudaMemcpyHostToDevice,
                           st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(plan->d_Mfrag, hFrag.data(), hFrag.size() * sizeof(uint32_t), cudaMemcpyHostToDevice,
                           st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(plan->d_Mrec, hRec.data(), hRec.size() * sizeof(uint32_t), cudaMemcpyHostToDevice,
                           st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(plan->d_units, plan->h_units.data(), plan->U * sizeof(UnitDesc),
                           cudaMemcpyHostToDevice, st)) != cudaSuccess ||
      (e = cudaStreamSynchronize(st)) != cudaSuccess) {
    free_device(plan);
    return cuda_fail(e, "plan upload copy");
  }
  plan->device = dev;
  kvtc_status ds = prepare_decode(plan);
  if (ds == KVTC_OK) ds = prepare_rope(plan);
  if (ds != KVTC_OK) {
    free_device(plan);
    return ds;
  }
  return KVTC_OK;
}

uint64_t kvtc_cache_bytes(const kvtc_plan* plan, uint64_t pages_per_unit) {
  if (!plan) return 0;
  uint64_t t = 0;
  for (int u = 0; u < plan->U; ++u) t += 16ull * plan->r[u] * plan->b[u];
  return t * pages_per_unit;
}

uint64_t kvtc_unit_pool_offset(const kvtc_plan* plan, int unit, uint64_t pages_per_unit) {
  if (!plan || unit < 0 || unit > plan->U) return 0;
  uint64_t t = 0;
  for (int u = 0; u < unit; ++u) t += 16ull * plan->r[u] * plan->b[u];
  return t * pages_per_unit;
}

}  // extern "C"
