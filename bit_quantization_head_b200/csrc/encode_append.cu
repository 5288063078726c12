// kvtc_encode_append: canonical-order per-token encode on CUDA cores.
//
// KV-COBRA project page, "How KV-COBRA Works" (Inference): each key (and value) is
// rotated and truncated with H.V^T and quantized with the unit's b-bit quantizer.  One
// thread computes one latent coordinate y_j of one token of one unit in the canonical
// fp32 order (eight fma chains over k mod 8, then a fixed pairwise sum: the arithmetic
// the oracle reproduces bit for bit), quantizes it and merges its bits into the page
// word.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kvtc_internal.h"
#include "layout.cuh"
#include "ptx.cuh"

namespace kvtc {

struct AppendArgs {
  const UnitDesc* units;  // device, all units of the plan
  int unit0;              // first unit of the layer
  int n_units;            // units in the layer (2 * H)
  int H;
  const void* k;
  const void* v;
  int bf16;
  const int32_t* cu_seqlens;
  const int32_t* pos_start;
  int n_seq;
  int n_tok;
  char* pool;
  uint64_t pages_per_unit;
  const int32_t* block_table;
  int max_pages;
  int32_t* status;
};

__device__ __forceinline__ uint8_t quantize_code(float y, float inv_delta, int b) {
  const float t = __fmul_rn(y, inv_delta);
  const float u = __fadd_rn(t, static_cast<float>(1 << (b - 1)));
  float f = floorf(u);
  f = fmaxf(f, 0.0f);                                   // NaN -> 0
  f = fminf(f, static_cast<float>((1 << b) - 1));
  return static_cast<uint8_t>(f);
}

// Overwrites the b-bit code (t, j) of a page: clears its bits, then sets them.
__device__ __forceinline__ void store_code(uint32_t* page, int kind, int r, int b, int t, int j, uint32_t c) {
  const int np = code_nparts(b);
  for (int i = 0; i < np; ++i) {
    int lo, w;
    code_part(b, i, lo, w);
    const FieldPos f = field_pos(kind, r, lo, w, t, j);
    const uint32_t mask = ((1u << w) - 1u) << f.bit;
    const uint32_t bits = ((c >> lo) & ((1u << w) - 1u)) << f.bit;
    atomicAnd(page + f.word, ~mask);
    if (bits) atomicOr(page + f.word, bits);
  }
}

// CTA = (token, unit of the layer); thread j computes coordinate j.  The token's row is
// staged in shared memory once; each thread holds its row of M in registers; the fma
// chains then run in the canonical order from registers and broadcast reads.
__global__ void __launch_bounds__(128) encode_append_kernel(const __grid_constant__ AppendArgs a) {
  __shared__ float xs[kD];
  __shared__ int s_seq;
  __shared__ long long s_pos;
  const int tok = blockIdx.x, ul = blockIdx.y, j = threadIdx.x;
  const int u = a.unit0 + ul;
  // The plan (unit descriptor, bf16 row of M) is constant: read it before waiting for
  // the producer of k/v (programmatic dependent launch), so the loads overlap its tail.
  const UnitDesc ud = a.units[u];
  uint4 mr[16];
  const bool raw = ud.b == kRawBits;  // uncompressed value unit (keys-only plans)
  if (a.bf16 && j < ud.r && !raw) {
    const uint4* m4 = reinterpret_cast<const uint4*>(ud.Mbf + static_cast<size_t>(j) * kD);
#pragma unroll
    for (int c = 0; c < 16; ++c) mr[c] = m4[c];
  }
  griddep_wait();
  // let the next kernel (typically the decode of this layer) start its prologue
  griddep_launch_dependents();
  const int kind = ul & 1;
  const int head = ul >> 1;
  const size_t xoff = (static_cast<size_t>(tok) * a.H + head) * kD;
  // The inputs go out together: the token's row element, and its sequence and position
  // (thread i tests whether the token lies in [cu_seqlens[i], cu_seqlens[i + 1]), so one
  // round of loads finds it; more sequences than threads take a binary search).
  const float xv = a.bf16 ? __bfloat162float((static_cast<const __nv_bfloat16*>(kind ? a.v : a.k) + xoff)[j])
                          : (static_cast<const float*>(kind ? a.v : a.k) + xoff)[j];
  if (j == 0) {  // (a token no interval holds is reported as a bad position)
    s_seq = 0;
    s_pos = -1;
  }
  __syncthreads();
  if (a.n_seq <= static_cast<int>(blockDim.x)) {
    if (j < a.n_seq) {
      const int c0 = a.cu_seqlens[j], c1 = a.cu_seqlens[j + 1];
      const int ps = a.pos_start[j];
      if (c0 <= tok && tok < c1) {
        s_seq = j;
        s_pos = static_cast<long long>(ps) + (tok - c0);
      }
    }
  } else if (j == 0) {
    int lo = 0, hi = a.n_seq - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.cu_seqlens[mid] <= tok)
        lo = mid;
      else
        hi = mid - 1;
    }
    s_seq = lo;
    s_pos = static_cast<long long>(a.pos_start[lo]) + (tok - a.cu_seqlens[lo]);
  }
  xs[j] = xv;
  __syncthreads();
  if (j >= ud.r) return;
  // token -> page: the block-table entry is loaded before the arithmetic below
  const int s = s_seq;
  const long long pos = s_pos;
  const bool pos_ok = pos >= 0 && pos < static_cast<long long>(a.max_pages) * kPage;
  const int lp = pos_ok ? static_cast<int>(pos / kPage) : 0;
  const int slot = pos_ok ? static_cast<int>(pos % kPage) : 0;
  const int32_t pid = pos_ok ? a.block_table[static_cast<size_t>(s) * a.max_pages + lp] : -1;

  uint32_t code = 0;
  if (raw) {
    code = __half_as_ushort(__float2half_rn(xs[j]));
  } else {
    // canonical projection: eight chains a_e = fma(x_k, M_jk, a_e) over k = e (mod 8)
    // ascending, then ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7))
    float ch[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    if (a.bf16) {
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t w[4] = {mr[c].x, mr[c].y, mr[c].z, mr[c].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          ch[2 * q] = __fmaf_rn(xs[8 * c + 2 * q], __uint_as_float(w[q] << 16), ch[2 * q]);
          ch[2 * q + 1] = __fmaf_rn(xs[8 * c + 2 * q + 1], __uint_as_float(w[q] & 0xFFFF0000u), ch[2 * q + 1]);
        }
      }
    } else {
      const float4* m4 = reinterpret_cast<const float4*>(ud.M + static_cast<size_t>(j) * kD);
#pragma unroll 4
      for (int c = 0; c < 16; ++c) {
        const float4 m0 = m4[2 * c], m1 = m4[2 * c + 1];
        ch[0] = __fmaf_rn(xs[8 * c], m0.x, ch[0]);
        ch[1] = __fmaf_rn(xs[8 * c + 1], m0.y, ch[1]);
        ch[2] = __fmaf_rn(xs[8 * c + 2], m0.z, ch[2]);
        ch[3] = __fmaf_rn(xs[8 * c + 3], m0.w, ch[3]);
        ch[4] = __fmaf_rn(xs[8 * c + 4], m1.x, ch[4]);
        ch[5] = __fmaf_rn(xs[8 * c + 5], m1.y, ch[5]);
        ch[6] = __fmaf_rn(xs[8 * c + 6], m1.z, ch[6]);
        ch[7] = __fmaf_rn(xs[8 * c + 7], m1.w, ch[7]);
      }
    }
    const float acc = __fadd_rn(__fadd_rn(__fadd_rn(ch[0], ch[1]), __fadd_rn(ch[2], ch[3])),
                                __fadd_rn(__fadd_rn(ch[4], ch[5]), __fadd_rn(ch[6], ch[7])));
    code = quantize_code(acc, ud.inv_delta, ud.b);
  }

  if (!pos_ok) {
    if (a.status) atomicOr(a.status, KVTC_STATUS_BAD_POS);
    return;
  }
  if (pid < 0 || static_cast<uint64_t>(pid) >= a.pages_per_unit) {
    if (a.status) atomicOr(a.status, KVTC_STATUS_BAD_PAGE);
    return;
  }
  uint32_t* page = reinterpret_cast<uint32_t*>(a.pool + a.pages_per_unit * ud.prefix +
                                               static_cast<uint64_t>(pid) * ud.page_bytes);
  if (raw) {
    // raw page: row j of 64 words, token pair slot / 2 at position (slot / 2) XOR 4 (j % 8),
    // the even token in the low half
    const int word = j * (kPage / 2) + ((slot >> 1) ^ ((j & 7) << 2));
    reinterpret_cast<uint16_t*>(page)[2 * word + (slot & 1)] = static_cast<uint16_t>(code);
    return;
  }
  store_code(page, kind, ud.r, ud.b, slot, j, code);
}

// Test-only: the fp32 latent y = M x of rows of one unit in the same canonical order as
// encode_append_kernel (CTA = token, thread j = coordinate), written instead of codes.
// Raw value units (keys-only plans) have no projection: y = x.
__global__ void __launch_bounds__(128) debug_latent_kernel(const UnitDesc* units, int u, const void* x, int bf16,
                                                            float* y) {
  __shared__ float xs[kD];
  const int tok = blockIdx.x, j = threadIdx.x;
  const UnitDesc ud = units[u];
  const size_t xoff = static_cast<size_t>(tok) * kD;
  xs[j] = bf16 ? __bfloat162float((static_cast<const __nv_bfloat16*>(x) + xoff)[j])
               : (static_cast<const float*>(x) + xoff)[j];
  __syncthreads();
  if (j >= ud.r) return;
  float out;
  if (ud.b == kRawBits) {
    out = xs[j];
  } else {
    float ch[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    if (bf16) {
      const uint4* m4 = reinterpret_cast<const uint4*>(ud.Mbf + static_cast<size_t>(j) * kD);
      for (int c = 0; c < 16; ++c) {
        const uint4 mr = m4[c];
        const uint32_t w[4] = {mr.x, mr.y, mr.z, mr.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          ch[2 * q] = __fmaf_rn(xs[8 * c + 2 * q], __uint_as_float(w[q] << 16), ch[2 * q]);
          ch[2 * q + 1] = __fmaf_rn(xs[8 * c + 2 * q + 1], __uint_as_float(w[q] & 0xFFFF0000u), ch[2 * q + 1]);
        }
      }
    } else {
      const float* m = ud.M + static_cast<size_t>(j) * kD;
      for (int k = 0; k < kD; ++k) ch[k & 7] = __fmaf_rn(xs[k], m[k], ch[k & 7]);
    }
    out = __fadd_rn(__fadd_rn(__fadd_rn(ch[0], ch[1]), __fadd_rn(ch[2], ch[3])),
                    __fadd_rn(__fadd_rn(ch[4], ch[5]), __fadd_rn(ch[6], ch[7])));
  }
  y[static_cast<size_t>(tok) * ud.r + j] = out;
}

}  // namespace kvtc

using namespace kvtc;

extern "C" kvtc_status kvtc_debug_encode_latent(const kvtc_plan* plan, int layer, int head, int kind, const void* x,
                                                kvtc_dtype dtype, int n_tok, float* y_out, void* stream) {
  kvtc_status st = check_uploaded(plan);
  if (st != KVTC_OK) return st;
  if (layer < 0 || layer >= plan->L || head < 0 || head >= plan->H || (kind != 0 && kind != 1))
    return fail(KVTC_EINVAL, "layer, head or kind out of range");
  if (dtype != KVTC_F32 && dtype != KVTC_BF16) return fail(KVTC_EINVAL, "dtype must be F32 or BF16");
  if (n_tok < 0) return fail(KVTC_EINVAL, "n_tok must be >= 0");
  if (n_tok == 0) return KVTC_OK;
  if (!x || !y_out) return fail(KVTC_EINVAL, "null device pointer");
  if (reinterpret_cast<uintptr_t>(x) & 15) return fail(KVTC_EINVAL, "x must be 16-byte aligned");
  const int u = (layer * plan->H + head) * 2 + kind;
  debug_latent_kernel<<<n_tok, 128, 0, static_cast<cudaStream_t>(stream)>>>(plan->d_units, u, x,
                                                                            dtype == KVTC_BF16 ? 1 : 0, y_out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "debug latent launch");
  return KVTC_OK;
}

extern "C" kvtc_status kvtc_encode_append(const kvtc_plan* plan, const kvtc_cache* cache, int layer,
                                          const void* k, const void* v, kvtc_dtype dtype,
                                          const int32_t* cu_seqlens, const int32_t* pos_start, int n_tok,
                                          void* stream) {
  kvtc_status st = check_uploaded(plan);
  if (st != KVTC_OK) return st;
  if (!cache || !cache->pool || !cache->block_table) return fail(KVTC_EINVAL, "cache is incomplete");
  if (layer < 0 || layer >= plan->L) return fail(KVTC_EINVAL, "layer out of range");
  if (dtype != KVTC_F32 && dtype != KVTC_BF16) return fail(KVTC_EINVAL, "dtype must be F32 or BF16");
  if (n_tok < 0 || cache->n_seq < 1 || cache->max_pages < 1) return fail(KVTC_EINVAL, "bad sizes");
  if (n_tok == 0) return KVTC_OK;
  if (!k || !v || !cu_seqlens || !pos_start) return fail(KVTC_EINVAL, "null device pointer");
  if (reinterpret_cast<uintptr_t>(cache->pool) & 15) return fail(KVTC_EINVAL, "pool must be 16-byte aligned");
  AppendArgs a;
  a.units = plan->d_units;
  a.unit0 = layer * plan->H * 2;
  a.n_units = plan->H * 2;
  a.H = plan->H;
  a.k = k;
  a.v = v;
  a.bf16 = dtype == KVTC_BF16;
  a.cu_seqlens = cu_seqlens;
  a.pos_start = pos_start;
  a.n_seq = cache->n_seq;
  a.n_tok = n_tok;
  a.pool = static_cast<char*>(cache->pool);
  a.pages_per_unit = cache->pages_per_unit;
  a.block_table = cache->block_table;
  a.max_pages = cache->max_pages;
  a.status = cache->status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n_tok), static_cast<unsigned>(a.n_units));
  cfg.blockDim = dim3(128);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, encode_append_kernel, a);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "encode_append launch");
  return KVTC_OK;
}
