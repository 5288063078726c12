// kvtc_encode_prefill: the per-token projection of a page-aligned span as tensor-core
// GEMM tiles (tcgen05, TMEM accumulator), with the quantize + pack epilogue.
//
// KV-COBRA project page, "How KV-COBRA Works" (Inference: rotate and truncate with
// H.V^T, quantize with the unit's b-bit quantizer) and "Efficiency" (packed b-bit codes).
//
// One CTA = one 128-token tile (one page) x one unit.  X [128 tok x 128] and M_bf16
// [r x 128] are staged in shared memory in the no-swizzle K-major core-matrix layout
// (8 rows x 16 bytes per core matrix), a single thread issues eight
// tcgen05.mma.kind::f16 (M = 128, N = r rounded up to 16, K = 16 each) into a TMEM
// accumulator, and tcgen05.commit signals an mbarrier.  Each thread then owns one token
// (one TMEM lane) and quantizes its r latents.
//
// Bit-exactness with the canonical chain: the tensor core sums the same exact bf16
// products in another order.  |y_tc - y_canonical| <= beta = 2^-14 * ||x||_2 * ||M_j||_2
// (both sums are within 127 * 2^-24 * sum_k |x_k M_jk| of the exact value for the
// canonical chain, and within 256 * 2^-23 of it for any fp32 accumulation order that
// errs by at most one ulp per operation; Cauchy-Schwarz bounds the sum of |products|).
// The quantizer is monotone, so when Q(y_tc - beta) == Q(y_tc + beta) (endpoints rounded
// outward) that code is the canonical code; otherwise the thread recomputes y with the
// canonical fp32 fma chain (k = 0..127 in order), exactly as kvtc_encode_append does.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kvtc_internal.h"
#include "layout.cuh"
#include "ptx.cuh"

namespace kvtc {
namespace {

constexpr int kThreads = 128;
constexpr uint32_t kRowGroupBytes = 2048;  // 16 core matrices (128 K-elements) per 8 rows
constexpr uint32_t kCoreBytes = 128;

struct PrefillArgs {
  const UnitDesc* units;
  int unit0, H;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  int seq, pos_start, n_tok;
  char* pool;
  uint64_t pages_per_unit;
  const int32_t* block_table;
  int max_pages;
  int32_t* status;
  uint64_t* stats;  // [0] codes produced, [1] codes recomputed in canonical order
};

// Byte offset of element (row, col) (bf16) in the core-matrix layout.
__device__ __forceinline__ uint32_t core_off(int row, int col) {
  return (row >> 3) * kRowGroupBytes + (col >> 3) * kCoreBytes + (row & 7) * 16 + (col & 7) * 2;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// SM100 shared-memory matrix descriptor, no swizzle, K-major: LBO = stride between core
// matrices along K, SBO = stride between 8-row groups; version field = 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

__device__ __forceinline__ uint8_t quant(float y, float inv_delta, int b) {
  const float t = __fmul_rn(y, inv_delta);
  const float u = __fadd_rn(t, static_cast<float>(1 << (b - 1)));
  float f = floorf(u);
  f = fmaxf(f, 0.0f);
  f = fminf(f, static_cast<float>((1 << b) - 1));
  return static_cast<uint8_t>(f);
}

__global__ void __launch_bounds__(kThreads) prefill_kernel(const PrefillArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* sA = smem;                    // 32 KB: X tile
  unsigned char* sB = smem + 32768;            // up to 32 KB: M (bf16)
  unsigned char* sC = smem + 65536;            // 128 x r code bytes
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 65536 + 16384);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 65536 + 16384 + 8);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int tile = blockIdx.x, ul = blockIdx.y;
  const int u = a.unit0 + ul, kind = ul & 1, head = ul >> 1;
  const UnitDesc ud = a.units[u];
  const int r = ud.r, b = ud.b;
  const int rpad = (r + 15) & ~15;
  const int t0 = tile * kPage;
  const int n_valid = min(kPage, a.n_tok - t0);
  const __nv_bfloat16* X = (kind ? a.v : a.k) + static_cast<size_t>(head) * kD;
  const size_t row_stride = static_cast<size_t>(a.H) * kD;

  // ---- stage X and M in shared memory (rows beyond the span / beyond r are zero) ----
  const uint32_t sA_u = smem_u32(sA), sB_u = smem_u32(sB);
  for (int i = tid; i < kPage * 16; i += kThreads) {
    const int row = i >> 4, ch = i & 15;
    const bool ok = row < n_valid;
    const __nv_bfloat16* src = X + (static_cast<size_t>(ok ? t0 + row : t0)) * row_stride + ch * 8;
    cp_async16(sA_u + core_off(row, ch * 8), src, ok);
  }
  for (int i = tid; i < rpad * 16; i += kThreads) {
    const int row = i >> 4, ch = i & 15;
    const bool ok = row < r;
    const uint16_t* src = ud.Mbf + static_cast<size_t>(ok ? row : 0) * kD + ch * 8;
    cp_async16(sB_u + core_off(row, ch * 8), src, ok);
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;\n" ::"r"(smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  cp_async_wait_all();
  fence_proxy_async_smem();
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  // ---- Y = X * M^T on the tensor cores ----
  if (tid == 0) {
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(rpad >> 3) << 17) |
                           (static_cast<uint32_t>(128 >> 4) << 24);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t da = umma_desc(sA_u + kk * 2 * kCoreBytes, kCoreBytes, kRowGroupBytes);
      const uint64_t db = umma_desc(sB_u + kk * 2 * kCoreBytes, kCoreBytes, kRowGroupBytes);
      const uint32_t acc = kk > 0 ? 1u : 0u;
      asm volatile(
          "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
          " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
          "l"(da), "l"(db), "r"(idesc), "r"(acc)
          : "memory");
    }
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
                 : "memory");
  }

  // While the MMA runs: this thread's token norm ||x||_2 (for the error bound).
  const int tok = tid;
  float nx = 0.0f;
#pragma unroll 4
  for (int ch = 0; ch < 16; ++ch) {
    const uint4 xv = *reinterpret_cast<const uint4*>(sA + core_off(tok, ch * 8));
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float x0 = __uint_as_float(xw[q] << 16), x1 = __uint_as_float(xw[q] & 0xFFFF0000u);
      nx = fmaf(x1, x1, fmaf(x0, x0, nx));
    }
  }
  const float beta = ldexpf(sqrtf(nx) * 1.001f, -14) * ud.mnorm;

  bool ok = mbar_wait_bounded_warp(bar, 0);
  if (!ok && (tid & 31) == 0 && a.status) atomicOr(a.status, KVTC_STATUS_TIMEOUT);
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");

  // ---- epilogue: TMEM lane = token; quantize r latents ----
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  uint32_t n_fix = 0;
  for (int c0 = 0; c0 < rpad; c0 += 16) {
    uint32_t v[16];
    __syncwarp();  // tcgen05.ld is .sync.aligned: reconverge after the fixup branches
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(lane_addr + c0));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int j = c0 + i;
      if (j < r) {
        const float y = __uint_as_float(v[i]);
        const uint8_t qlo = quant(__fsub_rd(y, beta), ud.inv_delta, b);
        const uint8_t qhi = quant(__fadd_ru(y, beta), ud.inv_delta, b);
        uint8_t code = qlo;
        if (qlo != qhi || !ok) {
          // canonical chain (the arithmetic of kvtc_encode_append)
          float acc = 0.0f;
          for (int ch = 0; ch < 16; ++ch) {
            const uint4 xv = *reinterpret_cast<const uint4*>(sA + core_off(tok, ch * 8));
            const uint4 mv = *reinterpret_cast<const uint4*>(sB + core_off(j, ch * 8));
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, mw[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // k = 8ch + 2q, then 8ch + 2q + 1: ascending
              acc = __fmaf_rn(__uint_as_float(xw[q] << 16), __uint_as_float(mw[q] << 16), acc);
              acc = __fmaf_rn(__uint_as_float(xw[q] & 0xFFFF0000u), __uint_as_float(mw[q] & 0xFFFF0000u), acc);
            }
          }
          code = quant(acc, ud.inv_delta, b);
          ++n_fix;
        }
        sC[tok * r + j] = code;
      }
    }
  }
  if (a.stats) {
#pragma unroll
    for (int o = 16; o; o >>= 1) n_fix += __shfl_xor_sync(0xffffffffu, n_fix, o);
    if ((tid & 31) == 0 && n_fix) atomicAdd(reinterpret_cast<unsigned long long*>(a.stats + 1), n_fix);
    if (tid == 0) atomicAdd(reinterpret_cast<unsigned long long*>(a.stats), static_cast<unsigned long long>(kPage) * r);
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;\n" ::"r"(tmem) : "memory");
  }

  // ---- pack the page ----
  const long long pos = static_cast<long long>(a.pos_start) + t0;
  const int lp = static_cast<int>(pos / kPage);
  if (lp >= a.max_pages) {
    if (tid == 0 && a.status) atomicOr(a.status, KVTC_STATUS_BAD_POS);
    return;
  }
  const int32_t pid = a.block_table[static_cast<size_t>(a.seq) * a.max_pages + lp];
  if (pid < 0 || static_cast<uint64_t>(pid) >= a.pages_per_unit) {
    if (tid == 0 && a.status) atomicOr(a.status, KVTC_STATUS_BAD_PAGE);
    return;
  }
  uint32_t* page = reinterpret_cast<uint32_t*>(a.pool + a.pages_per_unit * ud.prefix +
                                               static_cast<uint64_t>(pid) * ud.page_bytes);
  const int n_words = 4 * r * b;
  const bool full = n_valid == kPage;
  for (int wi = tid; wi < n_words; wi += kThreads) {
    // locate the part plane, row, owner and word-in-owner of word wi
    int lo = 0, w = 0, pw = wi;
    const int np = code_nparts(b);
    for (int p = 0; p < np; ++p) {
      int plo, pwd;
      code_part(b, p, plo, pwd);
      const int plane_words = 4 * r * pwd;
      if (pw < plane_words) {
        lo = plo;
        w = pwd;
        break;
      }
      pw -= plane_words;
    }
    const int per_word = 16 / w;
    const uint32_t fmask = (1u << w) - 1u;
    uint32_t word = 0, vmask = 0;
    if (kind == 0) {
      const int row = pw / (8 * w), inrow = pw % (8 * w);
      const int o = inrow / w, q = inrow % w;
      for (int i = 0; i < per_word; ++i) {
        const int pi = q * per_word + i;
        const int t = 16 * (pi >> 1) + 8 * (pi & 1) + o;
        if (t < n_valid) {
          const uint32_t c0 = (sC[t * r + 2 * row] >> lo) & fmask;
          const uint32_t c1 = (sC[t * r + 2 * row + 1] >> lo) & fmask;
          word |= (c0 << (i * w)) | (c1 << (i * w + 16));
          vmask |= (fmask << (i * w)) | (fmask << (i * w + 16));
        }
      }
    } else {
      const int row = pw / (4 * w), inrow = pw % (4 * w);
      const int o = inrow / w, q = inrow % w;
      for (int i = 0; i < per_word; ++i) {
        const int pi = q * per_word + i;
        const int t = 16 * (pi >> 1) + 8 * (pi & 1) + 2 * o;
        if (t < n_valid) {
          word |= ((sC[t * r + row] >> lo) & fmask) << (i * w);
          vmask |= fmask << (i * w);
        }
        if (t + 1 < n_valid) {
          word |= ((sC[(t + 1) * r + row] >> lo) & fmask) << (i * w + 16);
          vmask |= fmask << (i * w + 16);
        }
      }
    }
    if (full) {
      page[wi] = word;
    } else if (vmask) {
      atomicAnd(page + wi, ~vmask);
      atomicOr(page + wi, word);
    }
  }
}

}  // namespace
}  // namespace kvtc

using namespace kvtc;

extern "C" kvtc_status kvtc_encode_prefill(const kvtc_plan* plan, const kvtc_cache* cache, int layer,
                                           const void* k, const void* v, int seq, int pos_start, int n_tok,
                                           void* stream) {
  kvtc_status st = check_uploaded(plan);
  if (st != KVTC_OK) return st;
  if (!cache || !cache->pool || !cache->block_table) return fail(KVTC_EINVAL, "cache is incomplete");
  if (layer < 0 || layer >= plan->L) return fail(KVTC_EINVAL, "layer out of range");
  if (seq < 0 || seq >= cache->n_seq) return fail(KVTC_EINVAL, "seq out of range");
  if (pos_start < 0 || (pos_start % kPage) != 0) return fail(KVTC_EINVAL, "pos_start must be a multiple of 128");
  if (n_tok <= 0) return fail(KVTC_EINVAL, "n_tok must be > 0");
  if (!k || !v) return fail(KVTC_EINVAL, "null device pointer");
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15)
    return fail(KVTC_EINVAL, "k and v must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(cache->pool) & 15) return fail(KVTC_EINVAL, "pool must be 16-byte aligned");
  PrefillArgs a;
  a.units = plan->d_units;
  a.unit0 = layer * plan->H * 2;
  a.H = plan->H;
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.seq = seq;
  a.pos_start = pos_start;
  a.n_tok = n_tok;
  a.pool = static_cast<char*>(cache->pool);
  a.pages_per_unit = cache->pages_per_unit;
  a.block_table = cache->block_table;
  a.max_pages = cache->max_pages;
  a.status = cache->status;
  a.stats = plan->d_stats;
  const size_t smem = 65536 + 16384 + 64;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (prefill)");
  dim3 grid((n_tok + kPage - 1) / kPage, 2 * plan->H);
  prefill_kernel<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return KVTC_OK;
}

extern "C" kvtc_status kvtc_plan_prefill_stats(const kvtc_plan* plan, uint64_t* codes, uint64_t* recomputed,
                                               int reset) {
  kvtc_status st = check_uploaded(plan);
  if (st != KVTC_OK) return st;
  uint64_t h[2] = {0, 0};
  cudaError_t e = cudaMemcpy(h, plan->d_stats, sizeof(h), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "prefill stats copy");
  if (codes) *codes = h[0];
  if (recomputed) *recomputed = h[1];
  if (reset) {
    e = cudaMemset(plan->d_stats, 0, sizeof(h));
    if (e != cudaSuccess) return cuda_fail(e, "prefill stats reset");
  }
  return KVTC_OK;
}
