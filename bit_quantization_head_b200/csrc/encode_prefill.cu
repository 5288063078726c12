// kvtc_encode_prefill: the per-token projection of a page-aligned span as tensor-core
// tiles (tcgen05, TMEM accumulators), quantized and packed by an epilogue in which each
// thread owns one latent coordinate of a page.
//
// KV-COBRA project page, "How KV-COBRA Works" (Inference: rotate and truncate with
// H.V^T, quantize with the unit's b-bit quantizer) and "Efficiency" (packed b-bit codes).
//
// Persistent kernel, one CTA per SM, nine warps.  A work item is one 128-token page tile
// of one KV head; a CTA takes a contiguous run of items (head-major, so M_K and M_V stay
// in shared memory across the run).
//  * warp 8 (producer): loads the item's K and V tiles with TMA (128-byte swizzled,
//    K-major) and issues D_K = M_K X_K^T and D_V = M_V X_V^T (M = 128 coordinate rows,
//    zero beyond r; N = 128 tokens; K = 128 dims, bf16 operands, fp32 accumulate) into
//    one of two TMEM accumulator stages, so the next item's MMAs overlap this item's
//    epilogue.
//  * warps 0-7 (epilogue): warp w reads TMEM lanes 32 (w % 4) .. +31 of D_K (w < 4) or
//    D_V (w >= 4): lane = coordinate j, columns = tokens.  A thread quantizes its
//    coordinate for the 128 tokens and builds its row of the page layout in registers
//    (a layout row is one coordinate for V and one coordinate pair for K, the pair's two
//    halves coming from neighbouring lanes), then writes it with 16-byte stores.
//
// Bit-exactness with the canonical arithmetic (eight fp32 fma chains over k mod 8, then
// a fixed pairwise sum): both the canonical value and the tensor-core sum are within
// (639 * 2^-24) * sum_k |x_k M_jk| of the exact dot product of the same bf16 operands
// (at most 19 roundings on any path of the canonical order; at most one rounding of the
// fp32 accumulator per product for the tensor core, counted twice), and Cauchy-Schwarz
// bounds that by beta = 2^-14 * ||x||_2 * ||M_j||_2.  The quantizer is monotone, and with
// U = fl(fl(y * inv_delta) + 2^(b-1)) a change of y by at most beta moves U by at most
// eps = beta * inv_delta * (1 + 2^-20) + 2^-21 * (2^b + 1).  So when U is farther than eps
// from every code boundary n in [1, 2^b - 1], floor(U) clamped is the canonical code;
// otherwise the code is queued and recomputed in the canonical order afterwards.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kvtc_internal.h"
#include "layout.cuh"
#include "ptx.cuh"

namespace kvtc {
namespace {

constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = kEpiThreads + 32;
constexpr uint32_t kHalfBytes = 128 * 128;     // one 64-column half of a 128-row bf16 tile
constexpr uint32_t kTileBytes = 2 * kHalfBytes;  // 128 rows x 128 bf16
constexpr int kQueueCap = 2048;
constexpr int kTmemCols = 512;                  // two stages x (D_K, D_V) x 128 columns
constexpr uint32_t kWaitLimit = 1u << 16;      // sleeps of up to 20 us per wait

struct PrefillArgs {
  const UnitDesc* units;
  int unit0, H;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  int seq, pos_start, n_tok, n_tiles, n_items;
  char* pool;
  uint64_t pages_per_unit;
  const int32_t* block_table;
  int max_pages;
  int32_t* status;
  uint64_t* stats;  // [0] codes produced, [1] codes recomputed in canonical order
};

struct __align__(1024) Smem {
  unsigned char x[2][2][kTileBytes];  // [stage][K, V] input tiles (SW128, K-major)
  unsigned char a[2][kTileBytes];     // M_K, M_V (bf16 rows, zero beyond r; SW128, K-major)
  float eps[2][128];                  // per-token threshold band (K, V)
  uint32_t queue[kQueueCap];          // codes to recompute: t | j << 7 | kind << 14
  int qcount;
  int overflow;
  int dead;
  uint32_t tmem_base;
  uint64_t x_full[2], x_empty[2];     // per X stage
  uint64_t tm_full[2], tm_empty[2];   // per TMEM stage
  uint64_t epi_done;                  // one phase per finished item (M may be replaced)
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(kEpiThreads) : "memory"); }
// Barrier of the epilogue warps that also ORs a predicate over them (a uniform answer).
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kEpiThreads)
      : "memory");
  return r != 0;
}

// SM100 shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row groups 1024
// bytes apart (SBO), LBO unused (1), version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (static_cast<uint64_t>(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

// Bounded wait on an mbarrier phase.  Returns false after the limit, or at once when the
// CTA has given up (dead), so that no role can wait forever on another.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t phase, volatile int* dead) {
  if (mbar_try_wait(bar, phase)) return true;
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait_sleep(bar, phase, 20000u)) return true;  // sleeps up to 20 us
    if (*dead) return false;
  }
  return false;
}

// ------------------------------------------------------------------ code parts
__host__ __device__ constexpr int n_parts(int b) { return (b >> 3 & 1) + (b >> 2 & 1) + (b >> 1 & 1) + (b & 1); }
__host__ __device__ constexpr int part_w(int b, int p) {
  int k = 0;
  for (int w = 8; w >= 1; w >>= 1)
    if (b & w) {
      if (k == p) return w;
      ++k;
    }
  return 0;
}
__host__ __device__ constexpr int part_lo(int b, int p) {
  int k = 0, lo = 0;
  for (int w = 8; w >= 1; w >>= 1)
    if (b & w) {
      if (k == p) return lo;
      lo += w;
      ++k;
    }
  return 0;
}

__device__ __forceinline__ int quant_code(float y, float inv_delta, float half, int maxc) {
  const float u = __fadd_rn(__fmul_rn(y, inv_delta), half);
  return min(max(__float2int_rd(u), 0), maxc);  // NaN -> 0, +-inf -> the end codes
}

// Overwrites code (t, j) of a page with atomics (field by field).
__device__ __forceinline__ void patch_code(uint32_t* page, int kind, int r, int b, int t, int j, uint32_t code) {
  const int np = code_nparts(b);
  for (int i = 0; i < np; ++i) {
    int lo, w;
    code_part(b, i, lo, w);
    const FieldPos f = field_pos(kind, r, lo, w, t, j);
    const uint32_t mask = ((1u << w) - 1u) << f.bit;
    atomicAnd(page + f.word, ~mask);
    atomicOr(page + f.word, ((code >> lo) & ((1u << w) - 1u)) << f.bit);
  }
}

// Everything one epilogue thread needs about its row of the current item.
struct RowCtx {
  uint32_t taddr;       // TMEM address of this warp's lanes, column of token 0
  int j;                // coordinate (row of D)
  int r;                // rows of the unit
  float inv_delta, half;
  int maxc;
  const float* eps;     // [128] threshold band of each token (shared memory)
  uint32_t* page;       // the unit's page, or nullptr when it cannot be written
  int kind;
  Smem* sm;
};

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Quantize one chunk of 32 tokens (t0 .. t0 + 31) of this thread's coordinate: codes and
// the mask of codes within eps of a boundary.  FMA/ALU pipes only: U = fma(y, 1/delta, h)
// (one rounding where the canonical quantizer has two; eps covers the difference), the
// clamped U is rounded to an integer by adding 2^23, and floor follows from that.
__device__ __forceinline__ uint32_t quant_chunk(const RowCtx& c, int t0, const float (&v)[32], int (&code)[32]) {
  uint32_t flags = 0;
  const float top = static_cast<float>(c.maxc) + 0.5f;
  const float4* e4 = reinterpret_cast<const float4*>(c.eps + t0);
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const float4 ev = e4[g];
    const float eps[4] = {ev.x, ev.y, ev.z, ev.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 4 * g + q;
      const float u = __fmaf_rn(v[i], c.inv_delta, c.half);
      const float vc = fminf(fmaxf(u, 0.0f), top);           // NaN -> 0
      const float vm = __fadd_rn(vc, 8388608.0f);             // 2^23 + rint(vc)
      const float n = __fsub_rn(vm, 8388608.0f);              // rint(vc)
      code[i] = (__float_as_int(vm) - 0x4B000000) - (n > vc ? 1 : 0);  // floor(vc)
      // near a boundary (clamp boundaries 0 and 2^b included, harmlessly); NaN is near
      flags |= !(fabsf(u - n) > eps[q]) ? (1u << i) : 0u;
    }
  }
  return flags;
}

// Queue the flagged codes of a chunk (a set overflow flag sends the item to the slow path).
__device__ __forceinline__ void queue_flags(const RowCtx& c, int t0, uint32_t flags) {
  while (flags) {
    const int i = __ffs(flags) - 1;
    flags &= flags - 1;
    const int idx = atomicAdd(&c.sm->qcount, 1);
    if (idx < kQueueCap)
      c.sm->queue[idx] = static_cast<uint32_t>(t0 + i) | (static_cast<uint32_t>(c.j) << 7) |
                         (static_cast<uint32_t>(c.kind) << 14);
    else
      c.sm->overflow = 1;
  }
}

// Full-page row, in a loop over four 32-token chunks.  Layout (per part of width w, with
// P = 16 / w pairs per word, pair index pi = t / 8): K row rho = j / 2 holds coordinates
// (2 rho, 2 rho + 1), owner o = t % 8 has words [o w, o w + w), the field of pair pi sits
// in word o w + pi / P at bit (pi % P) w (+16 for odd j); V row j, owner o = (t % 8) / 2,
// half t % 2 adds 16.  A chunk covers pi = 4c .. 4c + 3, so:
//   w = 1, 2: the chunk fills part of word column c / (P / 4), at shift (4c % P) w; the
//     row's words stay in registers until the page is done (one 16-byte store per w);
//   w = 4, 8: the chunk completes word columns c (w = 4) or 2c, 2c + 1 (w = 8); they are
//     stored at once.
// For K the pair's two lanes (j, j ^ 1) each build their half and swap owners 0-3 / 4-7.
template <int KIND, int B>
__device__ __noinline__ void encode_row_full(const RowCtx& c) {
  constexpr int NO = KIND == 0 ? 8 : 4;       // owners per row
  constexpr int NP = n_parts(B);
  const bool row_ok = c.j < c.r;
  const bool odd = c.j & 1;
  // words of the w <= 2 parts, kept for the whole page: [owner][w]
  uint32_t Wk[NP][NO * 2];
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int i = 0; i < NO * 2; ++i) Wk[p][i] = 0u;
  // the row of part p starts at word 4 r lo (plane) + row offset
  for (int ch = 0; ch < 4; ++ch) {
    float v[32];
    __syncwarp();
    tmem_ld32(c.taddr + 32 * ch, v);
    int code[32];
    uint32_t flags = quant_chunk(c, 32 * ch, v, code);
    if (!row_ok) flags = 0u;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int w = part_w(B, p), lo = part_lo(B, p);
      const uint32_t fm = (1u << w) - 1u;
      // chunk-local words [owner][qq], qq = 0 (w <= 4) or the two columns of w = 8
      uint32_t L[NO][2];
#pragma unroll
      for (int o = 0; o < NO; ++o) L[o][0] = L[o][1] = 0u;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int o = KIND == 0 ? (i & 7) : ((i & 7) >> 1);
        const int pl = i >> 3;  // pi - 4c
        const int qq = w == 8 ? (pl >> 1) : 0;
        const int off = (w == 8 ? (pl & 1) * 8 : pl * w) + (KIND == 1 ? 16 * (i & 1) : 0);
        const uint32_t f = NP == 1 ? static_cast<uint32_t>(code[i]) : (static_cast<uint32_t>(code[i]) >> lo) & fm;
        L[o][qq] += f << off;
      }
      if (KIND == 0) {
#pragma unroll
        for (int o = 0; o < NO; ++o) {
          L[o][0] = odd ? (L[o][0] << 16) : L[o][0];
          L[o][1] = odd ? (L[o][1] << 16) : L[o][1];
        }
      }
      if (w <= 2) {
        // merge into the kept words: column q = c / (P / 4), shift (4c % P) w
        const int P = 16 / w;
        const int q = (4 * ch) / P;
        const int sh = ((4 * ch) % P) * w;
#pragma unroll
        for (int o = 0; o < NO; ++o) {
          const uint32_t val = L[o][0] << sh;
#pragma unroll
          for (int qi = 0; qi < w; ++qi) Wk[p][o * w + qi] |= (qi == q) ? val : 0u;
        }
      } else {
        // complete words: w = 4 -> word o*4 + c; w = 8 -> words o*8 + 2c, +1
        uint32_t out[4][2];
        if (KIND == 0) {
#pragma unroll
          for (int o = 0; o < 4; ++o) {
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
              const uint32_t send = odd ? L[o][qq] : L[o + 4][qq];
              const uint32_t keep = odd ? L[o + 4][qq] : L[o][qq];
              out[o][qq] = keep | __shfl_xor_sync(0xffffffffu, send, 1);
            }
          }
        } else {
#pragma unroll
          for (int o = 0; o < 4; ++o) out[o][0] = L[o][0], out[o][1] = L[o][1];
        }
        if (row_ok && c.page) {
          uint32_t* rowp = c.page + 4 * c.r * lo +
                           (KIND == 0 ? (c.j >> 1) * 8 * w + (c.j & 1) * 4 * w : c.j * 4 * w);
#pragma unroll
          for (int o = 0; o < 4; ++o) {
            if (w == 4) {
              rowp[o * 4 + ch] = out[o][0];
            } else {
              *reinterpret_cast<uint2*>(rowp + o * 8 + 2 * ch) = make_uint2(out[o][0], out[o][1]);
            }
          }
        }
      }
    }
    if (flags) queue_flags(c, 32 * ch, flags);
  }
  __syncwarp();
  // the w <= 2 parts: swap halves (K) and store the row with 16-byte stores
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int w = part_w(B, p), lo = part_lo(B, p);
    if (w > 2) continue;
    uint32_t out[8];
    if (KIND == 0) {
#pragma unroll
      for (int i = 0; i < 4 * w; ++i) {
        const uint32_t mine_lo = Wk[p][i], mine_hi = Wk[p][4 * w + i];
        const uint32_t send = odd ? mine_lo : mine_hi;
        const uint32_t keep = odd ? mine_hi : mine_lo;
        out[i] = keep | __shfl_xor_sync(0xffffffffu, send, 1);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4 * w; ++i) out[i] = Wk[p][i];
    }
    if (row_ok && c.page) {
      uint32_t* dst = c.page + 4 * c.r * lo + (KIND == 0 ? (c.j >> 1) * 8 * w + (c.j & 1) * 4 * w : c.j * 4 * w);
#pragma unroll
      for (int q = 0; q < w; ++q)
        reinterpret_cast<uint4*>(dst)[q] = make_uint4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
    }
  }
}

// Partial page (the last tile of a span): each valid code is written with atomics (the
// slots of tokens beyond the span keep their bits).
__device__ __noinline__ void encode_row_generic(const RowCtx& c, int b, int n_valid) {
  const bool row_ok = c.j < c.r;
  for (int ch = 0; ch < 4; ++ch) {
    float v[32];
    __syncwarp();
    tmem_ld32(c.taddr + 32 * ch, v);
    int code[32];
    uint32_t flags = quant_chunk(c, 32 * ch, v, code);
    if (!row_ok) continue;
    const int nv = min(max(n_valid - 32 * ch, 0), 32);
    flags &= nv == 32 ? 0xFFFFFFFFu : ((1u << nv) - 1u);
    if (c.page) {
#pragma unroll 4
      for (int i = 0; i < nv; ++i) patch_code(c.page, c.kind, c.r, b, 32 * ch + i, c.j, static_cast<uint32_t>(code[i]));
    }
    if (flags) queue_flags(c, 32 * ch, flags);
  }
}

template <int KIND>
__device__ __forceinline__ void encode_row_dispatch(const RowCtx& c, int b) {
  switch (b) {
    case 2: encode_row_full<KIND, 2>(c); break;
    case 3: encode_row_full<KIND, 3>(c); break;
    case 4: encode_row_full<KIND, 4>(c); break;
    case 5: encode_row_full<KIND, 5>(c); break;
    case 6: encode_row_full<KIND, 6>(c); break;
    case 7: encode_row_full<KIND, 7>(c); break;
    default: encode_row_full<KIND, 8>(c); break;
  }
}

// The canonical projection of the item's token t against row j of M, both read from the
// swizzled tiles in shared memory (16-byte chunk c of row r sits at chunk c ^ (r % 8) of
// its 128-byte line).
__device__ __forceinline__ float canonical_y_smem(const unsigned char* xt, const unsigned char* at, int t, int j) {
  float ch[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 4
  for (int c16 = 0; c16 < 16; ++c16) {
    const int half = c16 >> 3, c = c16 & 7;
    const uint4 xv = *reinterpret_cast<const uint4*>(xt + half * kHalfBytes + t * 128 + ((c ^ (t & 7)) << 4));
    const uint4 mv = *reinterpret_cast<const uint4*>(at + half * kHalfBytes + j * 128 + ((c ^ (j & 7)) << 4));
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, mw[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      ch[2 * q] = __fmaf_rn(__uint_as_float(xw[q] << 16), __uint_as_float(mw[q] << 16), ch[2 * q]);
      ch[2 * q + 1] =
          __fmaf_rn(__uint_as_float(xw[q] & 0xFFFF0000u), __uint_as_float(mw[q] & 0xFFFF0000u), ch[2 * q + 1]);
    }
  }
  return __fadd_rn(__fadd_rn(__fadd_rn(ch[0], ch[1]), __fadd_rn(ch[2], ch[3])),
                   __fadd_rn(__fadd_rn(ch[4], ch[5]), __fadd_rn(ch[6], ch[7])));
}

// ------------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ PrefillArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the swizzled tiles need a 1024-byte aligned base: round up inside the allocation
  // (the launch asks for sizeof(Smem) + 1024 bytes)
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int per_cta = (a.n_items + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
  const int first = static_cast<int>(blockIdx.x) * per_cta;
  const int n_my = min(a.n_items, first + per_cta) - first;
  if (n_my <= 0) return;  // the whole CTA, before any barrier or allocation

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.x_full[s], 1);
      mbar_init(&sm.x_empty[s], 1);
      mbar_init(&sm.tm_full[s], 1);
      mbar_init(&sm.tm_empty[s], 1);
    }
    mbar_init(&sm.epi_done, 1);
    sm.qcount = 0;
    sm.overflow = 0;
    sm.dead = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&sm.tmem_base)),
                 "n"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* dead = &sm.dead;

  if (warp == kEpiWarps) {
    // ================= producer: TMA loads and MMA issue =================
    // Item k uses X stage k % 2 and TMEM stage k % 2.  Order per item: MMAs of item k,
    // then the tile copies of item k + 1 (whose stage item k - 1's epilogue releases).
    int cur_head = -1;
    int issued = 0;      // items whose MMAs were committed
    int tma_issued = 0;  // items whose tiles were requested
    auto issue_tiles = [&](int kk) {  // lane 0
      const int it = first + kk, hd = it / a.n_tiles, tl = it % a.n_tiles;
      const int xs = kk & 1;
      mbar_arrive_expect_tx(&sm.x_full[xs], 2 * kTileBytes);
      for (int kind = 0; kind < 2; ++kind) {
        const CUtensorMap* map = kind ? &tmV : &tmK;
        tma_load_3d(sm.x[xs][kind], map, 0, tl * kPage, hd, &sm.x_full[xs]);
        tma_load_3d(sm.x[xs][kind] + kHalfBytes, map, 64, tl * kPage, hd, &sm.x_full[xs]);
      }
      tma_issued = kk + 1;
    };
    if (lane == 0) issue_tiles(0);
    for (int k = 0; k < n_my; ++k) {
      const int item = first + k, head = item / a.n_tiles;
      const int s = k & 1;
      bool ok = true;
      if (head != cur_head) {
        // the previous item's epilogue reads M (canonical recomputation): let it finish
        if (k > 0) ok = wait_phase(&sm.epi_done, (k - 1) & 1, dead);
        if (ok) {
          for (int kind = 0; kind < 2; ++kind) {
            const UnitDesc ud = a.units[a.unit0 + 2 * head + kind];
            const uint32_t base = smem_u32(sm.a[kind]);
            for (int i = lane; i < 128 * 16; i += 32) {
              const int row = i >> 4, c16 = i & 15;  // 16-byte chunk c16 of the 256-byte row
              const int half = c16 >> 3, c = c16 & 7;
              const uint32_t dst = base + half * kHalfBytes + row * 128 + ((c ^ (row & 7)) << 4);
              const bool valid = row < ud.r;
              cp_async16(dst, ud.Mbf + static_cast<size_t>(valid ? row : 0) * kD + c16 * 8, valid);
            }
          }
          cp_async_wait_all();
          fence_proxy_async_smem();
          cur_head = head;
        }
      }
      __syncwarp();
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0 && ok) {
        ok = wait_phase(&sm.x_full[s], (k >> 1) & 1, dead);
        if (ok && k >= 2) ok = wait_phase(&sm.tm_empty[s], ((k - 2) >> 1) & 1, dead);
        if (ok) {
          tc_fence_after();
          // D = M X^T: M = 128 (rows), N = 128 (tokens), bf16 x bf16 -> fp32, both K-major
          const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(128 >> 3) << 17) |
                                 (static_cast<uint32_t>(128 >> 4) << 24);
          for (int kind = 0; kind < 2; ++kind) {
            const uint32_t d = tmem + static_cast<uint32_t>(s * 256 + kind * 128);
            const uint32_t sa = smem_u32(sm.a[kind]), sx = smem_u32(sm.x[s][kind]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;  // 16 bf16 = 32 bytes
              const uint64_t da = desc_sw128(sa + off), db = desc_sw128(sx + off);
              const uint32_t acc = kk > 0 ? 1u : 0u;
              asm volatile(
                  "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                  " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
                  "l"(da), "l"(db), "r"(idesc), "r"(acc)
                  : "memory");
            }
          }
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                           smem_u32(&sm.tm_full[s]))
                       : "memory");
          issued = k + 1;
          // prefetch the next item's tiles into the other stage once item k - 1 is done
          if (k + 1 < n_my) {
            if (k >= 1) ok = wait_phase(&sm.x_empty[(k + 1) & 1], ((k - 1) >> 1) & 1, dead);
            if (ok) issue_tiles(k + 1);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) {
        if (lane == 0) {
          *dead = 1;
          if (a.status) atomicOr(a.status, KVTC_STATUS_TIMEOUT);
        }
        break;
      }
      if (__shfl_sync(0xffffffffu, *dead, 0)) break;
    }
    // drain (bounded, also when the CTA gave up): the last tile copies and the last
    // committed MMAs must complete before the CTA exits and frees TMEM
    if (lane == 0) {
      volatile int never = 0;
      if (tma_issued > 0) (void)wait_phase(&sm.x_full[(tma_issued - 1) & 1], ((tma_issued - 1) >> 1) & 1, &never);
      if (issued > 0) (void)wait_phase(&sm.tm_full[(issued - 1) & 1], ((issued - 1) >> 1) & 1, &never);
    }
    __syncwarp();
  } else {
    // ================= epilogue: quantize and pack =================
    const int kind = warp >> 2, quarter = warp & 3;
    const int j = 32 * quarter + lane;
    uint64_t n_codes = 0, n_fix = 0;
    for (int k = 0; k < n_my; ++k) {
      const int item = first + k, head = item / a.n_tiles, tile = item % a.n_tiles;
      const int s = k & 1;
      bool ok = wait_phase(&sm.tm_full[s], (k >> 1) & 1, dead);
      // the X tile's TMA completed before the MMAs were issued; waiting on its barrier
      // (still in this item's phase) makes the tile visible to this thread
      if (ok) ok = wait_phase(&sm.x_full[s], (k >> 1) & 1, dead);
      if (epi_any(!ok)) {
        if (tid == 0) {
          *dead = 1;
          if (a.status) atomicOr(a.status, KVTC_STATUS_TIMEOUT);
        }
        break;
      }
      tc_fence_after();
      const UnitDesc dK = a.units[a.unit0 + 2 * head], dV = a.units[a.unit0 + 2 * head + 1];
      const int t0 = tile * kPage;
      const int n_valid = min(kPage, a.n_tok - t0);
      // ---- per-token threshold band from ||x||_2 (thread = (kind, token))
      {
        const int nk = tid >> 7, t = tid & 127;
        const UnitDesc& ud = nk ? dV : dK;
        const unsigned char* row = sm.x[s][nk] + t * 128;
        float ss = 0.0f;
        uint32_t any = 0u;  // OR of the magnitude bits: 0 only for a row of +-0
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            // chunk c of the swizzled row (the sum is order-free; reading the lane's own
            // swizzle keeps eight neighbouring rows on distinct banks)
            const uint4 xv = *reinterpret_cast<const uint4*>(row + half * kHalfBytes + ((c ^ (t & 7)) << 4));
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float x0 = __uint_as_float(xw[q] << 16), x1 = __uint_as_float(xw[q] & 0xFFFF0000u);
              ss = fmaf(x1, x1, fmaf(x0, x0, ss));
              any |= xw[q] & 0x7FFF7FFFu;
            }
          }
        }
        float nrm = sqrtf(ss) * 1.001f;
        // a row of tiny values can underflow ss (or lose it to subnormal rounding) while its
        // sums still matter at a small step: bound ||x||_2 by sqrt(128) * max |x| instead
        if (ss < 0x1p-100f && any != 0u) {
          float am = 0.0f;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint4 xv = *reinterpret_cast<const uint4*>(row + (c >> 3) * kHalfBytes + ((c & 7) << 4));
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
              am = fmaxf(am, fmaxf(fabsf(__uint_as_float(xw[q] << 16)), fabsf(__uint_as_float(xw[q] & 0xFFFF0000u))));
          }
          nrm = am * 11.32f;
        }
        float e = ldexpf(nrm, -14) * ud.mnorm * ud.inv_delta * (1.0f + 0x1p-20f) +
                  0x1p-21f * static_cast<float>((1 << ud.b) + 1);
        if (!(nrm < INFINITY)) e = INFINITY;  // non-finite input: recompute every code
        if (any == 0u) e = -1.0f;             // zero token: every sum is exactly 0
        sm.eps[nk][t] = e;
      }
      epi_sync();
      // ---- destination pages (K and V units of this head)
      uint32_t* pages[2] = {nullptr, nullptr};
      {
        const long long pos = static_cast<long long>(a.pos_start) + t0;
        const int lp = static_cast<int>(pos / kPage);
        if (lp < a.max_pages) {
          const int32_t pid = a.block_table[static_cast<size_t>(a.seq) * a.max_pages + lp];
          if (pid >= 0 && static_cast<uint64_t>(pid) < a.pages_per_unit) {
            pages[0] = reinterpret_cast<uint32_t*>(a.pool + a.pages_per_unit * dK.prefix +
                                                   static_cast<uint64_t>(pid) * dK.page_bytes);
            pages[1] = reinterpret_cast<uint32_t*>(a.pool + a.pages_per_unit * dV.prefix +
                                                   static_cast<uint64_t>(pid) * dV.page_bytes);
          } else if (tid == 0 && a.status) {
            atomicOr(a.status, KVTC_STATUS_BAD_PAGE);
          }
        } else if (tid == 0 && a.status) {
          atomicOr(a.status, KVTC_STATUS_BAD_POS);
        }
      }
      // ---- codes
      const UnitDesc& ud = kind ? dV : dK;
      if (32 * quarter < ud.r) {
        RowCtx c;
        c.taddr = tmem + (static_cast<uint32_t>(32 * quarter) << 16) + static_cast<uint32_t>(s * 256 + kind * 128);
        c.j = j;
        c.r = ud.r;
        c.inv_delta = ud.inv_delta;
        c.half = static_cast<float>(1 << (ud.b - 1));
        c.maxc = (1 << ud.b) - 1;
        c.eps = sm.eps[kind];
        c.page = pages[kind];
        c.kind = kind;
        c.sm = &sm;
        if (n_valid == kPage) {
          if (kind == 0)
            encode_row_dispatch<0>(c, ud.b);
          else
            encode_row_dispatch<1>(c, ud.b);
        } else {
          encode_row_generic(c, ud.b, n_valid);
        }
        if (j < ud.r) n_codes += static_cast<uint64_t>(n_valid);
      }
      tc_fence_before();
      epi_sync();
      if (tid == 0) mbar_arrive(&sm.tm_empty[s]);  // TMEM stage s may be overwritten
      // ---- codes near a threshold: the canonical order decides (operands from the
      // tiles in shared memory, which stay until this item releases its X stage)
      const int nq = min(sm.qcount, kQueueCap);
      for (int e = tid; e < nq; e += kEpiThreads) {
        const uint32_t ent = sm.queue[e];
        const int t = ent & 127, jj = (ent >> 7) & 127, kd = (ent >> 14) & 1;
        const UnitDesc& u2 = kd ? dV : dK;
        const float y = canonical_y_smem(sm.x[s][kd], sm.a[kd], t, jj);
        const uint32_t code = static_cast<uint32_t>(
            quant_code(y, u2.inv_delta, static_cast<float>(1 << (u2.b - 1)), (1 << u2.b) - 1));
        if (pages[kd]) patch_code(pages[kd], kd, u2.r, u2.b, t, jj, code);
      }
      n_fix += static_cast<uint64_t>(nq);
      // ---- queue overflow (pathological inputs): recompute every code of the item
      epi_sync();
      if (sm.overflow) {
        for (int e = tid; e < 2 * 128 * 128; e += kEpiThreads) {
          const int kd = e >> 14, jj = (e >> 7) & 127, t = e & 127;
          const UnitDesc& u2 = kd ? dV : dK;
          if (jj >= u2.r || t >= n_valid || !pages[kd]) continue;
          const float y = canonical_y_smem(sm.x[s][kd], sm.a[kd], t, jj);
          const uint32_t code = static_cast<uint32_t>(
              quant_code(y, u2.inv_delta, static_cast<float>(1 << (u2.b - 1)), (1 << u2.b) - 1));
          patch_code(pages[kd], kd, u2.r, u2.b, t, jj, code);
        }
        n_fix += static_cast<uint64_t>(n_valid) * (dK.r + dV.r);
        epi_sync();
      }
      if (tid == 0) {
        sm.qcount = 0;
        sm.overflow = 0;
        mbar_arrive(&sm.x_empty[s]);  // the X stage may be refilled
        mbar_arrive(&sm.epi_done);    // M may be replaced
      }
      // the next item's queue pushes come after its first epi_sync; stop together
      if (epi_any(*dead)) break;
    }
    if (a.stats) {
      // codes counted per row-owning thread; one atomic per warp
      unsigned long long c0 = n_codes, c1 = (tid == 0) ? n_fix : 0ull;
#pragma unroll
      for (int o = 16; o; o >>= 1) c0 += __shfl_xor_sync(0xffffffffu, c0, o);
      if (lane == 0 && c0) atomicAdd(reinterpret_cast<unsigned long long*>(a.stats), c0);
      if (tid == 0 && c1) atomicAdd(reinterpret_cast<unsigned long long*>(a.stats + 1), c1);
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "n"(kTmemCols) : "memory");
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [n_tok][H][128] bf16 as a 3-D tensor (dim, token, head) with 64 x 128 x 1 boxes,
// 128-byte swizzle: one box is one K-half of a 128-token tile in the MMA's layout.
kvtc_status make_map(CUtensorMap* m, const void* base, int n_tok, int H) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return fail(KVTC_ECUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(n_tok), static_cast<cuuint64_t>(H)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(H) * kD * 2, static_cast<cuuint64_t>(kD) * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KVTC_ECUDA, "cuTensorMapEncodeTiled failed (prefill input)");
  return KVTC_OK;
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
  for (int u = layer * plan->H * 2; u < (layer + 1) * plan->H * 2; ++u)
    if (plan->b[u] == kRawBits)
      return fail(KVTC_EINVAL, "prefill encodes compressed units only; use kvtc_encode_append for keys-only plans");
  if (seq < 0 || seq >= cache->n_seq) return fail(KVTC_EINVAL, "seq out of range");
  if (pos_start < 0 || (pos_start % kPage) != 0) return fail(KVTC_EINVAL, "pos_start must be a multiple of 128");
  if (n_tok <= 0) return fail(KVTC_EINVAL, "n_tok must be > 0");
  if (!k || !v) return fail(KVTC_EINVAL, "null device pointer");
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15)
    return fail(KVTC_EINVAL, "k and v must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(cache->pool) & 15) return fail(KVTC_EINVAL, "pool must be 16-byte aligned");
  CUtensorMap mk, mv;
  st = make_map(&mk, k, n_tok, plan->H);
  if (st != KVTC_OK) return st;
  st = make_map(&mv, v, n_tok, plan->H);
  if (st != KVTC_OK) return st;
  PrefillArgs a;
  a.units = plan->d_units;
  a.unit0 = layer * plan->H * 2;
  a.H = plan->H;
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.seq = seq;
  a.pos_start = pos_start;
  a.n_tok = n_tok;
  a.n_tiles = (n_tok + kPage - 1) / kPage;
  a.n_items = a.n_tiles * plan->H;
  a.pool = static_cast<char*>(cache->pool);
  a.pages_per_unit = cache->pages_per_unit;
  a.block_table = cache->block_table;
  a.max_pages = cache->max_pages;
  a.status = cache->status;
  a.stats = plan->d_stats;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (prefill)");
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  // equal runs of items per CTA (a run never starts past the end)
  int grid = std::min(a.n_items, n_sm);
  const int per = (a.n_items + grid - 1) / grid;
  grid = (a.n_items + per - 1) / per;
  prefill_kernel<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(mk, mv, a);
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
