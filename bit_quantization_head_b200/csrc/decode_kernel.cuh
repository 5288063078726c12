// Decode kernels (templates).  Included by decode.cu and the per-b_K instantiation units.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <utility>

#include "kvtc_internal.h"
#include "ptx.cuh"

namespace kvtc {
namespace dec {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kPartStride = 132;     // floats per partial: m, l, z[128], pad
constexpr int kTargetCtas = 2 * 148; // two CTAs per SM on a B200
constexpr int kMaxHeadsPerLaunch = 64;
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeArgs {
  const UnitDesc* units;
  int layer, H, G, n_hg;
  int heads[kMaxHeadsPerLaunch];  // KV heads handled by this launch
  int n_heads;
  const void* q;
  int q_bf16;
  const int32_t* seq_lens;
  int n_seq;
  const char* pool;
  uint64_t pages_per_unit;
  const int32_t* block_table;
  int max_pages;
  int32_t* status;
  float scale;
  int n_split, pages_per_split, n_stage;
  uint32_t stage_bytes;
  float* ws;  // partials [n_seq][Hq][n_split * kWarps][kPartStride]
};

// Compile-time description of a b-bit code's parts (widths 8/4/2/1, lowest bits first).
template <int B>
struct CodeParts {
  static constexpr int n = (B & 8 ? 1 : 0) + (B & 4 ? 1 : 0) + (B & 2 ? 1 : 0) + (B & 1);
  __host__ __device__ static constexpr int width(int i) {
    int k = 0;
    for (int w = 8; w >= 1; w >>= 1)
      if (B & w) {
        if (k == i) return w;
        ++k;
      }
    return 0;
  }
  __host__ __device__ static constexpr int low(int i) {
    int k = 0, lo = 0;
    for (int w = 8; w >= 1; w >>= 1)
      if (B & w) {
        if (k == i) return lo;
        lo += w;
        ++k;
      }
    return 0;
  }
  static constexpr bool fast = (B == 2 || B == 4 || B == 8);
  // bit offset e of the code inside each fp16 half after extraction (fast path only)
  __host__ __device__ static constexpr int e(int blk, int eta) {
    return B == 2 ? 4 * (blk & 1) + 2 * eta : (B == 4 ? 4 * eta : 0);
  }
};

// Bit offset of the (blk, eta) pair inside a part word of width w.
__host__ __device__ constexpr int pair_offset(int w, int blk, int eta) {
  return ((2 * blk + eta) % (16 / w)) * w;
}

// The pair of codes of (blk, eta) from the part words W[p] (one per part), as an fp16x2
// whose halves are the subnormals c * 2^(e - 24).
template <int B, int BLK, int ETA>
__device__ __forceinline__ uint32_t extract_pair(const uint32_t (&W)[CodeParts<B>::n]) {
  using P = CodeParts<B>;
  if constexpr (P::fast) {
    constexpr int off = pair_offset(B, BLK, ETA);
    constexpr uint32_t m = (1u << B) - 1u;
    if constexpr (off >= 8) {
      return (W[0] >> 8) & ((m << (off - 8)) | (m << (off + 8)));
    } else {
      return W[0] & ((m << off) | (m << (off + 16)));
    }
  } else {
    uint32_t v = 0;
#pragma unroll
    for (int p = 0; p < P::n; ++p) {
      const int w = P::width(p), lo = P::low(p);
      const int off = pair_offset(w, BLK, ETA);
      const uint32_t m = (1u << w) - 1u;
      v |= ((W[p] >> off) & (m | (m << 16))) << lo;
    }
    return v;
  }
}

// Shared-memory layout of one CTA.
struct SmemHead {
  float q[8][128];   // the launch's query heads (zero beyond G)
  float qt[8][128];  // q~ = M_K q
  float S[8];        // sum_j q~_j
  int E[8];          // power-of-two normalisation of q~ for fp16
};

// Per-warp running state (kept in registers; every index below is compile-time).
struct WarpState {
  const uint32_t* pk;  // K page in shared memory
  const uint32_t* pv;  // V page in shared memory
  int tok0, seq_len, rK, rV, nks, nmt, g, tq;
  float alpha[2], beta[2];
  uint32_t bh[8][2], bl[8][2];
  float z[8][4];
  float m_run[2], l_run[2];
};

// One 16-token block of a page: scores, online softmax, value accumulation.
template <int BK, int BV, int BLK>
__device__ __forceinline__ void do_block(WarpState& w) {
  using PK = CodeParts<BK>;
  using PV = CodeParts<BV>;
  // ---- scores: S[tok][head] = sum_j codeK[tok][j] * q^[head][j]
  float sc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    if (ks < w.nks) {
      uint32_t W0[PK::n], W1[PK::n];
      const int rho0 = 8 * ks + w.tq, rho1 = rho0 + 4;
#pragma unroll
      for (int pp = 0; pp < PK::n; ++pp) {
        const int wd = PK::width(pp), lo = PK::low(pp);
        const uint32_t* plane = w.pk + 4 * w.rK * lo;
        const int wsel = w.g * wd + (BLK * wd) / 8;
        W0[pp] = 2 * rho0 < w.rK ? plane[rho0 * 8 * wd + wsel] : 0u;
        W1[pp] = 2 * rho1 < w.rK ? plane[rho1 * 8 * wd + wsel] : 0u;
      }
      const uint32_t A0 = extract_pair<BK, BLK, 0>(W0), A1 = extract_pair<BK, BLK, 1>(W0);
      const uint32_t A2 = extract_pair<BK, BLK, 0>(W1), A3 = extract_pair<BK, BLK, 1>(W1);
      mma_16816(sc, A0, A1, A2, A3, w.bh[ks][0], w.bh[ks][1]);
      mma_16816(sc, A0, A1, A2, A3, w.bl[ks][0], w.bl[ks][1]);
    }
  }
  // rows: sc[0..1] token tok0 + 16*BLK + g (eta 0), sc[2..3] that + 8 (eta 1)
  constexpr int eK0 = PK::fast ? PK::e(BLK, 0) : 0;
  constexpr int eK1 = PK::fast ? PK::e(BLK, 1) : 0;
  const int t0 = w.tok0 + 16 * BLK + w.g, t1 = t0 + 8;
  float s2[4];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    s2[c] = t0 < w.seq_len ? fmaf(w.alpha[c] * (1.0f / (1 << eK0)), sc[c], -w.beta[c]) : -INFINITY;
    s2[2 + c] = t1 < w.seq_len ? fmaf(w.alpha[c] * (1.0f / (1 << eK1)), sc[2 + c], -w.beta[c]) : -INFINITY;
  }
  // ---- online softmax (log2 domain); block max over the 16 tokens of each head
  float resc[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    float v = fmaxf(s2[c], s2[2 + c]);
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
    const float mn = fmaxf(w.m_run[c], v);
    resc[c] = mn == -INFINITY ? 1.0f : ex2(w.m_run[c] - mn);
    w.m_run[c] = mn;
    w.l_run[c] *= resc[c];
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    w.z[mt][0] *= resc[0];
    w.z[mt][1] *= resc[1];
    w.z[mt][2] *= resc[0];
    w.z[mt][3] *= resc[1];
  }
  // probabilities, stored scaled by 2^(7 - e_V(row)) for the value MMA
  constexpr int eV0 = PV::fast ? PV::e(BLK, 0) : 0;
  constexpr int eV1 = PV::fast ? PV::e(BLK, 1) : 0;
  float pr[4];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const float mm = w.m_run[c] == -INFINITY ? 0.0f : w.m_run[c];
    pr[c] = ex2(s2[c] - mm);
    pr[2 + c] = ex2(s2[2 + c] - mm);
  }
  constexpr float sv0 = static_cast<float>(1 << (7 - eV0)), sv1 = static_cast<float>(1 << (7 - eV1));
  const uint32_t P0 = pack_half2(pr[0] * sv0, pr[1] * sv0);
  const uint32_t P1 = pack_half2(pr[2] * sv1, pr[3] * sv1);
  // l from the same fp16-rounded weights the value MMA uses, so that the centering
  // z - m_V * l cancels consistently
  {
    const float2 f0 = half2_to_float2(P0), f1 = half2_to_float2(P1);
    w.l_run[0] += fmaf(f0.x, 1.0f / sv0, f1.x * (1.0f / sv1));
    w.l_run[1] += fmaf(f0.y, 1.0f / sv0, f1.y * (1.0f / sv1));
  }
  const uint32_t b0 = movmatrix_trans(P0), b1 = movmatrix_trans(P1);
  // ---- values: Z^T[j][head] += sum_tok codeV[tok][j] * P[tok][head]
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    if (mt < w.nmt) {
      uint32_t W0[PV::n], W1[PV::n];
      const int j0 = 16 * mt + w.g, j1 = j0 + 8;
#pragma unroll
      for (int pp = 0; pp < PV::n; ++pp) {
        const int wd = PV::width(pp), lo = PV::low(pp);
        const uint32_t* plane = w.pv + 4 * w.rV * lo;
        const int wsel = w.tq * wd + (BLK * wd) / 8;
        W0[pp] = j0 < w.rV ? plane[j0 * 4 * wd + wsel] : 0u;
        W1[pp] = j1 < w.rV ? plane[j1 * 4 * wd + wsel] : 0u;
      }
      const uint32_t A0 = extract_pair<BV, BLK, 0>(W0), A1 = extract_pair<BV, BLK, 0>(W1);
      const uint32_t A2 = extract_pair<BV, BLK, 1>(W0), A3 = extract_pair<BV, BLK, 1>(W1);
      mma_16816(w.z[mt], A0, A1, A2, A3, b0, b1);
    }
  }
}

template <int BK, int BV, int... BLK>
__device__ __forceinline__ void do_page(WarpState& w, std::integer_sequence<int, BLK...>) {
  (do_block<BK, BV, BLK>(w), ...);
}

template <int BK, int BV>
__global__ void __launch_bounds__(kThreads, 2) decode_split_kernel(const DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  SmemHead& sh = *reinterpret_cast<SmemHead*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sizeof(SmemHead));
  unsigned char* stages = smem + ((sizeof(SmemHead) + 8 * kWarps * 8 + 127) / 128) * 128;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int split = blockIdx.x;
  const int hi = blockIdx.y / a.n_hg, hg = blockIdx.y % a.n_hg;
  const int s = blockIdx.z;
  const int h = a.heads[hi];
  const int uK = (a.layer * a.H + h) * 2, uV = uK + 1;
  const UnitDesc dK = a.units[uK], dV = a.units[uV];
  const int rK = dK.r, rV = dV.r;
  const int Hq = a.H * a.G;
  const int g0 = hg * 8, ng = min(8, a.G - g0);

  int seq_len = a.seq_lens[s];
  if (seq_len < 0 || seq_len > a.max_pages * kPage) {
    if (tid == 0 && a.status) atomicOr(a.status, KVTC_STATUS_BAD_POS);
    seq_len = seq_len < 0 ? 0 : a.max_pages * kPage;
  }
  const int n_pages = (seq_len + kPage - 1) / kPage;
  const int p_begin = split * a.pages_per_split;
  const int p_end = min(p_begin + a.pages_per_split, n_pages);
  const int n_my = p_end > p_begin + warp ? (p_end - p_begin - warp + kWarps - 1) / kWarps : 0;

  // ---- prologue: barriers, query, first copies, q~ = M_K q ----
  if (lane == 0)
    for (int i = 0; i < a.n_stage; ++i) mbar_init(&bars[warp * 8 + i], 1);
  for (int i = tid; i < 8 * 128; i += kThreads) {
    const int gg = i >> 7, k = i & 127;
    float v = 0.0f;
    if (gg < ng) {
      const size_t off = (static_cast<size_t>(s) * Hq + h * a.G + g0 + gg) * kD + k;
      v = a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[off])
                   : static_cast<const float*>(a.q)[off];
    }
    sh.q[gg][k] = v;
  }
  fence_mbar_init();
  __syncthreads();

  const uint32_t bytesK = static_cast<uint32_t>(dK.page_bytes), bytesV = static_cast<uint32_t>(dV.page_bytes);
  const char* poolK = a.pool + a.pages_per_unit * dK.prefix;
  const char* poolV = a.pool + a.pages_per_unit * dV.prefix;
  const int32_t* bt = a.block_table + static_cast<size_t>(s) * a.max_pages;
  auto stage_ptr = [&](int i) {
    return stages + (static_cast<size_t>(warp) * a.n_stage + (i % a.n_stage)) * a.stage_bytes;
  };
  // Fill the stage of this warp's i-th page (lane 0).  Every use of a stage completes
  // its barrier phase exactly once: with the copies' bytes, or by a plain arrival when
  // the page id is invalid.
  auto issue = [&](int i) {
    const int p = p_begin + warp + i * kWarps;
    const int32_t pid = bt[p];
    uint64_t* bar = &bars[warp * 8 + (i % a.n_stage)];
    if (pid < 0 || static_cast<uint64_t>(pid) >= a.pages_per_unit) {
      mbar_arrive(bar);
      return;
    }
    unsigned char* st = stage_ptr(i);
    mbar_arrive_expect_tx(bar, bytesK + bytesV);
    bulk_copy_g2s(st, poolK + static_cast<uint64_t>(pid) * bytesK, bytesK, bar);
    bulk_copy_g2s(st + bytesK, poolV + static_cast<uint64_t>(pid) * bytesV, bytesV, bar);
  };
  const int n_first = min(a.n_stage, n_my);
  if (lane == 0)
    for (int i = 0; i < n_first; ++i) issue(i);

  for (int i = tid; i < 8 * 128; i += kThreads) {
    const int gg = i >> 7, j = i & 127;
    float acc = 0.0f;
    if (gg < ng && j < rK) {
      const float* m = dK.M + static_cast<size_t>(j) * kD;
      for (int k = 0; k < kD; ++k) acc = __fmaf_rn(m[k], sh.q[gg][k], acc);
    }
    sh.qt[gg][j] = acc;
  }
  __syncthreads();
  if (tid < 8) {
    float S = 0.0f, amax = 0.0f;
    for (int j = 0; j < rK; ++j) {
      S += sh.qt[tid][j];
      amax = fmaxf(amax, fabsf(sh.qt[tid][j]));
    }
    sh.S[tid] = S;
    sh.E[tid] = amax > 0.0f ? ilogbf(amax) - 14 : 0;
  }
  __syncthreads();

  WarpState w;
  w.rK = rK;
  w.rV = rV;
  w.nks = (rK + 15) >> 4;
  w.nmt = (rV + 15) >> 4;
  w.g = g;
  w.tq = tq;
  w.seq_len = seq_len;
  // B fragments of q^ = q~ * 2^-E (hi and lo fp16 parts) for head n = g.
  {
    const float scl = ldexpf(1.0f, -sh.E[g]);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int k0 = 16 * ks + 8 * half + 2 * tq;
        const float x0 = sh.qt[g][k0] * scl, x1 = sh.qt[g][k0 + 1] * scl;
        const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
        const __half l0 = __float2half_rn(x0 - __half2float(h0)), l1 = __float2half_rn(x1 - __half2float(h1));
        w.bh[ks][half] = static_cast<uint32_t>(__half_as_ushort(h0)) | (static_cast<uint32_t>(__half_as_ushort(h1)) << 16);
        w.bl[ks][half] = static_cast<uint32_t>(__half_as_ushort(l0)) | (static_cast<uint32_t>(__half_as_ushort(l1)) << 16);
      }
    }
  }
  // Score constants (log2 domain) for this lane's heads n = 2tq, 2tq + 1:
  // s2 = alpha_n * 2^-e * acc - beta_n.
  {
    const float mK = 0.5f * static_cast<float>((1 << BK) - 1);
    const float base = a.scale * dK.delta * kLog2e;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int n = 2 * tq + c;
      w.alpha[c] = n < ng ? base * ldexpf(1.0f, sh.E[n] + 24) : 0.0f;
      w.beta[c] = n < ng ? base * mK * sh.S[n] : 0.0f;
      w.m_run[c] = -INFINITY;
      w.l_run[c] = 0.0f;
    }
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) w.z[mt][0] = w.z[mt][1] = w.z[mt][2] = w.z[mt][3] = 0.0f;

  // ---- main loop over this warp's pages ----
  bool dead = false;
  int next_issue = n_first;
  for (int i = 0; i < n_my; ++i) {
    const int p = p_begin + warp + i * kWarps;
    const int32_t pid = bt[p];
    const bool valid = pid >= 0 && static_cast<uint64_t>(pid) < a.pages_per_unit;
    if (!mbar_wait_bounded_warp(&bars[warp * 8 + (i % a.n_stage)], (i / a.n_stage) & 1)) {
      if (lane == 0 && a.status) atomicOr(a.status, KVTC_STATUS_TIMEOUT);
      dead = true;
      // drain (bounded) the copies issued after this page
      for (int i2 = i + 1; i2 < next_issue; ++i2)
        (void)mbar_wait_bounded_warp(&bars[warp * 8 + (i2 % a.n_stage)], (i2 / a.n_stage) & 1);
      break;
    }
    if (valid) {
      const unsigned char* st = stage_ptr(i);
      w.pk = reinterpret_cast<const uint32_t*>(st);
      w.pv = reinterpret_cast<const uint32_t*>(st + bytesK);
      w.tok0 = p * kPage;
      do_page<BK, BV>(w, std::make_integer_sequence<int, 8>{});
    } else if (lane == 0 && a.status) {
      atomicOr(a.status, KVTC_STATUS_BAD_PAGE);
    }
    // release the stage: every lane is done reading it, then refill it
    __syncwarp();
    if (next_issue < n_my && next_issue == i + a.n_stage) {
      if (lane == 0) issue(next_issue);
      ++next_issue;
    }
    __syncwarp();
  }

  // ---- write this warp's partials: (m, l, z) per query head ----
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    float l = w.l_run[c];
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    w.l_run[c] = l;
  }
  const int part = split * kWarps + warp;
  const int n_part = a.n_split * kWarps;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int n = 2 * tq + c;
    if (n < ng) {
      float* dst = a.ws + ((static_cast<size_t>(s) * Hq + h * a.G + g0 + n) * n_part + part) * kPartStride;
      if (g == 0) {
        dst[0] = dead ? -INFINITY : w.m_run[c];
        dst[1] = dead ? 0.0f : w.l_run[c];
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        if (mt < w.nmt) {
          const int j0 = 16 * mt + g, j1 = j0 + 8;
          if (j0 < rV) dst[2 + j0] = dead ? 0.0f : w.z[mt][c];
          if (j1 < rV) dst[2 + j1] = dead ? 0.0f : w.z[mt][2 + c];
        }
      }
    }
  }
}

}  // namespace dec
}  // namespace kvtc

namespace kvtc {
namespace dec {
using SplitFn = void (*)(const DecodeArgs);
template <int BK> SplitFn split_fn_bk(int bV);
}  // namespace dec
}  // namespace kvtc
