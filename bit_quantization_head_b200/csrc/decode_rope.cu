// kvtc_decode_attention_rope: decode attention over a cache whose keys were coded before
// the rotary position embedding.
//
// KV-COBRA project page, Results (its caption: keys are compressed pre-RoPE).  The codes
// hold keys before the rotation, so q~ = M_K q (the shortcut of kvtc_decode_attention)
// no longer applies: the rotation of token t depends on t.  Per 16-token block a warp
//   * reconstructs K-hat = delta_K (C - m_K) M_K in d-space on the tensor cores (A = the
//     codes as exact fp16 subnormals, B = M_K^T as fp16 hi + lo fragments read through L1;
//     the centring is the column sums of M_K times m_K, subtracted in fp32);
//   * rotates each row by its offset rho < 16 inside the block (rotate-half pairs
//     (i, i + 64), angles rho w_i from a table), and scores it against the query rotated
//     back by the block's start: s_t = q . R(t) k_t = (R(-(t0 + 16 a)) q) . (R(rho) k_t)
//     with t = t0 + 16 a + rho (t0 the page start; the page part of the angle is reduced
//     in fp64, the block part advances by a fixed rotation);
//   * runs the same lazy online softmax and latent value MMAs as the split decode.
// The query is taken as given (already rotated to its own position, as a model applies
// RoPE to q before attention); cached token t sits at position t.  The partials are
// merged and back-projected by the last CTA of each (sequence, KV head, head group), as
// in kvtc_decode_attention, through the same workspace.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <utility>
#include <vector>

#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
namespace rope {

constexpr int kRopeStages = 2;

struct RopeArgs {
  DecodeArgs d;
  double omega[64];        // w_i = base^(-2i/128), fp64 (page angles t0 w_i)
  float2 rot1[16][64];     // (cos rho w_i, sin rho w_i), rho < 16 (computed in fp64)
  float2 rot16[64];        // (cos 16 w_i, sin 16 w_i)
};

struct __align__(16) RopeSmem {
  float2 rot1[16][64];     // R(rho) for the key rows
  float2 rot16[64];        // the block step of the query rotation
  float2 page[kWarps][64]; // per warp: (cos t0 w_i, sin t0 w_i) of its current page
  float msum[128];         // m_K * sum_j M_K[j][i]
  float qs[8][128];        // the group's queries, head n scaled by 2^-Eq[n]
  float S[8];
  int Eq[8];               // power-of-two scaling of q for fp16
  int last;
};

// A-fragment pair of a block at run-time block index: the b-bit field of pair index
// pi = 2 blk + eta from word W (fast widths: one field; e = 0, the code in bits [0, b) of
// each half, i.e. the fp16 subnormal c * 2^-24).
template <int B>
__device__ __forceinline__ uint32_t pair_rt(const uint32_t* row_words, int blk, int eta) {
  constexpr int per = 16 / B;
  const int pi = 2 * blk + eta;
  const uint32_t W = row_words[pi / per];
  const int off = (pi % per) * B;
  constexpr uint32_t m = (1u << B) - 1u;
  return (W >> off) & (m | (m << 16));
}

// Run-time part description of a b-bit code, indexed by log2 of the width (8/4/2/1):
// has[lw] says whether the width-2^lw part exists, lo[lw] its lowest code bit.
struct Parts {
  bool has[4];
  int lo[4];
};
__device__ __forceinline__ Parts parts_of(int b) {
  Parts P;
  int lo = 0;
#pragma unroll
  for (int lw = 3; lw >= 0; --lw) {
    P.has[lw] = (b >> lw) & 1;
    P.lo[lw] = lo;
    if (P.has[lw]) lo += 1 << lw;
  }
  return P;
}

// Generic widths at run-time block index (parts of width 8/4/2/1, assembled at e = 0).
__device__ __forceinline__ uint32_t pair_gen_rt(const uint32_t* page, int r, int row, int owner, bool is_k,
                                                const Parts& P, int blk, int eta) {
  uint32_t v = 0;
  const int pi = 2 * blk + eta;
#pragma unroll
  for (int lw = 3; lw >= 0; --lw) {
    if (P.has[lw]) {
      const int wd = 1 << lw;
      const uint32_t* plane = page + 4 * r * P.lo[lw];
      const int row_words = (is_k ? 8 : 4) * wd;
      const uint32_t W = plane[row * row_words + owner * wd + pi / (16 / wd)];
      const int off = (pi % (16 / wd)) * wd;
      const uint32_t m = (1u << wd) - 1u;
      v |= ((W >> off) & (m | (m << 16))) << P.lo[lw];
    }
  }
  return v;
}

template <int BK>
__device__ __forceinline__ uint32_t k_pair(const uint32_t* pk, int rK, int row, int g, const Parts& P, int blk,
                                           int eta) {
  if constexpr (BK != 0) {
    return pair_rt<BK>(pk + row * 8 * BK + g * BK, blk, eta);
  } else {
    return pair_gen_rt(pk, rK, row, g, true, P, blk, eta);
  }
}

template <int BV>
__device__ __forceinline__ uint32_t v_pair(const uint32_t* pv, int rV, int row, int tq, const Parts& P, int blk,
                                           int eta) {
  if constexpr (BV != 0) {
    return pair_rt<BV>(pv + row * 4 * BV + tq * BV, blk, eta);
  } else {
    return pair_gen_rt(pv, rV, row, tq, false, P, blk, eta);
  }
}

__device__ __forceinline__ uint32_t split_hi_lo(float x0, float x1, uint32_t& lo) {
  const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
  const __half l0 = __float2half_rn(x0 - __half2float(h0)), l1 = __float2half_rn(x1 - __half2float(h1));
  lo = static_cast<uint32_t>(__half_as_ushort(l0)) | (static_cast<uint32_t>(__half_as_ushort(l1)) << 16);
  return static_cast<uint32_t>(__half_as_ushort(h0)) | (static_cast<uint32_t>(__half_as_ushort(h1)) << 16);
}

// Per-warp state.  Lane (g, t) holds, for its query head g of the group, the query
// coordinates k(ks, m) = 16 ks + 2t + (m & 1) + 8 (m >> 1), ks < 8 (the B fragments of the
// score MMA); coordinate pairs (i, i + 64) are (ks, m) and (ks + 4, m).
struct RopeWS {
  float qq[8][4];     // q of head g (scaled by 2^-Eq[g]) rotated back to the current block's start
  float alpha[2], m_run[2], lsum[2];
  float z[kNT][4];
};

template <int BK, int BV>
__device__ __forceinline__ void rope_block(RopeWS& w, const RopeSmem& sm, const uint32_t* pk, const uint32_t* pv,
                                           const uint32_t* mrec, int rK, int rV, int nks, int nmt,
                                           const Parts& PK, const Parts& PV, int blk, int tok0, int seq_len,
                                           int g, int tq, float mV, uint32_t cmV) {
  // ---- K-hat block (16 tokens x 128 dims): acc[nt] rows g, g + 8, columns 8 nt + 2t, + 1
  float acc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
  for (int ks = 0; ks < nks; ++ks) {
    const int r0 = 8 * ks + tq, r1 = r0 + 4;
    const uint32_t A0 = k_pair<BK>(pk, rK, r0, g, PK, blk, 0);
    const uint32_t A1 = k_pair<BK>(pk, rK, r0, g, PK, blk, 1);
    const uint32_t A2 = k_pair<BK>(pk, rK, r1, g, PK, blk, 0);
    const uint32_t A3 = k_pair<BK>(pk, rK, r1, g, PK, blk, 1);
    const uint4* fr = reinterpret_cast<const uint4*>(mrec) + static_cast<size_t>(ks) * 16 * 32 + (g * 4 + tq);
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const uint4 b = __ldg(fr + nt * 32);
      mma_16816(acc[nt], A0, A1, A2, A3, b.x, b.y);
      mma_16816(acc[nt], A0, A1, A2, A3, b.z, b.w);
    }
  }
  // ---- centring (codes are c * 2^-24) and the rotation of row rho by rho w_i
  const int rho0 = g, rho1 = g + 8;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int i = 8 * nt + 2 * tq + c;
      const float s1 = sm.msum[i], s2 = sm.msum[i + 64];
      const float a1 = fmaf(acc[nt][c], 16777216.0f, -s1), a2 = fmaf(acc[nt + 8][c], 16777216.0f, -s2);
      const float b1 = fmaf(acc[nt][2 + c], 16777216.0f, -s1), b2 = fmaf(acc[nt + 8][2 + c], 16777216.0f, -s2);
      const float2 r0 = sm.rot1[rho0][i], r1 = sm.rot1[rho1][i];
      acc[nt][c] = fmaf(a1, r0.x, -a2 * r0.y);
      acc[nt + 8][c] = fmaf(a2, r0.x, a1 * r0.y);
      acc[nt][2 + c] = fmaf(b1, r1.x, -b2 * r1.y);
      acc[nt + 8][2 + c] = fmaf(b2, r1.x, b1 * r1.y);
    }
  }
  // ---- scores: rotated K-hat (fp16 hi + lo) against the query rotated back (hi + lo)
  float sc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int kd = 0; kd < 8; ++kd) {
    uint32_t al0, al1, al2, al3, bl0, bl1;
    const uint32_t ah0 = split_hi_lo(acc[2 * kd][0], acc[2 * kd][1], al0);
    const uint32_t ah1 = split_hi_lo(acc[2 * kd][2], acc[2 * kd][3], al1);
    const uint32_t ah2 = split_hi_lo(acc[2 * kd + 1][0], acc[2 * kd + 1][1], al2);
    const uint32_t ah3 = split_hi_lo(acc[2 * kd + 1][2], acc[2 * kd + 1][3], al3);
    const uint32_t bh0 = split_hi_lo(w.qq[kd][0], w.qq[kd][1], bl0);
    const uint32_t bh1 = split_hi_lo(w.qq[kd][2], w.qq[kd][3], bl1);
    mma_16816(sc, ah0, ah1, ah2, ah3, bh0, bh1);
    mma_16816(sc, al0, al1, al2, al3, bh0, bh1);
    mma_16816(sc, ah0, ah1, ah2, ah3, bl0, bl1);
  }
  // ---- online softmax (log2 domain; P scaled by 2^7 for the value MMA), lazy rescale
  float x[4];
  x[0] = fmaf(w.alpha[0], sc[0], 7.0f - (w.m_run[0] == -INFINITY ? 0.0f : w.m_run[0]));
  x[1] = fmaf(w.alpha[1], sc[1], 7.0f - (w.m_run[1] == -INFINITY ? 0.0f : w.m_run[1]));
  x[2] = fmaf(w.alpha[0], sc[2], 7.0f - (w.m_run[0] == -INFINITY ? 0.0f : w.m_run[0]));
  x[3] = fmaf(w.alpha[1], sc[3], 7.0f - (w.m_run[1] == -INFINITY ? 0.0f : w.m_run[1]));
  {
    const int t0 = tok0 + 16 * blk + g;
    if (t0 >= seq_len) x[0] = x[1] = -INFINITY;
    if (t0 + 8 >= seq_len) x[2] = x[3] = -INFINITY;
  }
  bool grow = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3])) > kLazy + 7.0f;
  grow |= w.m_run[0] == -INFINITY || w.m_run[1] == -INFINITY;
  if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float v = fmaxf(x[c], x[2 + c]) - 7.0f;
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
      const float old = w.m_run[c];
      float shift = 0.0f;
      if (v == -INFINITY) {
      } else if (old == -INFINITY) {
        w.m_run[c] = v;
        shift = v;
      } else if (v > 0.0f) {
        w.m_run[c] = old + v;
        shift = v;
        const float resc = ex2(-v);
#pragma unroll
        for (int mt = 0; mt < kNT; ++mt) {
          w.z[mt][c] *= resc;
          w.z[mt][2 + c] *= resc;
        }
        w.lsum[c] *= resc;
      }
      x[c] -= shift;
      x[2 + c] -= shift;
    }
  }
  const uint32_t P0 = pack_half2(ex2(x[0]), ex2(x[1]));
  const uint32_t P1 = pack_half2(ex2(x[2]), ex2(x[3]));
  {
    const float2 f0 = half2_to_float2(P0), f1 = half2_to_float2(P1);
    w.lsum[0] += fmaf(f0.x, 0.0078125f, f1.x * 0.0078125f);
    w.lsum[1] += fmaf(f0.y, 0.0078125f, f1.y * 0.0078125f);
  }
  uint32_t bp[2];
  bp[0] = movmatrix_trans(P0);
  bp[1] = movmatrix_trans(P1);
  // ---- values: z[j][head] += sum_tok (c_V - floor(m_V)) P (raw values: the fp16 as stored)
#pragma unroll
  for (int mt = 0; mt < kNT; ++mt) {
    if (mt >= nmt) break;
    uint32_t A0, A1, A2, A3;
    const int j0 = 16 * mt + g, j1 = j0 + 8;
    if constexpr (BV == kRawBits) {
      const int rsw = tq ^ (g << 2);
      const uint32_t* row0 = pv + j0 * (kPage / 2);
      const int c0 = (8 * blk) ^ rsw, c1 = (8 * blk + 4) ^ rsw;
      A0 = row0[c0];
      A1 = row0[8 * (kPage / 2) + c0];
      A2 = row0[c1];
      A3 = row0[8 * (kPage / 2) + c1];
    } else {
      A0 = hsub2_bits(v_pair<BV>(pv, rV, j0, tq, PV, blk, 0), cmV);
      A1 = hsub2_bits(v_pair<BV>(pv, rV, j1, tq, PV, blk, 0), cmV);
      A2 = hsub2_bits(v_pair<BV>(pv, rV, j0, tq, PV, blk, 1), cmV);
      A3 = hsub2_bits(v_pair<BV>(pv, rV, j1, tq, PV, blk, 1), cmV);
    }
    mma_16816(w.z[mt], A0, A1, A2, A3, bp[0], bp[1]);
  }
  (void)mV;
}

// Rotates the lane's query coordinates back, in place, by the angles (c, s) of each pair:
// (x_i, x_{i+64}) -> (x_i c + x_{i+64} s, x_{i+64} c - x_i s).
__device__ __forceinline__ void rotate_back(float (&x)[8][4], const float2* cs, int tq) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int i = 16 * ks + 2 * tq + (m & 1) + 8 * (m >> 1);
      const float2 a = cs[i];
      const float x1 = x[ks][m], x2 = x[ks + 4][m];
      x[ks][m] = fmaf(x1, a.x, x2 * a.y);
      x[ks + 4][m] = fmaf(x2, a.x, -x1 * a.y);
    }
  }
}

template <int BK, int BV>
__global__ void __launch_bounds__(kThreads, 2) decode_rope_kernel(const __grid_constant__ RopeArgs ra) {
  const DecodeArgs& a = ra.d;
  extern __shared__ __align__(128) unsigned char smem[];
  RopeSmem& sm = *reinterpret_cast<RopeSmem*>(smem);
  constexpr size_t kBar = (sizeof(RopeSmem) + 15) / 16 * 16;
  constexpr size_t kRing = ((kBar + 8 * kWarps * 8 + 127) / 128) * 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBar);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  int hi = 0;
  while (hi + 1 < a.n_heads && static_cast<int>(blockIdx.x) >= a.split_prefix[hi + 1]) ++hi;
  const int split = blockIdx.x - a.split_prefix[hi];
  const int n_split = a.split_prefix[hi + 1] - a.split_prefix[hi];
  const int hg = blockIdx.y;
  const int s = blockIdx.z;
  const int h = a.heads[hi];
  const int uK = (a.layer * a.H + h) * 2, uV = uK + 1;
  const UnitDesc dK = a.units[uK], dV = a.units[uV];
  const int rK = dK.r, rV = dV.r;
  const int nks = (rK + 15) >> 4, nmt = (rV + 15) >> 4;
  const int Hq = a.H * a.G;
  const int g0 = hg * 8, ng = min(8, a.G - g0);
  const uint32_t* mrec = dK.Mrec;  // read through L1: every CTA of the head on an SM shares it
  unsigned char* stages = smem + kRing;
  // constant plan data and tables before the wait: the rotation tables, the centring sums,
  // L2 prefetches of the reconstruction fragments of M_K and of M_V
  if (lane == 0)
    for (int i = 0; i < a.n_stage; ++i) mbar_init(&bars[warp * 8 + i], 1);
  if (tid == 0) {
    prefetch_l2(dK.Mrec, static_cast<uint32_t>(nks) * 16 * 32 * 16);
    if (dV.b != kRawBits) prefetch_l2(dV.M, static_cast<uint32_t>(rV) * kD * 4);
  }
  for (int i = tid; i < 16 * 64; i += kThreads) sm.rot1[i >> 6][i & 63] = ra.rot1[i >> 6][i & 63];
  if (tid < 64) sm.rot16[tid] = ra.rot16[tid];
  {
    const float mK = 0.5f * static_cast<float>((1 << dK.b) - 1);
    if (tid < 128) sm.msum[tid] = mK * dK.Msum[tid];
  }
  if (a.wait_first) griddep_wait();
  griddep_launch_dependents();

  int seq_len = a.seq_lens[s];
  if (seq_len < 0 || seq_len > a.max_pages * kPage) {
    if (tid == 0 && a.status) atomicOr(a.status, KVTC_STATUS_BAD_POS);
    seq_len = seq_len < 0 ? 0 : a.max_pages * kPage;
  }
  const int n_pages = (seq_len + kPage - 1) / kPage;
  const int n_workers = n_split * kWarps;
  const int worker = split * kWarps + warp;
  const int p_begin = static_cast<int>(static_cast<long long>(worker) * n_pages / n_workers);
  const int n_my = static_cast<int>(static_cast<long long>(worker + 1) * n_pages / n_workers) - p_begin;
  const int32_t* bt = a.block_table + static_cast<size_t>(s) * a.max_pages;
  fence_mbar_init();
  __syncwarp();

  const uint32_t bytesK = static_cast<uint32_t>(dK.page_bytes), bytesV = static_cast<uint32_t>(dV.page_bytes);
  const char* poolK = a.pool + a.pages_per_unit * dK.prefix;
  const char* poolV = a.pool + a.pages_per_unit * dV.prefix;
  unsigned char* const warp_stages = stages + static_cast<size_t>(warp) * a.n_stage * a.stage_bytes;
  auto stage_ptr = [&](int slot) { return warp_stages + static_cast<size_t>(slot) * a.stage_bytes; };
  int pid_win = -1, pid_base = -1;
  auto pid_of = [&](int i) {
    const int base = i & ~31;
    if (base != pid_base) {
      const int ii = base + lane;
      pid_win = ii < n_my ? bt[p_begin + ii] : -1;
      pid_base = base;
    }
    return __shfl_sync(0xffffffffu, pid_win, i & 31);
  };
  uint32_t vmask = 0;
  auto issue = [&](int slot, int pid) {
    uint64_t* bar = &bars[warp * 8 + slot];
    if (pid < 0 || static_cast<uint64_t>(pid) >= a.pages_per_unit) {
      vmask &= ~(1u << slot);
      mbar_arrive(bar);
      return;
    }
    vmask |= 1u << slot;
    unsigned char* st = stage_ptr(slot);
    mbar_arrive_expect_tx(bar, bytesK + bytesV);
    bulk_copy_g2s(st, poolK + static_cast<uint64_t>(pid) * bytesK, bytesK, bar);
    bulk_copy_g2s(st + bytesK, poolV + static_cast<uint64_t>(pid) * bytesV, bytesV, bar);
  };
  const int n_first = min(a.n_stage, n_my);
  for (int i = 0; i < n_first; ++i) {
    const int pid = pid_of(i);
    if (lane == 0) issue(i, pid);
  }

  // ---- the query: per head the fp16 scaling exponent (warp w: heads 2w, 2w + 1), then
  // each lane its head's coordinates (scaled)
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int gg = 2 * warp + hh;
    float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (gg < ng) {
      const size_t off = (static_cast<size_t>(s) * Hq + h * a.G + g0 + gg) * kD + 4 * lane;
      if (a.q_bf16) {
        const uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.q) + off);
        v = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                        __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u));
      } else {
        v = *reinterpret_cast<const float4*>(static_cast<const float*>(a.q) + off);
      }
    }
    float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) sm.Eq[gg] = (amax > 0.0f && amax < INFINITY) ? ilogbf(amax) - 14 : 0;
  }
  __syncthreads();
  // the group's queries into shared memory, scaled per head (rows past the group zero)
  for (int i = tid; i < 8 * 128; i += kThreads) {
    const int n = i >> 7, k = i & 127;
    float x = 0.0f;
    if (n < ng) {
      const size_t off = (static_cast<size_t>(s) * Hq + h * a.G + g0 + n) * kD + k;
      x = a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[off]) : static_cast<const float*>(a.q)[off];
    }
    sm.qs[n][k] = x * ldexpf(1.0f, -sm.Eq[n]);
  }
  __syncthreads();
  RopeWS w;
  {
    const float lb = a.scale * dK.delta * kLog2e;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int n = 2 * tq + c;
      w.alpha[c] = n < ng ? lb * ldexpf(1.0f, sm.Eq[n]) : 0.0f;
      w.m_run[c] = -INFINITY;
      w.lsum[c] = 0.0f;
    }
#pragma unroll
    for (int mt = 0; mt < kNT; ++mt) w.z[mt][0] = w.z[mt][1] = w.z[mt][2] = w.z[mt][3] = 0.0f;
  }
  const Parts PK = parts_of(dK.b), PV = parts_of(dV.b);
  const float mV = dV.b == kRawBits ? 0.0f : 0.5f;
  const uint32_t cmV = dV.b == kRawBits ? 0u : ((1u << (dV.b - 1)) - 1u) * 0x10001u;
  bool dead = false;
  int next_issue = n_first;
  int slot = 0;
  uint32_t phase = 0;
  for (int i = 0; i < n_my; ++i) {
    const int p = p_begin + i;
    const bool valid = (__shfl_sync(0xffffffffu, vmask, 0) >> slot) & 1u;
    const bool got = mbar_wait_bounded_warp(&bars[warp * 8 + slot], phase);
    if (!got || dead) {
      if (!got && lane == 0 && a.status) atomicOr(a.status, KVTC_STATUS_TIMEOUT);
      dead = true;
      int s2 = slot;
      uint32_t ph2 = phase;
      for (int i2 = i + 1; i2 < next_issue; ++i2) {
        if (++s2 == a.n_stage) {
          s2 = 0;
          ph2 ^= 1u;
        }
        (void)mbar_wait_bounded_warp(&bars[warp * 8 + s2], ph2);
      }
      break;
    }
    if (valid) {
      const unsigned char* st = stage_ptr(slot);
      const uint32_t* pk = reinterpret_cast<const uint32_t*>(st);
      const uint32_t* pv = reinterpret_cast<const uint32_t*>(st + bytesK);
      const int tok0 = p * kPage;
      // the page part of the angle, t0 w_i, reduced mod 2 pi in fp64 (lane: i = lane, lane + 32)
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int i = lane + 32 * k;
        const double th = static_cast<double>(tok0) * ra.omega[i];
        const double n = rint(th * 0.15915494309189535);
        const double red = fma(-n, 1.2246467991473532e-16, fma(-n, 6.283185307179586, th));
        float sn, cs;
        sincosf(static_cast<float>(red), &sn, &cs);
        sm.page[warp][i] = make_float2(cs, sn);
      }
      __syncwarp();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
#pragma unroll
        for (int m = 0; m < 4; ++m) w.qq[ks][m] = sm.qs[g][16 * ks + 2 * tq + (m & 1) + 8 * (m >> 1)];
      rotate_back(w.qq, sm.page[warp], tq);
      const int nblk = min(8, (seq_len - tok0 + 15) >> 4);
      for (int blk = 0; blk < nblk; ++blk) {
        if (blk > 0) rotate_back(w.qq, sm.rot16, tq);
        rope_block<BK, BV>(w, sm, pk, pv, mrec, rK, rV, nks, nmt, PK, PV, blk, tok0, seq_len, g, tq, mV, cmV);
      }
    } else if (lane == 0 && a.status) {
      atomicOr(a.status, KVTC_STATUS_BAD_PAGE);
    }
    __syncwarp();
    if (next_issue < n_my && next_issue == i + a.n_stage) {
      const int npid = pid_of(next_issue);
      if (lane == 0) issue(slot, npid);
      ++next_issue;
    }
    __syncwarp();
    if (++slot == a.n_stage) {
      slot = 0;
      phase ^= 1u;
    }
  }

  // ---- l per head column, centring, and the CTA merge (as the split decode) ----
  float l_out[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    float l = w.lsum[c];
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    l_out[c] = l;
    const float dl = mV * ldexpf(l, -17);
#pragma unroll
    for (int mt = 0; mt < kNT; ++mt) {
      w.z[mt][c] -= dl;
      w.z[mt][2 + c] -= dl;
    }
  }
  float* mb = reinterpret_cast<float*>(stages);
  __syncthreads();
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int n = 2 * tq + c;
    if (n < ng) {
      float* dst = mb + (warp * 8 + n) * kPartStride;
      if (g == 0) {
        dst[0] = dead ? -INFINITY : w.m_run[c];
        dst[1] = dead ? 0.0f : l_out[c];
      }
#pragma unroll
      for (int mt = 0; mt < kNT; ++mt) {
        if (mt < nmt) {
          const int j0 = 16 * mt + g, j1 = j0 + 8;
          if (j0 < rV) dst[4 + j0] = dead ? 0.0f : w.z[mt][c];
          if (j1 < rV) dst[4 + j1] = dead ? 0.0f : w.z[mt][2 + c];
        }
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < ng * (rV + 2); idx += kThreads) {
    const int n = idx / (rV + 2), e = idx - n * (rV + 2);
    float mw[kWarps], M = -INFINITY;
#pragma unroll
    for (int q = 0; q < kWarps; ++q) {
      mw[q] = mb[(q * 8 + n) * kPartStride];
      M = fmaxf(M, mw[q]);
    }
    float acc = 0.0f;
    if (M != -INFINITY) {
      const int src = e == 0 ? 1 : 4 + (e - 1);
      if (e <= rV) {
#pragma unroll
        for (int q = 0; q < kWarps; ++q)
          if (mw[q] != -INFINITY) acc = fmaf(ex2(mw[q] - M), mb[(q * 8 + n) * kPartStride + src], acc);
      }
    }
    float* dst = a.ws + ((static_cast<size_t>(s) * Hq + h * a.G + g0 + n) * a.part_stride + split) * kPartStride;
    if (e == 0) {
      dst[0] = M;
      dst[1] = acc;
    } else if (e <= rV) {
      dst[4 + (e - 1)] = acc;
    }
  }
  __threadfence();
  __syncthreads();
  int* ticket = a.tickets + ((static_cast<size_t>(s) * a.H + h) * a.n_hg + hg) * kTicketInts;
  if (tid == 0) sm.last = atomicAdd(ticket, 1) == n_split - 1;
  __syncthreads();
  if (sm.last) {
    __threadfence();
    merge_project(a, dV, mb, s, h * a.G + g0, ng, 0, 1, n_split, warp, lane, tid);
    if (tid == 0) atomicExch(ticket, 0);
  }
  if (!a.wait_first) griddep_wait();
}

using RopeFn = void (*)(const RopeArgs);

RopeFn rope_fn(int bK, int bV) {
  const bool k2 = bK == 2;
  if (bV == kRawBits) return k2 ? decode_rope_kernel<2, kRawBits> : decode_rope_kernel<0, kRawBits>;
  if (bV == 2) return k2 ? decode_rope_kernel<2, 2> : decode_rope_kernel<0, 2>;
  return k2 ? decode_rope_kernel<2, 0> : decode_rope_kernel<0, 0>;
}

constexpr size_t kSmemPerSM = 233472;
constexpr size_t kReadSlack = 2048;

size_t head_bytes() {
  const size_t bar = (sizeof(RopeSmem) + 15) / 16 * 16;
  return ((bar + 8 * kWarps * 8 + 127) / 128) * 128;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_rope(void (*fn)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, std::forward<Args>(args)...);
}

}  // namespace rope
}  // namespace dec

// The pre-RoPE launches of every layer: heads grouped by kernel variant, the stage size
// of each group and the stage count and occupancy that fit (two CTAs per SM, the register
// limit, when the ring allows it).  A group whose page does not fit in shared memory is
// kept with no kernel; a pre-RoPE decode of its layer then fails with EINVAL (the plan
// stays usable for every other call).  Sets each variant's shared-memory attribute once.
kvtc_status prepare_rope(kvtc_plan* plan) {
  using namespace dec;
  using namespace dec::rope;
  plan->rope_groups.assign(plan->L, {});
  const size_t merge_bytes = std::max<size_t>(static_cast<size_t>(kWarps) * 8 * kPartStride, kMergeFloats) * sizeof(float);
  for (int layer = 0; layer < plan->L; ++layer) {
    std::vector<RopeGroup>& gs = plan->rope_groups[layer];
    for (int h = 0; h < plan->H; ++h) {
      const int uK = (layer * plan->H + h) * 2;
      const void* fn = reinterpret_cast<const void*>(rope_fn(plan->b[uK], plan->b[uK + 1]));
      auto it = std::find_if(gs.begin(), gs.end(), [&](const RopeGroup& x) { return x.fn == fn; });
      if (it == gs.end()) {
        gs.emplace_back();
        it = gs.end() - 1;
        it->fn = fn;
      }
      it->heads.push_back(h);
      const uint32_t pb = static_cast<uint32_t>(16 * (plan->r[uK] * plan->b[uK] + plan->r[uK + 1] * plan->b[uK + 1]));
      it->stage_bytes = std::max(it->stage_bytes, (pb + 127u) / 128u * 128u);
    }
    for (RopeGroup& gr : gs) {
      int n_stage = kRopeStages;
      size_t smem = 0;
      for (; n_stage >= 1; --n_stage) {
        smem = head_bytes() + std::max<size_t>(static_cast<size_t>(kWarps) * n_stage * gr.stage_bytes, merge_bytes) +
               kReadSlack;
        // two CTAs per SM (the register limit) when the ring allows it
        if (smem <= kSmemPerSM / 2 - 1024 || (n_stage == 1 && smem <= kSmemPerSM - 1024)) break;
      }
      if (n_stage < 1) {
        gr.fn = nullptr;
        continue;
      }
      gr.n_stage = n_stage;
      gr.smem = smem;
      // the attribute is per kernel (shared with other plans): the largest size
      cudaError_t e = cudaFuncSetAttribute(gr.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kSmemPerSM - 1024));
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (rope decode)");
      int occ = 1;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gr.fn, kThreads, smem) != cudaSuccess || occ < 1) occ = 1;
      gr.per_sm = occ;
    }
  }
  return KVTC_OK;
}
}  // namespace kvtc

using namespace kvtc;
using namespace kvtc::dec;
using namespace kvtc::dec::rope;

extern "C" kvtc_status kvtc_decode_attention_rope(const kvtc_plan* plan, const kvtc_cache* cache, int layer,
                                                  const void* q, kvtc_dtype q_dtype, const int32_t* seq_lens,
                                                  int max_seq_len, float softmax_scale, double rope_base, void* out,
                                                  kvtc_dtype out_dtype, void* workspace, uint64_t workspace_bytes,
                                                  void* stream) {
  kvtc_status st = check_uploaded(plan);
  if (st != KVTC_OK) return st;
  if (!cache || !cache->pool || !cache->block_table) return fail(KVTC_EINVAL, "cache is incomplete");
  if (layer < 0 || layer >= plan->L) return fail(KVTC_EINVAL, "layer out of range");
  if (!q || !seq_lens || !out || !workspace) return fail(KVTC_EINVAL, "null device pointer");
  if ((q_dtype != KVTC_F32 && q_dtype != KVTC_BF16) || (out_dtype != KVTC_F32 && out_dtype != KVTC_BF16))
    return fail(KVTC_EINVAL, "dtype must be F32 or BF16");
  if (cache->n_seq < 1 || cache->max_pages < 1 || max_seq_len < 0) return fail(KVTC_EINVAL, "bad sizes");
  if (max_seq_len > cache->max_pages * kPage) return fail(KVTC_EINVAL, "max_seq_len exceeds the block table");
  if (reinterpret_cast<uintptr_t>(cache->pool) & 15) return fail(KVTC_EINVAL, "pool must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(workspace) & 15) return fail(KVTC_EINVAL, "workspace must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(q) & 15) return fail(KVTC_EINVAL, "q must be 16-byte aligned");
  if (!(rope_base >= 0.0) || !std::isfinite(rope_base) || (rope_base > 0.0 && rope_base <= 1.0))
    return fail(KVTC_EINVAL, "rope_base must be 0 (500000) or greater than 1");
  const double base = rope_base > 0.0 ? rope_base : 500000.0;
  const int n_seq = cache->n_seq;
  const uint64_t need = kvtc_decode_workspace_bytes(plan, n_seq, max_seq_len);
  if (workspace_bytes < need) return fail(KVTC_ECAPACITY, "decode workspace too small");
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(plan->d));
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int n_hg = (plan->G + 7) / 8;
  const int n_pages = std::max(1, (max_seq_len + kPage - 1) / kPage);
  const int cap = std::max(1, std::min(kMaxSplits, (n_pages + 7) / 8));
  RopeArgs ra;
  for (int i = 0; i < 64; ++i) {
    ra.omega[i] = std::pow(base, -2.0 * i / 128.0);
    for (int rho = 0; rho < 16; ++rho)
      ra.rot1[rho][i] = make_float2(static_cast<float>(std::cos(rho * ra.omega[i])),
                                    static_cast<float>(std::sin(rho * ra.omega[i])));
    ra.rot16[i] = make_float2(static_cast<float>(std::cos(16.0 * ra.omega[i])),
                              static_cast<float>(std::sin(16.0 * ra.omega[i])));
  }
  DecodeArgs& a = ra.d;
  a.units = plan->d_units;
  a.layer = layer;
  a.H = plan->H;
  a.G = plan->G;
  a.n_hg = n_hg;
  a.part_stride = cap;
  a.q = q;
  a.q_bf16 = q_dtype == KVTC_BF16;
  a.out = out;
  a.out_bf16 = out_dtype == KVTC_BF16;
  a.seq_lens = seq_lens;
  a.n_seq = n_seq;
  a.pool = static_cast<const char*>(cache->pool);
  a.pages_per_unit = cache->pages_per_unit;
  a.block_table = cache->block_table;
  a.max_pages = cache->max_pages;
  a.part_pages = std::max(1, (max_seq_len + kPage - 1) / kPage);  // (this kernel splits by seq_len)
  a.status = cache->status;
  a.scale = scale;
  a.tickets = static_cast<int*>(workspace);
  // the workspace layout of kvtc_decode_attention: tickets [n_seq][H][n_hg][kTicketInts]
  // (this kernel counts arrivals in the first), then the partials
  const size_t tb = (static_cast<size_t>(n_seq) * plan->H * n_hg * kTicketInts * sizeof(int) + 255) / 256 * 256;
  a.ws = reinterpret_cast<float*>(static_cast<char*>(workspace) + tb);
  // one launch per (b_K, b_V) variant class (decided at plan upload); every KV head of
  // the layer in one of them
  bool first = true;
  for (const RopeGroup& gr : plan->rope_groups[layer]) {
    if (!gr.fn) return fail(KVTC_EINVAL, "a page of this plan does not fit in shared memory");
    const int n_stage = gr.n_stage;
    const size_t smem = gr.smem;
    const int occ = gr.per_sm;
    const int nh = static_cast<int>(gr.heads.size());
    if (nh > kMaxHeadsPerLaunch) return fail(KVTC_EINVAL, "at most 64 KV heads per layer");
    const int wave = std::max(nh, static_cast<int>(static_cast<double>(occ) * plan->sm_count * nh / plan->H));
    const int per_head = std::max(1, std::min(cap, wave / std::max(1, nh * n_hg * n_seq)));
    a.n_heads = nh;
    a.split_prefix[0] = 0;
    for (int i = 0; i < nh; ++i) {
      a.heads[i] = gr.heads[i];
      a.split_prefix[i + 1] = a.split_prefix[i] + per_head;
    }
    a.wait_first = first ? 1 : 0;
    a.n_stage = n_stage;
    a.stage_bytes = gr.stage_bytes;
    dim3 grid(a.split_prefix[nh], n_hg, n_seq);
    const cudaError_t e = launch_pdl_rope(reinterpret_cast<RopeFn>(const_cast<void*>(gr.fn)), grid, dim3(kThreads), smem, cs, ra);
    if (e != cudaSuccess) return cuda_fail(e, "rope decode launch");
    first = false;
  }
  return KVTC_OK;
}
