// Decode split kernel (templates).  Included by decode.cu and the per-variant
// instantiation units decode_v*.cu.
//
// One launch per layer and (b_K, b_V) group.  CTA = (context split, KV head [, head group
// of 8], sequence); four warps, each streaming its own pages through a ring of
// cp.async.bulk + mbarrier stages.  The CTA
//   * forms q~ = M_K q for its query heads on the tensor cores (M_K as fp16 hi + lo
//     fragments from the plan, q scaled to fp16 by a power of two per head), and keeps the
//     B fragments of q^ = q~ 2^-E (fp16 hi + lo) in shared memory for all four warps;
//   * per 16-token block scores its G (<= 8) query heads with m16n8k16 MMAs whose A operand
//     comes straight from the packed words: one AND leaves each code in the low mantissa
//     bits of an fp16 half, the exact subnormal c * 2^(e-24), e the field's bit offset
//     (undone in fp32), and widths 3, 5, 6 and 7 add their one or two minor parts with a
//     shift and an AND-OR each; for G <= 4 (packed mode) head n's hi and lo parts sit in
//     columns 2n and 2n + 1 of one MMA, so each lane adds its own two columns and holds one
//     head's scores for two token rows;
//   * runs an online softmax whose rescale is lazy: it happens only when a score exceeds
//     the running max by more than 2^8 (a warp vote), so the common block costs one FFMA
//     and one ex2 per score;
//   * stores P in fp16 scaled by 2^(7-e) so that P * A = p * c * 2^-17 for any e, moves it
//     into the B fragment with movmatrix, and accumulates the value latents with MMAs
//     whose A operand again comes straight from the packed value words.  l = sum p is
//     accumulated from the same rounded P, so z - m_V * l cancels consistently: in packed
//     mode by one more MMA whose A operand is a constant row of ones, otherwise by one
//     extra A row of ones (when r_V is not a multiple of 16) or per-lane sums.
// The value codes enter their MMAs shifted by floor(m_V) (an exact fp16x2 subtraction),
// so the tensor core accumulates signed terms near the size of the result; the 0.5 l left
// over is folded into z after every page in packed mode (once at the end otherwise).
// 2- and 3-bit value codes in packed mode skip the shift and fold the whole m_V l per page.
// A page's eight 16-token blocks are processed together (their MMA chains interleave).
// The four warps' (m, l, z) meet in shared memory and each CTA writes one partial per
// query head; the last min(G, splits) CTAs to complete a (sequence, KV head, head group)
// (an atomic arrival counter in the workspace; from 16 splits up, else the last CTA
// alone) each take a share of its query heads:
// once every split has written its partial, they merge the partials with a log-sum-exp,
// dequantize (delta_V) and back-project o = M_V^T y on several SMs at once; the last of
// them re-arms the counters.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <type_traits>
#include <utility>

#include "kvtc_internal.h"
#include "ptx.cuh"

namespace kvtc {
namespace dec {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kNT = 8;                // 16-row tiles of a rank (r <= 128)
constexpr int kIL = 8;                // blocks processed together (one page)
constexpr int kMinBlocks = 3;         // resident CTAs per SM the registers are sized for
constexpr int kPartStride = 132;      // floats per partial: m, l, 2 pad, z[128]
constexpr int kMaxHeadsPerLaunch = 64;
constexpr int kMaxSplits = 128;       // context splits per KV head (bounds the merge scratch)
constexpr int kTicketInts = 2;        // per (sequence, KV head, head group): arrivals, merges done
constexpr uint32_t kSpinLimit = 1u << 20;  // polls (100 ns apart) before a merge share gives up
constexpr int kParMerge = 16;         // splits from which the merge is shared among the last CTAs
// floats of merge scratch a merging CTA needs ((m, l) of every split, y, the warps'
// back-projections)
constexpr int kMergeFloats = 16 * kMaxSplits + 8 * 128 + 4 * 8 * 128 + 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;         // log2 of the growth allowed before a rescale

struct DecodeArgs {
  const UnitDesc* units;
  int layer, H, G, n_hg;
  int heads[kMaxHeadsPerLaunch];        // KV heads handled by this launch
  int split_prefix[kMaxHeadsPerLaunch + 1];  // CTAs of head i: [prefix[i], prefix[i+1])
  int n_heads;
  int part_stride;                       // partial slots per query head in the workspace
  const void* q;      // [n_seq][Hq][128] of q dtype
  int q_bf16;
  void* out;          // [n_seq][Hq][128] of out dtype
  int out_bf16;
  int wait_first;     // 1: wait for the preceding grid before reading; 0: at exit (see decode.cu)
  const int32_t* seq_lens;
  int n_seq;
  const char* pool;
  uint64_t pages_per_unit;
  const int32_t* block_table;
  int max_pages;
  int part_pages;     // pages the split partition covers: ceil(max_seq_len / 128)
  int32_t* status;
  float scale;
  int n_stage;          // stages per warp of the widest head of the launch
  uint32_t stage_bytes;  // that head's stage (K + V page, 128-byte rounded)
  int* tickets;       // [n_seq][H][n_hg][kTicketInts] arrival counters (zero between calls)
  float* ws;          // partials [n_seq][Hq][part_stride][kPartStride]
};

// ------------------------------------------------------------------ code extraction
// A b-bit code is stored as parts of width 8, 4, 2 and 1 (its binary expansion, lowest
// code bits first, each part in its own plane of the page).  The widest part (the major
// part, holding the code's low bits) decides where a pair's field lands after one AND:
// at bit offset e of each fp16 half.  Widths 2, 4 and 8 are a major part alone; 3 = 2 + 1,
// 5 = 4 + 1, 6 = 4 + 2 and 7 = 4 + 2 + 1 add one or two minor parts, each moved to bit
// e + (its low code bit).  The code then occupies bits [e, e + b) with e + b <= 11, where
// an fp16 bit pattern x still has the value x 2^-24 (the subnormals and the first normal
// binade).
__host__ __device__ constexpr int major_w(int B) { return B == 3 ? 2 : ((B >= 5 && B <= 7) ? 4 : B); }
__host__ __device__ constexpr int n_minor(int B) { return (B == 3 || B == 5 || B == 6) ? 1 : (B == 7 ? 2 : 0); }
// width and low code bit of minor part i
__host__ __device__ constexpr int minor_w(int B, int i) { return (B == 6 || (B == 7 && i == 0)) ? 2 : 1; }
__host__ __device__ constexpr int minor_lo(int B, int i) { return B == 3 ? 2 : ((B == 7 && i == 1) ? 6 : 4); }

// bit position of pair (blk, eta)'s field in its word, for a part of width w
__host__ __device__ constexpr int pair_offset(int w, int blk, int eta) { return ((2 * blk + eta) % (16 / w)) * w; }

// bit offset e of the code inside each fp16 half after extraction
template <int B>
__host__ __device__ constexpr int e_of(int blk, int eta) {
  return major_w(B) == 2 ? 4 * (blk & 1) + 2 * eta : (major_w(B) == 4 ? 4 * eta : 0);
}
template <int B>
__host__ __device__ constexpr int n_e() {
  return major_w(B) == 2 ? 4 : (major_w(B) == 4 ? 2 : 1);
}
template <int B>
__host__ __device__ constexpr int e_idx(int blk, int eta) {
  return major_w(B) == 2 ? 2 * (blk & 1) + eta : (major_w(B) == 4 ? eta : 0);
}

// W >> 8 as mul.hi (the FMA pipe), leaving the ALU pipe to the field extraction.
__device__ __forceinline__ uint32_t shr8(uint32_t w) {
  uint32_t r;
  asm("mul.hi.u32 %0, %1, 16777216;\n" : "=r"(r) : "r"(w));
  return r;
}

// A-fragment pair of block BLK (eta = 0: the lane's first row, 1: its second) from word
// W, or from Wh = W >> 8 when the field sits at bit 8 or above.
template <int B, int BLK, int ETA>
__device__ __forceinline__ uint32_t fast_pair(uint32_t W, uint32_t Wh) {
  constexpr int off = pair_offset(B, BLK, ETA);
  constexpr uint32_t m = (1u << B) - 1u;
  if constexpr (off >= 8) {
    return Wh & ((m << (off - 8)) | (m << (off + 8)));
  } else {
    return W & ((m << off) | (m << (off + 16)));
  }
}

// fp16x2 a - b (round to nearest, subnormals kept).  On the code operands it is exact:
// both are multiples of the same 2^(e-24) and the difference stays below 2^(b+e-24).
__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// floor(m_V) = 2^(b-1) - 1 at the bit offset e of the value codes of block BLK, row
// eta, in both halves: the offset the value operand is shifted by before its MMA.
template <int B, int BLK, int ETA>
__host__ __device__ constexpr uint32_t centre_bits() {
  return ((((1u << (B - 1)) - 1u) << e_of<B>(BLK, ETA)) * 0x10001u);
}

// Minor part I of a width-B code for pair (BLK, ETA): its field in word Wm, moved to bit
// e + (its low code bit) of each half.
template <int B, int BLK, int ETA, int I>
__device__ __forceinline__ uint32_t minor_field(uint32_t Wm) {
  constexpr int wm = minor_w(B, I);
  constexpr int off = pair_offset(wm, BLK, ETA);
  constexpr int to = e_of<B>(BLK, ETA) + minor_lo(B, I);
  constexpr uint32_t m = (1u << wm) - 1u;
  constexpr uint32_t mask = (m << to) | (m << (to + 16));
  if constexpr (to >= off) {
    return (Wm << (to - off)) & mask;
  } else {
    return (Wm >> (off - to)) & mask;
  }
}

// A-fragment pair (BLK, ETA) of a width-B code: the major part's field from W (or from
// Wh = W >> 8), the minor parts' fields from Wm[0], Wm[1].
template <int B, int BLK, int ETA>
__device__ __forceinline__ uint32_t code_pair(uint32_t W, uint32_t Wh, const uint32_t (&Wm)[2]) {
  uint32_t v = fast_pair<major_w(B), BLK, ETA>(W, Wh);
  if constexpr (n_minor(B) >= 1) v |= minor_field<B, BLK, ETA, 0>(Wm[0]);
  if constexpr (n_minor(B) >= 2) v |= minor_field<B, BLK, ETA, 1>(Wm[1]);
  return v;
}

// Minor-part words of block BLK out of a group's words M[part][word] (group of blocks
// starting at B0).
template <int B, int B0, int BLK>
__device__ __forceinline__ void pick_minor(const uint32_t (&M)[2][2], uint32_t (&out)[2]) {
  out[0] = M[0][(BLK * minor_w(B, 0)) / 8 - (B0 * minor_w(B, 0)) / 8];
  out[1] = M[1][(BLK * minor_w(B, 1)) / 8 - (B0 * minor_w(B, 1)) / 8];
}

// ------------------------------------------------------------------ shared memory
struct SmemHead {
  float qt[8][128];        // q~ = M_K q (zero beyond the head group and beyond r_K)
  union {
    struct {
      uint16_t hi[8][136];  // q of the group as fp16, scaled by 2^-Eq (rows padded: no conflicts)
      uint16_t lo[8][136];  // the fp16 residual of an fp32 q
    } q16;
    uint32_t frag[2][8][2][32];  // B fragments of q^: [hi, lo][k-step][half][lane]
  } u;
  float Spart[8][8];       // [m-tile][head]: sum of q~ over the tile's 16 rows
  int E[8];                // power-of-two normalisation of q~ for fp16 (from a bound on |q~|)
  int Eq[8];               // power-of-two normalisation of q for fp16
  int ticket;              // this CTA's arrival position, then whether its merge share may run
};

// ------------------------------------------------------------------ per-warp state
template <int BK, int BV, bool PACK>
struct WS {
  const uint32_t* pk;  // K page in shared memory
  const uint32_t* pv;  // V page in shared memory
  const uint32_t* fr;  // this lane's B fragments of q^ in shared memory (hi; lo at + 512)
  int tok0, seq_len;
  bool partial;        // the page holds positions at or beyond seq_len
  int rK, rV, nks, nmt, g, tq;
  int kmo[2], vmo[2];  // word offsets of the minor parts' planes in a K / V page
  int ones_mt, ones_lr;  // m-tile / local row of the ones row (ones_mt < 0: none)
  uint32_t ones_m0, ones_m1;  // lane masks: this lane's A rows g / g+8 are the ones row
  float alpha[2], beta[2], m_run[2];
  float al[2][n_e<BK>()], nb[2][n_e<BV>()];
  // PACK: l accumulator (row 0, column 2n: l of head n, times 2^-17) and the constant A
  // fragments of its ones row by block parity (a0, a2; nonzero in lanes g == 0 only)
  float zl[4];
  uint32_t onesA[2][2];
  int rsw;  // uncompressed value pages: swizzle of this lane's word positions (tq ^ 4 g)
  // Centring of the value sums: the operands are c - floor(m_V), so z accumulates
  // p * (c - m_V + 0.5); the 0.5 l left over is folded into z after every page (packed
  // mode) or once at the end.  mV = 0.5 (m_V for unshifted 2- and 3-bit codes, 0 for raw
  // values); lfold = the part of l
  // (times 2^-17) already folded.
  float mV;
  float lfold;
  float z[kNT][4];
  float lcvt[2];  // l accumulated from the fp16 P when there is no ones row
};

// Score argument constants: x = al * acc + nb, with e undone in al (key side) and the P
// scale 2^(7 - e_V) folded into nb (value side).
template <int BK, int BV, bool PACK>
__device__ __forceinline__ void refresh_constants(WS<BK, BV, PACK>& w) {
  constexpr int NEK = n_e<BK>();
  constexpr int NEV = n_e<BV>();
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int i = 0; i < NEK; ++i) {
      const int e = major_w(BK) == 2 ? (i >> 1) * 4 + (i & 1) * 2 : (major_w(BK) == 4 ? 4 * i : 0);
      w.al[c][i] = w.alpha[c] * (1.0f / static_cast<float>(1 << e));
    }
    const float base = -(w.beta[c] + (w.m_run[c] == -INFINITY ? 0.0f : w.m_run[c])) + 7.0f;
#pragma unroll
    for (int i = 0; i < NEV; ++i) {
      const int e = major_w(BV) == 2 ? (i >> 1) * 4 + (i & 1) * 2 : (major_w(BV) == 4 ? 4 * i : 0);
      w.nb[c][i] = base - static_cast<float>(e);
    }
  }
}

// Score MMA(s) of one block for k-step ks: W0, W1 are the major-part words of rows r0, r1
// of this lane that hold the block's fields (Wh = W >> 8), M0, M1 their minor-part words.
template <int BK, int BV, bool PACK, int BLK>
__device__ __forceinline__ void k_block(const uint32_t (&bh)[2], const uint32_t (&bl)[2], uint32_t W0, uint32_t W0h,
                                        uint32_t W1, uint32_t W1h, const uint32_t (&M0)[2], const uint32_t (&M1)[2],
                                        float (&sc)[4], float (&sd)[4]) {
  const uint32_t A0 = code_pair<BK, BLK, 0>(W0, W0h, M0);
  const uint32_t A1 = code_pair<BK, BLK, 1>(W0, W0h, M0);
  const uint32_t A2 = code_pair<BK, BLK, 0>(W1, W1h, M1);
  const uint32_t A3 = code_pair<BK, BLK, 1>(W1, W1h, M1);
  mma_16816(sc, A0, A1, A2, A3, bh[0], bh[1]);
  if constexpr (!PACK) mma_16816(sd, A0, A1, A2, A3, bl[0], bl[1]);
}

// Score arguments of one block: x = s - m_run + 7 - e_V (log2 domain), -inf if masked.
// Returns whether the block asks for a rescale (a score past the running max by 2^kLazy).
template <int BK, int BV, bool PACK, int BLK>
__device__ __forceinline__ bool x_block(const WS<BK, BV, PACK>& w, const float (&sc)[4], const float (&sd)[4],
                                        float (&x)[4]) {
  constexpr int ik0 = e_idx<BK>(BLK, 0), ik1 = e_idx<BK>(BLK, 1);
  constexpr int iv0 = e_idx<BV>(BLK, 0), iv1 = e_idx<BV>(BLK, 1);
  constexpr int ev0 = e_of<BV>(BLK, 0), ev1 = e_of<BV>(BLK, 1);
  constexpr float lim0 = kLazy + 7.0f - ev0, lim1 = kLazy + 7.0f - ev1;
  if constexpr (PACK) {
    // columns 2 tq (hi) and 2 tq + 1 (lo) of head tq: x[0] row g, x[1] row g + 8
    x[0] = fmaf(w.al[0][ik0], sc[0] + sc[1], w.nb[0][iv0]);
    x[1] = fmaf(w.al[0][ik1], sc[2] + sc[3], w.nb[0][iv1]);
    if (w.partial) {  // warp-uniform: only the last page of a sequence
      const int t0 = w.tok0 + 16 * BLK + w.g;
      if (t0 >= w.seq_len) x[0] = -INFINITY;
      if (t0 + 8 >= w.seq_len) x[1] = -INFINITY;
    }
    return x[0] > lim0 || x[1] > lim1;
  } else {
    float full[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) full[i] = sc[i] + sd[i];
    // rows: full[0..1] token tok0 + 16*BLK + g (eta 0), full[2..3] that + 8 (eta 1)
    x[0] = fmaf(w.al[0][ik0], full[0], w.nb[0][iv0]);
    x[1] = fmaf(w.al[1][ik0], full[1], w.nb[1][iv0]);
    x[2] = fmaf(w.al[0][ik1], full[2], w.nb[0][iv1]);
    x[3] = fmaf(w.al[1][ik1], full[3], w.nb[1][iv1]);
    if (w.partial) {  // warp-uniform: only the last page of a sequence
      const int t0 = w.tok0 + 16 * BLK + w.g, t1 = t0 + 8;
      if (t0 >= w.seq_len) x[0] = x[1] = -INFINITY;
      if (t1 >= w.seq_len) x[2] = x[3] = -INFINITY;
    }
    return fmaxf(x[0], x[1]) > lim0 || fmaxf(x[2], x[3]) > lim1;
  }
}

// Block maximum of s - m_run for head column c of one block (x with the e_V offset removed).
template <int BK, int BV, bool PACK, int BLK>
__device__ __forceinline__ float xmax_block(const WS<BK, BV, PACK>& w, const float (&x)[4], int c) {
  constexpr int ev0 = e_of<BV>(BLK, 0), ev1 = e_of<BV>(BLK, 1);
  if constexpr (PACK) return fmaxf(x[0] - (7.0f - ev0), x[1] - (7.0f - ev1));
  return fmaxf(x[c] - (7.0f - ev0), x[2 + c] - (7.0f - ev1));
}

// P of one block in fp16 (already scaled by 2^(7 - e_V) through x), transposed into the
// B fragment of the value MMA; l from the rounded P when there is no ones row.
template <int BK, int BV, bool PACK, int BLK>
__device__ __forceinline__ void p_block(WS<BK, BV, PACK>& w, const float (&x)[4], uint32_t (&bp)[2]) {
  if constexpr (PACK) {
    // 8x8 tile X[row g][column 2 tq] = P(token g (+8), head tq), odd columns 0; its
    // transpose is the B fragment with head n in column 2n (odd columns zero)
    bp[0] = movmatrix_trans(pack_half2(ex2(x[0]), 0.0f));
    bp[1] = movmatrix_trans(pack_half2(ex2(x[1]), 0.0f));
    // l: the ones row times the same rounded P
    mma_16816(w.zl, w.onesA[BLK & 1][0], 0u, w.onesA[BLK & 1][1], 0u, bp[0], bp[1]);
    return;
  }
  const uint32_t P0 = pack_half2(ex2(x[0]), ex2(x[1]));
  const uint32_t P1 = pack_half2(ex2(x[2]), ex2(x[3]));
  if (w.ones_mt < 0) {
    constexpr int ev0 = e_of<BV>(BLK, 0), ev1 = e_of<BV>(BLK, 1);
    const float2 f0 = half2_to_float2(P0), f1 = half2_to_float2(P1);
    constexpr float u0 = 1.0f / static_cast<float>(1 << (7 - ev0)), u1 = 1.0f / static_cast<float>(1 << (7 - ev1));
    w.lcvt[0] += fmaf(f0.x, u0, f1.x * u1);
    w.lcvt[1] += fmaf(f0.y, u0, f1.y * u1);
  }
  bp[0] = movmatrix_trans(P0);
  bp[1] = movmatrix_trans(P1);
}

// Value codes centred by the per-page fold alone (no operand shift): 2- and 3-bit codes in
// packed mode.
template <int BV, bool PACK>
constexpr bool kFoldOnly = PACK && (BV == 2 || BV == 3);

// Value MMA of one block for m-tile mt (words as in k_block, of rows j0 and j0 + 8).
// Rows past r_V hold whatever follows the page in shared memory: their z rows are never
// read, except the ones row, whose A value is replaced whole.
template <int BK, int BV, bool PACK, int BLK>
__device__ __forceinline__ void v_block(const WS<BK, BV, PACK>& w, uint32_t W0, uint32_t W0h, uint32_t W1,
                                        uint32_t W1h, const uint32_t (&M0)[2], const uint32_t (&M1)[2], bool ones,
                                        const uint32_t (&bp)[2], float (&z)[4]) {
  uint32_t A0 = code_pair<BV, BLK, 0>(W0, W0h, M0);
  uint32_t A1 = code_pair<BV, BLK, 0>(W1, W1h, M1);
  uint32_t A2 = code_pair<BV, BLK, 1>(W0, W0h, M0);
  uint32_t A3 = code_pair<BV, BLK, 1>(W1, W1h, M1);
  // Signed operands: the codes enter the MMA as c - floor(m_V), so the tensor core sums
  // terms of both signs near the size of the result (an unsigned sum of p c, about
  // m_V l, loses the centred result in the accumulation).  The remaining 0.5 l is
  // folded into z separately.  2- and 3-bit values in packed mode skip the shift: m_V l
  // is folded into z after every page, which bounds the unsigned part of the sums by one
  // page's (2^b - 1) l (measured: the same errors against the oracle at every budget;
  // wider codes need the shift).
  if constexpr (!kFoldOnly<BV, PACK>) {
    constexpr uint32_t c0 = centre_bits<BV, BLK, 0>(), c1 = centre_bits<BV, BLK, 1>();
    A0 = hsub2_bits(A0, c0);
    A1 = hsub2_bits(A1, c0);
    A2 = hsub2_bits(A2, c1);
    A3 = hsub2_bits(A3, c1);
  }
  if (ones) {  // the ones row (row r_V) accumulates l: its A value is all ones
    constexpr int ev0 = e_of<BV>(BLK, 0), ev1 = e_of<BV>(BLK, 1);
    constexpr uint32_t one0 = (1u << ev0) | (1u << (ev0 + 16)), one1 = (1u << ev1) | (1u << (ev1 + 16));
    A0 = (A0 & ~w.ones_m0) | (one0 & w.ones_m0);
    A2 = (A2 & ~w.ones_m0) | (one1 & w.ones_m0);
    A1 = (A1 & ~w.ones_m1) | (one0 & w.ones_m1);
    A3 = (A3 & ~w.ones_m1) | (one1 & w.ones_m1);
  }
  mma_16816(z, A0, A1, A2, A3, bp[0], bp[1]);
}

// Value MMA of one block for an uncompressed value unit (keys-only plans).  Word of
// coordinate j and token pair k: j * 64 + (k XOR 4 (j mod 8)); the block's pairs are
// k0 = 8 BLK + tq (a0, a1) and k0 + 4 (a2, a3), and since j mod 8 = g for both rows the
// positions are (8 BLK) XOR rsw and (8 BLK + 4) XOR rsw with rsw = tq XOR 4 g.  A is
// the fp16 value v itself, P carries 2^7 (e_V = 0), so z accumulates 2^-17 * (v 2^24) p.
template <int BK, int BV, bool PACK, int BLK>
__device__ __forceinline__ void raw_v_block(const WS<BK, BV, PACK>& w, const uint32_t* row0, const uint32_t (&bp)[2],
                                            float (&z)[4]) {
  const int c0 = (8 * BLK) ^ w.rsw, c1 = (8 * BLK + 4) ^ w.rsw;
  const uint32_t A0 = row0[c0], A1 = row0[8 * (kPage / 2) + c0];
  const uint32_t A2 = row0[c1], A3 = row0[8 * (kPage / 2) + c1];
  mma_16816(z, A0, A1, A2, A3, bp[0], bp[1]);
}

// Packed mode: subtract m_V times the l gathered since the last fold from this lane's
// value sums (head tq: z columns 2 tq, rows g and g + 8 of every tile).  zl[0] holds
// head tq's l * 2^-17 in lane tq (g = 0).
template <int BK, int BV, bool PACK>
__device__ __forceinline__ void fold_centre(WS<BK, BV, PACK>& w) {
  const float lnow = __shfl_sync(0xffffffffu, w.zl[0], w.tq);
  const float dl = w.mV * (lnow - w.lfold);
  w.lfold = lnow;
#pragma unroll
  for (int mt = 0; mt < kNT; ++mt) {
    w.z[mt][0] -= dl;
    w.z[mt][2] -= dl;
  }
}

// Blocks B0 .. B0 + IL - 1 of the page: scores, lazy online softmax, value accumulation.
template <int BK, int BV, bool PACK, int B0, int... BB>
__device__ __forceinline__ void do_group(WS<BK, BV, PACK>& w, std::integer_sequence<int, BB...>) {
  constexpr int IL = sizeof...(BB);
  float sc[IL][4], sd[IL][4];
#pragma unroll
  for (int bb = 0; bb < IL; ++bb)
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[bb][i] = sd[bb][i] = 0.0f;
  // The k-steps and m-tiles below run from a jump into an unrolled sequence (no per-step
  // test).  Rows past r_K meet zero q^ coefficients (q~ is zero there) and rows past r_V
  // are never read back, so both are read unmasked inside the last tile; the
  // shared-memory allocation has slack for that over-read.
  // major-part words: the first one the group needs and how many
  constexpr int KB = major_w(BK);
  constexpr int KW0 = (B0 * KB) / 8, KWN = ((B0 + IL - 1) * KB) / 8 - KW0 + 1;
  constexpr int VB = major_w(BV);
  constexpr int VW0 = (B0 * VB) / 8, VWN = ((B0 + IL - 1) * VB) / 8 - VW0 + 1;
  // ---- scores S[tok][head] = sum_j codeK[tok][j] * q^[head][j]
  auto kstep = [&](auto KSC) {
    constexpr int ks = decltype(KSC)::value;
    const int r0 = 8 * ks + w.tq, r1 = r0 + 4;
    uint32_t bh[2], bl[2];
    bh[0] = w.fr[ks * 64];
    bh[1] = w.fr[ks * 64 + 32];
    if constexpr (!PACK) {
      bl[0] = w.fr[512 + ks * 64];
      bl[1] = w.fr[512 + ks * 64 + 32];
    } else {
      bl[0] = bl[1] = 0u;
    }
    uint32_t W0[KWN], W1[KWN], W0h[KWN], W1h[KWN];
#pragma unroll
    for (int q = 0; q < KWN; ++q) {
      W0[q] = w.pk[r0 * 8 * KB + w.g * KB + KW0 + q];
      W1[q] = w.pk[r1 * 8 * KB + w.g * KB + KW0 + q];
      W0h[q] = shr8(W0[q]);
      W1h[q] = shr8(W1[q]);
    }
    // minor-part words (K row of width-w part: 8 w words, owner g's at g w)
    uint32_t M0[2][2] = {{0u, 0u}, {0u, 0u}}, M1[2][2] = {{0u, 0u}, {0u, 0u}};
#pragma unroll
    for (int i = 0; i < n_minor(BK); ++i) {
      const int wm = minor_w(BK, i), m0 = (B0 * wm) / 8, mn = ((B0 + IL - 1) * wm) / 8 - m0 + 1;
      const uint32_t* plane = w.pk + w.kmo[i];
#pragma unroll
      for (int q = 0; q < mn; ++q) {
        M0[i][q] = plane[r0 * 8 * wm + w.g * wm + m0 + q];
        M1[i][q] = plane[r1 * 8 * wm + w.g * wm + m0 + q];
      }
    }
    auto kb = [&](auto BLKC) {
      constexpr int BLK = decltype(BLKC)::value;
      constexpr int q = (BLK * KB) / 8 - KW0;
      uint32_t m0[2], m1[2];
      pick_minor<BK, B0, BLK>(M0, m0);
      pick_minor<BK, B0, BLK>(M1, m1);
      k_block<BK, BV, PACK, BLK>(bh, bl, W0[q], W0h[q], W1[q], W1h[q], m0, m1, sc[BLK - B0], sd[BLK - B0]);
    };
    (kb(std::integral_constant<int, B0 + BB>{}), ...);
  };
  switch (w.nks) {
    default: kstep(std::integral_constant<int, 7>{}); [[fallthrough]];
    case 7: kstep(std::integral_constant<int, 6>{}); [[fallthrough]];
    case 6: kstep(std::integral_constant<int, 5>{}); [[fallthrough]];
    case 5: kstep(std::integral_constant<int, 4>{}); [[fallthrough]];
    case 4: kstep(std::integral_constant<int, 3>{}); [[fallthrough]];
    case 3: kstep(std::integral_constant<int, 2>{}); [[fallthrough]];
    case 2: kstep(std::integral_constant<int, 1>{}); [[fallthrough]];
    case 1: kstep(std::integral_constant<int, 0>{});
  }
  float x[IL][4];
  bool grow = false;
  ((grow |= x_block<BK, BV, PACK, B0 + BB>(w, sc[BB], sd[BB], x[BB])), ...);
  // grow also while the running max is undefined (the first live block)
  grow |= w.m_run[0] == -INFINITY || (!PACK && w.m_run[1] == -INFINITY);
  // ---- lazy online softmax: rescale only when a score passes the running max by 2^kLazy
  if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
    for (int c = 0; c < (PACK ? 1 : 2); ++c) {
      float v = -INFINITY;
      ((v = fmaxf(v, xmax_block<BK, BV, PACK, B0 + BB>(w, x[BB], c))), ...);
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
      // v = max over the group of s - m_run (m_run taken as 0 while undefined)
      const float old = w.m_run[c];
      float shift = 0.0f;
      if (v == -INFINITY) {
        // no live token of this head here: nothing to do
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
        if constexpr (PACK) {
          w.zl[0] *= resc;
          w.lfold *= resc;
        } else {
          w.lcvt[c] *= resc;
        }
      }
#pragma unroll
      for (int bb = 0; bb < IL; ++bb) {
        if constexpr (PACK) {
          x[bb][0] -= shift;
          x[bb][1] -= shift;
        } else {
          x[bb][c] -= shift;
          x[bb][2 + c] -= shift;
        }
      }
    }
    refresh_constants(w);
  }
  // ---- probabilities -> B fragments
  uint32_t bp[IL][2];
  (p_block<BK, BV, PACK, B0 + BB>(w, x[BB], bp[BB]), ...);
  // ---- values: Z^T[j][head] += sum_tok codeV[tok][j] * P[tok][head] (m-tiles likewise
  // entered by a jump)
  auto vtile = [&](auto MTC) {
    constexpr int mt = decltype(MTC)::value;
    if constexpr (BV == kRawBits) {
      // uncompressed values: each A register is one stored word (a token pair of one
      // coordinate, fp16 as stored); rows 16 mt + g and + 8 of the raw page
      const uint32_t* row0 = w.pv + (16 * mt + w.g) * (kPage / 2);
      (raw_v_block<BK, BV, PACK, B0 + BB>(w, row0, bp[BB], w.z[mt]), ...);
      return;
    }
    const int j0 = 16 * mt + w.g, j1 = j0 + 8;
    const bool ones = !PACK && mt == w.ones_mt;
    uint32_t W0[VWN], W1[VWN], W0h[VWN], W1h[VWN];
#pragma unroll
    for (int q = 0; q < VWN; ++q) {
      W0[q] = w.pv[j0 * 4 * VB + w.tq * VB + VW0 + q];
      W1[q] = w.pv[j1 * 4 * VB + w.tq * VB + VW0 + q];
      W0h[q] = shr8(W0[q]);
      W1h[q] = shr8(W1[q]);
    }
    // minor-part words (V row of width-w part: 4 w words, owner tq's at tq w)
    uint32_t M0[2][2] = {{0u, 0u}, {0u, 0u}}, M1[2][2] = {{0u, 0u}, {0u, 0u}};
#pragma unroll
    for (int i = 0; i < n_minor(BV); ++i) {
      const int wm = minor_w(BV, i), m0 = (B0 * wm) / 8, mn = ((B0 + IL - 1) * wm) / 8 - m0 + 1;
      const uint32_t* plane = w.pv + w.vmo[i];
#pragma unroll
      for (int q = 0; q < mn; ++q) {
        M0[i][q] = plane[j0 * 4 * wm + w.tq * wm + m0 + q];
        M1[i][q] = plane[j1 * 4 * wm + w.tq * wm + m0 + q];
      }
    }
    auto vb = [&](auto BLKC) {
      constexpr int BLK = decltype(BLKC)::value;
      constexpr int q = (BLK * VB) / 8 - VW0;
      uint32_t m0[2], m1[2];
      pick_minor<BV, B0, BLK>(M0, m0);
      pick_minor<BV, B0, BLK>(M1, m1);
      v_block<BK, BV, PACK, BLK>(w, W0[q], W0h[q], W1[q], W1h[q], m0, m1, ones, bp[BLK - B0], w.z[mt]);
    };
    (vb(std::integral_constant<int, B0 + BB>{}), ...);
  };
  switch (w.nmt) {
    default: vtile(std::integral_constant<int, 7>{}); [[fallthrough]];
    case 7: vtile(std::integral_constant<int, 6>{}); [[fallthrough]];
    case 6: vtile(std::integral_constant<int, 5>{}); [[fallthrough]];
    case 5: vtile(std::integral_constant<int, 4>{}); [[fallthrough]];
    case 4: vtile(std::integral_constant<int, 3>{}); [[fallthrough]];
    case 3: vtile(std::integral_constant<int, 2>{}); [[fallthrough]];
    case 2: vtile(std::integral_constant<int, 1>{}); [[fallthrough]];
    case 1: vtile(std::integral_constant<int, 0>{});
  }
}

template <int BK, int BV, bool PACK, int... GG>
__device__ __forceinline__ void do_page_groups(WS<BK, BV, PACK>& w, std::integer_sequence<int, GG...>) {
  (do_group<BK, BV, PACK, GG * kIL>(w, std::make_integer_sequence<int, kIL>{}), ...);
}

template <int BK, int BV, bool PACK>
__device__ __forceinline__ void do_page(WS<BK, BV, PACK>& w) {
  do_page_groups<BK, BV, PACK>(w, std::make_integer_sequence<int, 8 / kIL>{});
}

// Bytes before the stage ring: the head, then the stage barriers (8 per warp, 16-byte
// aligned), rounded to 128.
constexpr size_t kBarOffset = (sizeof(SmemHead) + 15) / 16 * 16;
constexpr size_t kHeadBytes = ((kBarOffset + 8 * kWarps * 8 + 127) / 128) * 128;

// ---- q~ = M_K q for the CTA's query heads, on the tensor cores -------------------------
// q of head n (n < ng) is scaled by 2^-Eq[n] and stored as fp16 hi (+ lo for fp32 input);
// A = M_K's fp16 hi and lo fragments (plan), so q~ = (M_hi + M_lo)(q_hi + q_lo) with the
// lo x lo product dropped (below 2^-22 relative).  Warp w forms m-tiles w and w + 4; the
// result (column n = head n) lands in sh.qt, rows past r_K exactly zero (zero A rows),
// and each tile's sum over its rows in sh.Spart.
// Both tiles' fragments were loaded before the wait for the preceding grid (the plan is
// constant), and each tile accumulates in four independent chains (k-step parity x M
// part), so the MMA latency does not add up along the 8 k-steps.
__device__ __forceinline__ void qtilde_tile(SmemHead& sh, const uint4 (&fr)[16], int mt, int g, int tq, bool q_lo) {
  float c[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i][0] = c[i][1] = c[i][2] = c[i][3] = 0.0f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const uint4 ah = fr[2 * ks], alo = fr[2 * ks + 1];
    float (&ch)[4] = c[(ks & 1) * 2], (&cl)[4] = c[(ks & 1) * 2 + 1];
    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&sh.u.q16.hi[g][16 * ks + 2 * tq]);
    const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&sh.u.q16.hi[g][16 * ks + 8 + 2 * tq]);
    mma_16816(ch, ah.x, ah.y, ah.z, ah.w, b0, b1);
    mma_16816(cl, alo.x, alo.y, alo.z, alo.w, b0, b1);
    if (q_lo) {
      const uint32_t l0 = *reinterpret_cast<const uint32_t*>(&sh.u.q16.lo[g][16 * ks + 2 * tq]);
      const uint32_t l1 = *reinterpret_cast<const uint32_t*>(&sh.u.q16.lo[g][16 * ks + 8 + 2 * tq]);
      mma_16816(cl, ah.x, ah.y, ah.z, ah.w, l0, l1);
    }
  }
  float r[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) r[e] = (c[0][e] + c[2][e]) + (c[1][e] + c[3][e]);
  const int j = 16 * mt + g;
  const float s0 = ldexpf(1.0f, sh.Eq[2 * tq]), s1 = ldexpf(1.0f, sh.Eq[2 * tq + 1]);
  sh.qt[2 * tq][j] = r[0] * s0;
  sh.qt[2 * tq + 1][j] = r[1] * s1;
  sh.qt[2 * tq][j + 8] = r[2] * s0;
  sh.qt[2 * tq + 1][j + 8] = r[3] * s1;
  // the tile's share of S = sum_j q~_j for heads 2 tq, 2 tq + 1 (summed over g)
  float sa = (r[0] + r[2]) * s0, sb = (r[1] + r[3]) * s1;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    sa += __shfl_xor_sync(0xffffffffu, sa, o);
    sb += __shfl_xor_sync(0xffffffffu, sb, o);
  }
  if (g == 0) {
    sh.Spart[mt][2 * tq] = sa;
    sh.Spart[mt][2 * tq + 1] = sb;
  }
}

__device__ __forceinline__ void form_qtilde(SmemHead& sh, int nmtK, int warp, int lane, bool q_lo,
                                            const uint4 (&fr0)[16], const uint4 (&fr1)[16]) {
  const int g = lane >> 2, tq = lane & 3;
  if (warp < nmtK) qtilde_tile(sh, fr0, warp, g, tq, q_lo);
  if (warp + kWarps < nmtK) qtilde_tile(sh, fr1, warp + kWarps, g, tq, q_lo);
}

// ---- the last CTAs of a (sequence, KV head, head group): merge and back-project ----------
// Partials (m in the log2 domain, l, centred z times 2^-17) of every split.  The merge is
// the serial tail of the call, so it is written for memory-level parallelism: every
// (m, l) is fetched at once, then each thread owns one (head, 4-coordinate) slice of z
// over a share of the splits (all of its loads independent), the shares meet in shared
// memory, y = delta_V 2^17 z / l, and o = M_V^T y (warp w: rows w, w + 4, ... of M_V,
// lane: four output columns; the four warps' sums meet in shared memory).
// scratch: 2 * 8 * kMaxSplits (m, l) + 8 * 128 (y) + 4 * 8 * 128 (the reductions of the
// split shares and of the back-projection) + 8 (l per head) floats.
constexpr int kZBatch = 24;  // partials' z loads in flight per thread in the merge
constexpr int kVBatch = 16;  // M_V rows in flight per warp in the back-projection
// Merges the query heads n0, n0 + nstep, ... (< ng) of the group starting at query head
// qh0; nl of them, local index ln.
__device__ __forceinline__ void merge_project(const DecodeArgs& a, const UnitDesc& dV, float* scratch, int s,
                                              int qh0, int ng, int n0, int nstep, int n_split, int warp, int lane,
                                              int tid) {
  const int Hq = a.H * a.G;
  const int rV = dV.r;
  const bool raw = dV.b == kRawBits;
  const int nl = (ng - n0 + nstep - 1) / nstep;
  float* mbuf = scratch;                     // [nl][n_split]: the weights 2^(m - M)
  float* ybuf = scratch + 16 * kMaxSplits;   // [8][128]
  float* obuf = ybuf + 8 * 128;              // [4][8][128] (also the split-share reduction)
  float* Lsum = ybuf + 8 * 128 + 4 * 8 * 128;  // [8]
  const float dlt = raw ? 0x1p-24f : dV.delta;
  const size_t head_stride = static_cast<size_t>(a.part_stride) * kPartStride;
  const float* base0 = a.ws + (static_cast<size_t>(s) * Hq + qh0) * head_stride;
  // (1) per head (warp per head): every split's (m, l) in one batch of loads (lane i,
  // i + 32, ...), the largest m, the weights 2^(m - M) and l
  for (int n = warp; n < nl; n += kWarps) {
    const float* hb = base0 + (n0 + n * nstep) * head_stride;
    float mi[kMaxSplits / 32], li[kMaxSplits / 32];
#pragma unroll
    for (int k = 0; k < kMaxSplits / 32; ++k) {
      const int i = lane + 32 * k;
      float2 ml = make_float2(-INFINITY, 0.0f);
      if (i < n_split) ml = __ldcg(reinterpret_cast<const float2*>(hb + static_cast<size_t>(i) * kPartStride));
      mi[k] = ml.x;
      li[k] = ml.y;
    }
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kMaxSplits / 32; ++k) M = fmaxf(M, mi[k]);
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.0f;
#pragma unroll
    for (int k = 0; k < kMaxSplits / 32; ++k) {
      const int i = lane + 32 * k;
      const float wi = (mi[k] == -INFINITY || M == -INFINITY) ? 0.0f : ex2(mi[k] - M);
      if (i < n_split) mbuf[n * n_split + i] = wi;
      L = fmaf(wi, li[k], L);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) Lsum[n] = L;
  }
  __syncthreads();
  // (3) z: slice p = (head, 4-coordinate group) and split share u; U shares per slice.
  // The loads go out in explicit batches of kZBatch (a register array filled before it is
  // used): measured here, a plain loop over the splits issued one L2 round trip per split.
  const int quads = (rV + 3) >> 2;
  const int P = nl * quads;
  const int U = P >= kThreads ? 1 : kThreads / P;
  float4* red = reinterpret_cast<float4*>(obuf);  // [U][P] when U > 1 (U * P <= 128)
  for (int t = tid; t < P * U; t += kThreads) {
    const int p = t % P, u = t / P;
    const int n = p / quads, q = p - n * quads;
    const float* zp = base0 + (n0 + n * nstep) * head_stride + 4 + 4 * q;
    const float* wn = mbuf + n * n_split;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int i0 = u; i0 < n_split; i0 += kZBatch * U) {
      float4 zz[kZBatch];
      float ww[kZBatch];
#pragma unroll
      for (int k = 0; k < kZBatch; ++k) {
        const int i = i0 + k * U;
        const bool in = i < n_split;
        zz[k] = in ? __ldcg(reinterpret_cast<const float4*>(zp + static_cast<size_t>(i) * kPartStride))
                   : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        ww[k] = in ? wn[i] : 0.0f;
      }
#pragma unroll
      for (int k = 0; k < kZBatch; ++k) {
        acc.x = fmaf(ww[k], zz[k].x, acc.x);
        acc.y = fmaf(ww[k], zz[k].y, acc.y);
        acc.z = fmaf(ww[k], zz[k].z, acc.z);
        acc.w = fmaf(ww[k], zz[k].w, acc.w);
      }
    }
    if (U > 1) {
      red[u * P + p] = acc;
    } else {
      // z holds sum p (c - m_V) 2^-17: dequantize
      const float L = Lsum[n];
      const float f = L > 0.0f ? dlt * 131072.0f / L : 0.0f;
      reinterpret_cast<float4*>(ybuf + n * 128)[q] = make_float4(acc.x * f, acc.y * f, acc.z * f, acc.w * f);
    }
  }
  if (U > 1) {
    __syncthreads();
    for (int p = tid; p < P; p += kThreads) {
      const int n = p / quads, q = p - n * quads;
      float4 acc = red[p];
      for (int u = 1; u < U; ++u) {
        const float4 v = red[u * P + p];
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      const float L = Lsum[n];
      const float f = L > 0.0f ? dlt * 131072.0f / L : 0.0f;
      reinterpret_cast<float4*>(ybuf + n * 128)[q] = make_float4(acc.x * f, acc.y * f, acc.z * f, acc.w * f);
    }
  }
  __syncthreads();
  if (raw) {
    // an uncompressed value unit is already in d-space (identity back-projection)
    for (int i = tid; i < nl * 128; i += kThreads) {
      const int n = i >> 7, k = i & 127;
      const size_t off = (static_cast<size_t>(s) * Hq + qh0 + n0 + n * nstep) * kD + k;
      if (a.out_bf16)
        static_cast<__nv_bfloat16*>(a.out)[off] = __float2bfloat16_rn(ybuf[n * 128 + k]);
      else
        static_cast<float*>(a.out)[off] = ybuf[n * 128 + k];
    }
    return;
  }
  // (4) o = M_V^T y: warp w takes rows w, w + 4, ... (lane: four output columns; M_V was
  // prefetched into L2 by every CTA of the head), kVBatch rows' loads in flight at a time
  float4 o[8];
#pragma unroll
  for (int n = 0; n < 8; ++n) o[n] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int j0 = warp; j0 < rV; j0 += kVBatch * kWarps) {
    float4 m4[kVBatch];
#pragma unroll
    for (int k = 0; k < kVBatch; ++k) {
      const int j = j0 + k * kWarps;
      m4[k] = j < rV ? __ldg(reinterpret_cast<const float4*>(dV.M + static_cast<size_t>(j) * kD) + lane)
                     : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
#pragma unroll
    for (int k = 0; k < kVBatch; ++k) {
      const int j = j0 + k * kWarps;
      if (j >= rV) break;  // (warp-uniform; y past r_V is not written)
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        if (n < nl) {
          const float yj = ybuf[n * 128 + j];
          o[n].x = fmaf(m4[k].x, yj, o[n].x);
          o[n].y = fmaf(m4[k].y, yj, o[n].y);
          o[n].z = fmaf(m4[k].z, yj, o[n].z);
          o[n].w = fmaf(m4[k].w, yj, o[n].w);
        }
      }
    }
  }
#pragma unroll
  for (int n = 0; n < 8; ++n)
    if (n < nl) reinterpret_cast<float4*>(obuf + (warp * 8 + n) * 128)[lane] = o[n];
  __syncthreads();
  for (int i = tid; i < nl * 128; i += kThreads) {
    const int n = i >> 7, k = i & 127;
    const float v = (obuf[(0 * 8 + n) * 128 + k] + obuf[(1 * 8 + n) * 128 + k]) +
                    (obuf[(2 * 8 + n) * 128 + k] + obuf[(3 * 8 + n) * 128 + k]);
    const size_t off = (static_cast<size_t>(s) * Hq + qh0 + n0 + n * nstep) * kD + k;
    if (a.out_bf16)
      static_cast<__nv_bfloat16*>(a.out)[off] = __float2bfloat16_rn(v);
    else
      static_cast<float*>(a.out)[off] = v;
  }
}

template <int BK, int BV, bool PACK>
__global__ void __launch_bounds__(kThreads, kMinBlocks) decode_split_kernel(const __grid_constant__ DecodeArgs a) {
  // Programmatic dependent launch.  The first split launch of a call waits, once it has
  // read the plan, for the preceding grid (whatever wrote q and the newest cache slots),
  // and triggers its dependents only after that wait.  A later split launch of the same
  // call starts only after that point, so it reads at once and waits at exit instead,
  // which keeps the call's completion ordered behind every launch of it.
  extern __shared__ __align__(128) unsigned char smem[];
  SmemHead& sh = *reinterpret_cast<SmemHead*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  unsigned char* stages = smem + kHeadBytes;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  // CTA -> (KV head, context split): heads get splits in proportion to their work
  int hi = 0;
  while (hi + 1 < a.n_heads && static_cast<int>(blockIdx.x) >= a.split_prefix[hi + 1]) ++hi;
  const int split = blockIdx.x - a.split_prefix[hi];
  const int n_split = a.split_prefix[hi + 1] - a.split_prefix[hi];
  const int hg = blockIdx.y;
  const int s = blockIdx.z;
  const int h = a.heads[hi];
  const int uK = (a.layer * a.H + h) * 2, uV = uK + 1;
  // the plan is constant: its unit descriptors are read, the stage barriers set up and
  // M_K's fragments (for q~) and M_V (for the merge) prefetched into L2 before the wait for
  // the preceding grid
  const UnitDesc dK = a.units[uK], dV = a.units[uV];
  const int rK = dK.r, rV = dV.r;
  const int Hq = a.H * a.G;
  const int g0 = hg * 8, ng = min(8, a.G - g0);
  const int nmtK = (rK + 15) >> 4;
  // this head's stage (a K and a V page) and how many fit in the warp's share of the ring
  // (the launch sizes the ring for its widest head; narrower heads get deeper rings)
  const uint32_t stage_b = static_cast<uint32_t>((dK.page_bytes + dV.page_bytes + 127) / 128 * 128);
  const uint32_t ring_b = static_cast<uint32_t>(a.n_stage) * a.stage_bytes;
  const int n_stage = min(6, static_cast<int>(ring_b / stage_b));
  if (lane == 0)
    for (int i = 0; i < n_stage; ++i) mbar_init(&bars[warp * 8 + i], 1);
  fence_mbar_init();
  __syncwarp();
  if (tid == 0) {
    prefetch_l2(dK.Mfrag, static_cast<uint32_t>(nmtK) * 8 * 2 * 32 * 16);
    if (dV.b != kRawBits) prefetch_l2(dV.M, static_cast<uint32_t>(rV) * kD * 4);
  }
  // this warp's m-tiles of M_K fragments for q~ (tiles w and w + 4; 16 x 16 bytes per
  // lane each; a warp without a tile reads the unit's first tile, in bounds, and never
  // uses it)
  uint4 mfrag[16], mfrag1[16];
  {
    const uint4* src = reinterpret_cast<const uint4*>(dK.Mfrag) + static_cast<size_t>(warp < nmtK ? warp : 0) * 8 * 2 * 32 + lane;
    const uint4* src1 = reinterpret_cast<const uint4*>(dK.Mfrag) +
                        static_cast<size_t>(warp + kWarps < nmtK ? warp + kWarps : 0) * 8 * 2 * 32 + lane;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      mfrag[k] = __ldg(src + k * 32);
      mfrag1[k] = __ldg(src1 + k * 32);
    }
  }
  if (a.wait_first) griddep_wait();
  griddep_launch_dependents();

  // The head's pages, as many as the call's longest sequence may have, are cut into
  // n_split * kWarps contiguous runs whose lengths differ by at most one page; warp w of
  // split c takes run c * kWarps + w, cut short at this sequence's end.  The partition
  // does not depend on the sequence length, so the block-table window of the run goes
  // out together with the other inputs the preceding kernels may have written: the
  // sequence length and the group's queries (warp w: heads 2w, 2w + 1; lane l: elements
  // 4l .. 4l + 3).
  const int n_workers = n_split * kWarps;
  const int worker = split * kWarps + warp;
  const int p_begin = static_cast<int>(static_cast<long long>(worker) * a.part_pages / n_workers);
  const int p_run = static_cast<int>(static_cast<long long>(worker + 1) * a.part_pages / n_workers) - p_begin;
  const int32_t* bt = a.block_table + static_cast<size_t>(s) * a.max_pages;
  // lane l holds the id of page base + l of the current window of 32 (-1 past the run)
  int pid_win = lane < p_run ? bt[p_begin + lane] : -1;
  int seq_len = a.seq_lens[s];
  float4 qv[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int gg = 2 * warp + hh;
    qv[hh] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (gg < ng) {
      const size_t off = (static_cast<size_t>(s) * Hq + h * a.G + g0 + gg) * kD + 4 * lane;
      if (a.q_bf16) {
        const uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.q) + off);
        qv[hh] = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                             __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u));
      } else {
        qv[hh] = *reinterpret_cast<const float4*>(static_cast<const float*>(a.q) + off);
      }
    }
  }
  if (seq_len < 0 || seq_len > a.part_pages * kPage) {
    if (tid == 0 && a.status) atomicOr(a.status, KVTC_STATUS_BAD_POS);
    seq_len = seq_len < 0 ? 0 : a.part_pages * kPage;
  }
  const int n_pages = (seq_len + kPage - 1) / kPage;
  const int n_my = max(0, min(p_run, n_pages - p_begin));

  // ---- prologue: each warp's first copy (the barriers were set up by lane 0 of each warp,
  // which also issues the copies), then q~ while it is in flight ----

  const uint32_t bytesK = static_cast<uint32_t>(dK.page_bytes), bytesV = static_cast<uint32_t>(dV.page_bytes);
  const char* poolK = a.pool + a.pages_per_unit * dK.prefix;
  const char* poolV = a.pool + a.pages_per_unit * dV.prefix;
  unsigned char* const warp_stages = stages + static_cast<size_t>(warp) * ring_b;
  auto stage_ptr = [&](int slot) { return warp_stages + static_cast<size_t>(slot) * stage_b; };
  // Page ids of this warp's pages, 32 at a time (the first window was loaded above), so
  // no dependent global load is left in the loop.
  int pid_base = 0;
  auto pid_of = [&](int i) {  // warp-uniform i
    const int base = i & ~31;
    if (base != pid_base) {
      const int ii = base + lane;
      pid_win = ii < n_my ? bt[p_begin + ii] : -1;
      pid_base = base;
    }
    return __shfl_sync(0xffffffffu, pid_win, i & 31);
  };
  // Fill the stage of this warp's i-th page.  Every use of a stage completes its barrier
  // phase exactly once: with the copies' bytes, or by a plain arrival when the page id
  // is invalid.  vmask (lane 0) has bit slot set when the stage holds a page.
  uint32_t vmask = 0;
  auto issue = [&](int slot, int pid) {  // lane 0
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
  const int n_first = min(n_stage, n_my);
  // only the first page of each warp now: the rest of the ring is issued after q~ (a burst
  // of every warp's ring at once keeps the copy engine busy while q~ is formed)
  if (n_first > 0) {
    const int pid = pid_of(0);
    if (lane == 0) issue(0, pid);
  }

  // ---- q of the group into shared memory as fp16, scaled per head, and the fp16
  // normalisation of q~: |q~_j| <= ||M_K row j|| ||q||_2 <= mnorm ||q||_2 (Cauchy-Schwarz;
  // mnorm is rounded up, the factor 1.01 covers the rounding of the formed q~), so
  // q^ = q~ 2^-E with E = ilogb(bound) - 14 stays below 2^15
  const bool q_lo = !a.q_bf16;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int gg = 2 * warp + hh;
    const float4 v = qv[hh];
    float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
    float ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, v.w * v.w)));
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
    }
    // (||q||_2 from max |q| when the squares leave the fp32 range)
    const float qn = (ss > 0x1p-100f && ss < 0x1p100f) ? sqrtf(ss) : amax * 11.32f;
    const float bound = dK.mnorm * qn * 1.01f;
    // max |q| 2^-Eq in [2^14, 2^15): fp16 holds it with headroom
    const int Eq = (amax > 0.0f && amax < INFINITY) ? ilogbf(amax) - 14 : 0;
    const float sc = ldexpf(1.0f, -Eq);
    const float xs[4] = {v.x * sc, v.y * sc, v.z * sc, v.w * sc};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __half hq = __float2half_rn(xs[e]);
      sh.u.q16.hi[gg][4 * lane + e] = __half_as_ushort(hq);
      sh.u.q16.lo[gg][4 * lane + e] = __half_as_ushort(__float2half_rn(xs[e] - __half2float(hq)));
    }
    if (lane == 0) {
      sh.Eq[gg] = Eq;
      sh.E[gg] = (bound > 0.0f && bound < INFINITY) ? ilogbf(bound) - 14 : 0;
    }
  }
  __syncthreads();
  form_qtilde(sh, nmtK, warp, lane, q_lo, mfrag, mfrag1);
  __syncthreads();

  // B fragments of q^ = q~ * 2^-E of the k-steps below r_K, shared by the four warps:
  // [hi, lo][k-step][half][lane] (lane (g, t): rows 16 ks + 8 half + 2t, + 1, column g).
  // Packed (G <= 4): column n holds head n / 2, its hi part for even n and its lo part
  // for odd n.
  for (int idx = tid; idx < nmtK * 2 * 32; idx += kThreads) {
    const int ks = idx >> 6, half = (idx >> 5) & 1, ln = idx & 31;
    const int gl = ln >> 2, tql = ln & 3;
    const int hsrc = PACK ? (gl >> 1) : gl;
    const float scl = ldexpf(1.0f, -sh.E[hsrc]);
    const int k0 = 16 * ks + 8 * half + 2 * tql;
    const float x0 = sh.qt[hsrc][k0] * scl, x1 = sh.qt[hsrc][k0 + 1] * scl;
    const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
    const __half l0 = __float2half_rn(x0 - __half2float(h0)), l1 = __float2half_rn(x1 - __half2float(h1));
    const uint32_t hw = static_cast<uint32_t>(__half_as_ushort(h0)) | (static_cast<uint32_t>(__half_as_ushort(h1)) << 16);
    const uint32_t lw = static_cast<uint32_t>(__half_as_ushort(l0)) | (static_cast<uint32_t>(__half_as_ushort(l1)) << 16);
    if constexpr (PACK) {
      sh.u.frag[0][ks][half][ln] = (gl & 1) ? lw : hw;
    } else {
      sh.u.frag[0][ks][half][ln] = hw;
      sh.u.frag[1][ks][half][ln] = lw;
    }
  }
  __syncthreads();

  for (int i = 1; i < n_first; ++i) {
    const int pid = pid_of(i);
    if (lane == 0) issue(i, pid);  // page i < n_stage uses slot i
  }

  WS<BK, BV, PACK> w;
  w.fr = &sh.u.frag[0][0][0][lane];
  w.rK = rK;
  w.rV = rV;
  w.nks = nmtK;
  w.nmt = (rV + 15) >> 4;
  w.g = g;
  w.tq = tq;
  w.rsw = tq ^ (g << 2);
  w.seq_len = seq_len;
  w.partial = false;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    w.kmo[i] = 4 * rK * minor_lo(BK, i);
    w.vmo[i] = 4 * rV * minor_lo(BV, i);
  }
  w.ones_mt = (!PACK && (rV & 15)) ? (rV >> 4) : -1;
  w.ones_lr = rV & 15;
  w.ones_m0 = (w.ones_mt >= 0 && w.ones_lr == g) ? 0xFFFFFFFFu : 0u;
  w.ones_m1 = (w.ones_mt >= 0 && w.ones_lr == g + 8) ? 0xFFFFFFFFu : 0u;
  // Score constants (log2 domain) for this lane's heads.
  {
    const float mK = 0.5f * static_cast<float>((1 << dK.b) - 1);
    const float base = a.scale * dK.delta * kLog2e;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int n = PACK ? tq : 2 * tq + c;  // packed: one head per lane
      w.alpha[c] = n < ng ? base * ldexpf(1.0f, sh.E[n] + 24) : 0.0f;
      float S = 0.0f;  // sum_j q~_j of head n, tile by tile in a fixed order
      for (int mt = 0; mt < nmtK; ++mt) S += n < ng ? sh.Spart[mt][n] : 0.0f;
      w.beta[c] = n < ng ? base * mK * S : 0.0f;
      w.m_run[c] = -INFINITY;
      w.lcvt[c] = 0.0f;
    }
    refresh_constants(w);
    // ones row of the l MMA: fp16 subnormals 2^(e_V - 24), e_V of the block parity
#pragma unroll
    for (int p = 0; p < 2; ++p) {
#pragma unroll
      for (int eta = 0; eta < 2; ++eta) {
        const int e = e_of<BV>(p, eta);
        w.onesA[p][eta] = g == 0 ? ((1u << e) | (1u << (e + 16))) : 0u;
      }
    }
    w.zl[0] = w.zl[1] = w.zl[2] = w.zl[3] = 0.0f;
    w.mV = dV.b == kRawBits ? 0.0f : (kFoldOnly<BV, PACK> ? 0.5f * static_cast<float>((1 << dV.b) - 1) : 0.5f);
    w.lfold = 0.0f;
  }
#pragma unroll
  for (int mt = 0; mt < kNT; ++mt) w.z[mt][0] = w.z[mt][1] = w.z[mt][2] = w.z[mt][3] = 0.0f;

  // ---- main loop over this warp's pages ----
  bool dead = false;
  int next_issue = n_first;
  int slot = 0;        // stage of page i (i mod n_stage), kept incrementally
  uint32_t phase = 0;  // barrier phase of that use of the stage ((i / n_stage) & 1)
  for (int i = 0; i < n_my; ++i) {
    const int p = p_begin + i;
    const bool valid = (__shfl_sync(0xffffffffu, vmask, 0) >> slot) & 1u;
    if (!mbar_wait_bounded_warp(&bars[warp * 8 + slot], phase)) {
      if (lane == 0 && a.status) atomicOr(a.status, KVTC_STATUS_TIMEOUT);
      dead = true;
      // wait (bounded) for the copies still in flight before leaving
      int s2 = slot;
      uint32_t ph2 = phase;
      for (int i2 = i + 1; i2 < next_issue; ++i2) {
        if (++s2 == n_stage) {
          s2 = 0;
          ph2 ^= 1u;
        }
        (void)mbar_wait_bounded_warp(&bars[warp * 8 + s2], ph2);
      }
      break;
    }
    if (valid) {
      const unsigned char* st = stage_ptr(slot);
      w.pk = reinterpret_cast<const uint32_t*>(st);
      w.pv = reinterpret_cast<const uint32_t*>(st + bytesK);
      w.tok0 = p * kPage;
      w.partial = w.tok0 + kPage > w.seq_len;
      do_page<BK, BV, PACK>(w);
      if constexpr (PACK) fold_centre(w);
    } else if (lane == 0 && a.status) {
      atomicOr(a.status, KVTC_STATUS_BAD_PAGE);
    }
    // release the stage: every lane is done reading it, then refill it
    __syncwarp();
    if (next_issue < n_my && next_issue == i + n_stage) {
      const int npid = pid_of(next_issue);
      if (lane == 0) issue(slot, npid);  // page i + n_stage reuses page i's stage
      ++next_issue;
    }
    __syncwarp();
    if (++slot == n_stage) {
      slot = 0;
      phase ^= 1u;
    }
  }

  // ---- l: from the ones row, or the per-lane sums ----
  float l_out[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    if (PACK) {
      // row 0 of the l MMA: lane tq (g == 0) holds head tq's l * 2^-17
      l_out[c] = ldexpf(__shfl_sync(0xffffffffu, w.zl[0], tq), 17);
    } else if (w.ones_mt >= 0) {
      // select z[ones_mt][row] with a masked sum (a select here would be turned into a
      // run-time index and push the fragments to local memory)
      float v = 0.0f;
      const float lo_row = w.ones_lr < 8 ? 1.0f : 0.0f, hi_row = 1.0f - lo_row;
#pragma unroll
      for (int mt = 0; mt < kNT; ++mt) {
        const float on = mt == w.ones_mt ? 1.0f : 0.0f;
        v = fmaf(on * lo_row, w.z[mt][c], fmaf(on * hi_row, w.z[mt][2 + c], v));
      }
      // the value sits in lanes with g == ones_lr % 8 (same tq); z holds l * 2^-17
      const int src = ((w.ones_lr & 7) << 2) | tq;
      l_out[c] = ldexpf(__shfl_sync(0xffffffffu, v, src), 17);
    } else {
      float l = w.lcvt[c];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      l_out[c] = l;
    }
  }

  // ---- finish centring: the partial carries sum p (c - m_V) (times 2^-17) ----
  if constexpr (PACK) {
    fold_centre(w);
  } else {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const float dl = w.mV * ldexpf(l_out[c], -17);
#pragma unroll
      for (int mt = 0; mt < kNT; ++mt) {
        w.z[mt][c] -= dl;
        w.z[mt][2 + c] -= dl;
      }
    }
  }

  // ---- merge the four warps' (m, l, z) per query head in shared memory (the stage
  // buffers are free: every copy issued has been waited for), then write one partial per
  // CTA and query head ----
  float* mb = reinterpret_cast<float*>(stages);  // [kWarps][8][kPartStride]
  __syncthreads();
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    // head of z column 2 tq + c: packed mode keeps head tq in column 2 tq (odd columns 0)
    const int n = PACK ? tq : 2 * tq + c;
    const bool real = PACK ? (c == 0 && n < ng) : n < ng;
    if (real) {
      float* dst = mb + (warp * 8 + n) * kPartStride;
      if (g == 0) {
        dst[0] = dead ? -INFINITY : w.m_run[c];
        dst[1] = dead ? 0.0f : l_out[c];
      }
#pragma unroll
      for (int mt = 0; mt < kNT; ++mt) {
        if (mt < w.nmt) {
          const int j0 = 16 * mt + g, j1 = j0 + 8;
          if (j0 < rV) dst[4 + j0] = dead ? 0.0f : w.z[mt][c];
          if (j1 < rV) dst[4 + j1] = dead ? 0.0f : w.z[mt][2 + c];
        }
      }
    }
  }
  __syncthreads();
  float* dstb = a.ws + (static_cast<size_t>(s) * Hq + h * a.G + g0) * a.part_stride * kPartStride +
                static_cast<size_t>(split) * kPartStride;
  for (int idx = tid; idx < ng * (rV + 2); idx += kThreads) {
    const int n = idx / (rV + 2), e = idx - n * (rV + 2);
    float mw[kWarps], M = -INFINITY;
#pragma unroll
    for (int q = 0; q < kWarps; ++q) {
      mw[q] = mb[(q * 8 + n) * kPartStride];
      M = fmaxf(M, mw[q]);
    }
    float acc = 0.0f;
    const int src = e == 0 ? 1 : 4 + (e - 1);  // e == 0: l; e >= 1: z[e - 1]
    if (M != -INFINITY && e <= rV) {
#pragma unroll
      for (int q = 0; q < kWarps; ++q)
        if (mw[q] != -INFINITY) acc = fmaf(ex2(mw[q] - M), mb[(q * 8 + n) * kPartStride + src], acc);
    }
    float* dst = dstb + static_cast<size_t>(n) * a.part_stride * kPartStride;
    if (e == 0) {
      dst[0] = M;
      dst[1] = acc;
    } else if (e <= rV) {
      dst[src] = acc;
    }
  }

  // ---- arrival tickets: the last n_par = min(ng, n_split) CTAs to finish a (sequence, KV
  // head, head group) each merge a share of its query heads (the k-th last takes heads k,
  // k + n_par, ...) once every split has written its partial, so the merge runs on
  // several SMs at once; the last of them re-arms the counters.  With few splits the
  // merge is short and the last CTA does it alone (n_par = 1).  A CTA that takes a
  // share has finished its own work and waits (bounded) only for CTAs that hold a
  // ticket position after it, which have all started.
  __threadfence();
  __syncthreads();
  int* ticket = a.tickets + ((static_cast<size_t>(s) * a.H + h) * a.n_hg + hg) * kTicketInts;
  if (tid == 0) sh.ticket = atomicAdd(ticket, 1);
  __syncthreads();
  const int n_par = n_split >= kParMerge ? min(ng, n_split) : 1;
  const int k_last = n_split - 1 - sh.ticket;  // 0: this CTA finished last
  if (k_last >= 0 && k_last < n_par) {  // (a counter left non-zero by a broken call gives none)
    if (tid == 0) {
      uint32_t it = 0;
      while (ld_acquire_gpu(ticket) < n_split && it < kSpinLimit) {
        __nanosleep(100);
        ++it;
      }
      sh.ticket = it < kSpinLimit;
      if (it >= kSpinLimit && a.status) atomicOr(a.status, KVTC_STATUS_TIMEOUT);
    }
    __syncthreads();
    if (sh.ticket) {
      __threadfence();
      merge_project(a, dV, mb, s, h * a.G + g0, ng, k_last, n_par, n_split, warp, lane, tid);
    }
    if (tid == 0 && atomicAdd(ticket + 1, 1) == n_par - 1) {
      atomicExch(ticket, 0);
      atomicExch(ticket + 1, 0);
    }
  }
  if (!a.wait_first) griddep_wait();
}

using SplitFn = void (*)(const DecodeArgs);
// Kernel for (code width variants, packed); widths: 2, 4, 8 or 0 (any).
template <int BK>
SplitFn split_fn_bk(int bV, bool pack);

}  // namespace dec
}  // namespace kvtc
