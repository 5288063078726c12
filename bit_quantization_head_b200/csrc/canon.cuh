// The canonical per-token encode arithmetic, shared by the append kernel and the fused
// append of the decode step: the latent y_j = M_j . x in a fixed fp32 order (eight fma
// chains over k mod 8, then a fixed pairwise sum: the order the oracle reproduces bit for
// bit), the b-bit quantizer, and the store of one code into a page.
//
// KV-COBRA project page, "How KV-COBRA Works" (Inference): rotate and truncate with
// H.V^T, quantize with the unit's b-bit quantizer.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kvtc_internal.h"
#include "layout.cuh"

namespace kvtc {

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

// y_j for an input row xs[128] (fp32 values of the bf16 inputs) against the bf16 row of M
// held in registers as 16 x 16 bytes.
__device__ __forceinline__ float canon_dot_bf16(const float* xs, const uint4 (&mr)[16]) {
  float ch[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint32_t w[4] = {mr[c].x, mr[c].y, mr[c].z, mr[c].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      ch[2 * q] = __fmaf_rn(xs[8 * c + 2 * q], __uint_as_float(w[q] << 16), ch[2 * q]);
      ch[2 * q + 1] = __fmaf_rn(xs[8 * c + 2 * q + 1], __uint_as_float(w[q] & 0xFFFF0000u), ch[2 * q + 1]);
    }
  }
  return __fadd_rn(__fadd_rn(__fadd_rn(ch[0], ch[1]), __fadd_rn(ch[2], ch[3])),
                   __fadd_rn(__fadd_rn(ch[4], ch[5]), __fadd_rn(ch[6], ch[7])));
}

// y_j for an input row xs[128] (fp32 values of bf16 inputs) against the bf16 row of M
// read from memory, 16 bytes at a time (the same arithmetic as canon_dot_bf16).
__device__ __forceinline__ float canon_dot_bf16_mem(const float* xs, const uint4* m4) {
  float ch[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 4
  for (int c = 0; c < 16; ++c) {
    const uint4 m = m4[c];
    const uint32_t w[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      ch[2 * q] = __fmaf_rn(xs[8 * c + 2 * q], __uint_as_float(w[q] << 16), ch[2 * q]);
      ch[2 * q + 1] = __fmaf_rn(xs[8 * c + 2 * q + 1], __uint_as_float(w[q] & 0xFFFF0000u), ch[2 * q + 1]);
    }
  }
  return __fadd_rn(__fadd_rn(__fadd_rn(ch[0], ch[1]), __fadd_rn(ch[2], ch[3])),
                   __fadd_rn(__fadd_rn(ch[4], ch[5]), __fadd_rn(ch[6], ch[7])));
}

// y_j for an fp32 input row xs[128] against the fp32 row mrow[128] of M.
__device__ __forceinline__ float canon_dot_f32(const float* xs, const float* mrow) {
  float ch[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  const float4* m4 = reinterpret_cast<const float4*>(mrow);
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
  return __fadd_rn(__fadd_rn(__fadd_rn(ch[0], ch[1]), __fadd_rn(ch[2], ch[3])),
                   __fadd_rn(__fadd_rn(ch[4], ch[5]), __fadd_rn(ch[6], ch[7])));
}

}  // namespace kvtc
