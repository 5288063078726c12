// Internal declarations shared by the host side and the CUDA kernels of libkvtc.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "../../include/kvtc.h"

namespace kvtc {

constexpr int kPage = KVTC_PAGE_TOKENS;
constexpr int kD = KVTC_HEAD_DIM;
constexpr int kRawBits = KVTC_RAW_BITS;

// A unit's (r, b) is valid when r is even in [2, d] and b in [2, 8], or when it is an
// uncompressed value unit (kind 1): r = d, b = kRawBits.
inline bool valid_rb(int r, int b, int kind) {
  if (kind == 1 && r == kD && b == kRawBits) return true;
  return r >= 2 && r <= kD && (r & 1) == 0 && b >= 2 && b <= 8;
}

// Per-unit parameters as the kernels read them (device array, one per unit).
struct UnitDesc {
  int r;               // retained coordinates (even, 2..128)
  int b;               // bits per code (2..8), or kRawBits (uncompressed value unit)
  float delta;         // quantizer step
  float inv_delta;     // fp32(1/delta)
  uint64_t page_bytes; // 16 * r * b
  uint64_t prefix;     // sum of page_bytes over the units before this one
  const float* M;      // device fp32 [r][d]
  const uint16_t* Mbf; // device bf16 bits [r][d] (round-to-nearest-even of M)
  // device: M as fp16 hi + lo parts (hi = RN16(M), lo = RN16(M - hi)) in m16n8k16
  // A-fragment order, [ceil(r/16)][8 k-steps][2 parts][32 lanes][4 registers] (rows past r
  // are zero); the decode forms q~ = M q from it on the tensor cores
  const uint32_t* Mfrag;
  // device, key units only (else null): M^T as fp16 hi + lo parts in m16n8k16 B-fragment
  // order for K-hat = C M (C: codes, tokens x r), [ceil(r/16)][16 n-tiles][32 lanes][4]
  // = (hi b0, hi b1, lo b0, lo b1); then the column sums sum_j M[j][i] (fp32 [128])
  const uint32_t* Mrec;
  const float* Msum;
  float mnorm;         // largest row 2-norm of the bf16 M (rounded up)
};

// One decode launch of a layer: the KV heads whose (b_K, b_V) width classes share a split
// kernel variant, with the variant's shared-memory plan (decided once, at plan upload).
struct DecodeGroup {
  int wk = 0, wv = 0;           // code widths b_K (2..8) and b_V (2..8, or 16: raw values)
  std::vector<int> heads;       // KV heads of the layer in this launch
  std::vector<double> cost;     // modelled cost of one page of each head (warp instructions)
  uint32_t stage_bytes = 0;     // one K + V page of the widest head, 128-byte rounded
  int n_stage = 0;              // stages per warp
  size_t smem = 0;              // dynamic shared memory per CTA
  int per_sm = 1;               // resident CTAs per SM at that size
  const void* fn = nullptr;     // the kernel variant
};

// One pre-RoPE decode launch of a layer: the KV heads whose (b_K, b_V) share a kernel
// variant, with its shared-memory plan and occupancy (decided once, at plan upload).
struct RopeGroup {
  const void* fn = nullptr;     // the kernel variant
  std::vector<int> heads;       // KV heads of the layer in this launch
  uint32_t stage_bytes = 0;     // one K + V page of the widest head, 128-byte rounded
  int n_stage = 0;              // stages per warp
  size_t smem = 0;              // dynamic shared memory per CTA
  int per_sm = 1;               // resident CTAs per SM at that size
};

// Sets the thread-local error message and returns the status.
kvtc_status fail(kvtc_status s, const std::string& msg);
kvtc_status cuda_fail(int err, const char* what);

}  // namespace kvtc

struct kvtc_plan {
  int L = 0, H = 0, G = 0, d = 0, U = 0;
  std::vector<int> r, b;
  std::vector<double> delta, sigma, D;
  std::vector<float> inv_delta;
  std::vector<std::vector<float>> M;       // [U][r*d]
  std::vector<std::vector<double>> w, lam; // [U][d] (empty for imported plans)
  double mu = 0.0;
  double t_stats = 0.0, t_alloc = 0.0;     // kvtc_calibrate: seconds in the eigen step and in C1 + C2
  // device copy (kvtc_plan_upload)
  int device = -1;
  kvtc::UnitDesc* d_units = nullptr;
  float* d_M = nullptr;
  uint16_t* d_Mbf = nullptr;
  uint32_t* d_Mfrag = nullptr;
  uint32_t* d_Mrec = nullptr;                // key units: reconstruction fragments + column sums
  uint64_t* d_stats = nullptr;               // prefill counters (codes, recomputed)
  std::vector<kvtc::UnitDesc> h_units;      // descriptors with device pointers
  // decode launch plan, per layer (set at upload): the launches and the device's SM count
  std::vector<std::vector<kvtc::DecodeGroup>> dec_groups;
  std::vector<std::vector<kvtc::RopeGroup>> rope_groups;  // the same for the pre-RoPE decode
  int sm_count = 0;
};

namespace kvtc {
// Validates that the plan is uploaded to the current device.
kvtc_status check_uploaded(const kvtc_plan* plan);
// Fills plan->dec_groups and plan->sm_count for the current device and sets the kernel
// attributes the decode launches need (decode.cu; called by kvtc_plan_upload).
kvtc_status prepare_decode(kvtc_plan* plan);
// Fills plan->rope_groups and sets the pre-RoPE kernels' attributes (decode_rope.cu;
// called by kvtc_plan_upload after prepare_decode).
kvtc_status prepare_rope(kvtc_plan* plan);
}  // namespace kvtc
