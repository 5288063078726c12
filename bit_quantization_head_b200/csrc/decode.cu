// kvtc_decode_attention: one decode step of attention over the packed code cache.
//
// KV-COBRA project page, "Efficiency": the cache is stored as packed b-bit codes with the
// rotation folded into the basis, so dequantization and the inverse rotation run in one
// fused pass.  Here the inverse key rotation is folded into the query (q~ = M_K q, the
// same algebra as NOVA-KV's query-side fold on the pith.science review page) and values
// are accumulated in their latent basis, back-projected once per query head.
//
// Kernel 0 (decode_prep_kernel): q~ = M_K q for every query head, once per call.
// Kernel 1 (decode_split_kernel<BK, BV, PACK>): CTA = (context split, KV head [, head
// group of 8], sequence), four warps, each streaming its own pages through a ring of
// cp.async.bulk + mbarrier stages.  Per 16-token block a warp computes the G (<= 8) query
// heads' scores with m16n8k16 tensor-core MMAs whose A operand is taken directly from the
// packed words: one AND leaves each code c in the low mantissa bits of an fp16 half, i.e.
// the subnormal c * 2^(e-24) (exact), with e the field's bit offset; e is undone per row in
// fp32.  q~ is split into fp16 hi + lo (about 22 bits).  Online softmax per block; P goes
// to fp16 (scaled by 2^(7-e) so P * A = p * c * 2^-17 whatever e is), is transposed into
// the B fragment with movmatrix, and multiplies the value codes (A = V codes shifted by
// floor(m_V), rows = latent coordinates) into fp32 accumulators; the remaining 0.5 l is
// folded in, so each CTA writes one centred (m, l, z) partial per query head.  Keys-only
// plans feed the stored fp16 values to the same MMAs.
// Kernel 2 (decode_combine_kernel): log-sum-exp merge of the partials, dequantization
// (delta_V) and the back-projection o = M_V^T y.
// All launches use programmatic dependent launch, so each kernel's set-up overlaps the
// tail of the one before it.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
namespace {

// ---- kernel 0: q~ = M_K q for every query head (the split kernels read it) -------------
struct PrepArgs {
  const UnitDesc* units;
  int layer, H, G, n_hg;
  const void* q;
  int q_bf16;
  float* qt;  // [n_seq][Hq][128]
};

// Sum over the 32 lanes of eight per-lane values v[0..7] with nine shuffles (each step
// halves the values a lane keeps); lane l ends with the total of value (l >> 2) & 7.
__device__ __forceinline__ float warp_sum8(const float (&v)[8], int lane) {
  float a4[4], a2[2];
  const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = u16 ? v[i] : v[i + 4], keep = u16 ? v[i + 4] : v[i];
    a4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = u8 ? a4[i] : a4[i + 2], keep = u8 ? a4[i + 2] : a4[i];
    a2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float a1 = (u4 ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, u4 ? a2[0] : a2[1], 4);
  a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
  a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
  return a1;
}

// CTA = (16 rows of M_K, KV head x head group of 8, sequence); warp w forms rows
// 16 * chunk + 4w .. +3 for the group's query heads: lane l holds columns 4l..4l+3 of the
// row (one coalesced 512-byte load per row) and the partial dot products are summed
// across lanes with warp_sum8.
__global__ void __launch_bounds__(128) decode_prep_kernel(const __grid_constant__ PrepArgs a) {
  // The split kernels that follow may start now (they wait for this grid to complete).
  griddep_launch_dependents();
  const int chunk = blockIdx.x, h = blockIdx.y / a.n_hg, hg = blockIdx.y % a.n_hg, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const UnitDesc dK = a.units[(a.layer * a.H + h) * 2];
  const int rK = dK.r;
  const int j0 = 16 * chunk + 4 * warp;
  float4 m[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    m[i] = j0 + i < rK ? reinterpret_cast<const float4*>(dK.M + static_cast<size_t>(j0 + i) * kD)[lane]
                       : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  // q is the predecessor's output: wait for it (this also makes the completion of this
  // grid imply the completion of the one before it, which the split kernels rely on).
  griddep_wait();
  if (16 * chunk >= rK) return;
  const int Hq = a.H * a.G, g0 = hg * 8, ng = min(8, a.G - g0);
  float4 qv[8];
#pragma unroll
  for (int gg = 0; gg < 8; ++gg) {
    qv[gg] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (gg < ng) {
      const size_t off = (static_cast<size_t>(s) * Hq + h * a.G + g0 + gg) * kD + 4 * lane;
      if (a.q_bf16) {
        const uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.q) + off);
        qv[gg] = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                             __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u));
      } else {
        qv[gg] = *reinterpret_cast<const float4*>(static_cast<const float*>(a.q) + off);
      }
    }
  }
  const int head = (lane >> 2) & 7;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float v[8];
#pragma unroll
    for (int gg = 0; gg < 8; ++gg)
      v[gg] = fmaf(m[i].x, qv[gg].x, fmaf(m[i].y, qv[gg].y, fmaf(m[i].z, qv[gg].z, m[i].w * qv[gg].w)));
    const float t = warp_sum8(v, lane);
    if ((lane & 3) == 0 && head < ng && j0 + i < rK)
      a.qt[(static_cast<size_t>(s) * Hq + h * a.G + g0 + head) * kD + j0 + i] = t;
  }
}

// ---- kernel 2: merge the partials, dequantise, back-project -----------------------------
// CTA = (query head, sequence, block of 32 output columns), 128 threads.  The CTA's slice
// M_V[:, 32c .. 32c + 31] is loaded into shared memory before the wait for the split
// kernels; then the four warps fold the partials (lane l holds latent coordinates
// 4l..4l+3), meet in shared memory, and back-project the slice (each warp a quarter of
// the latent rows).  The merge is repeated by the four column blocks of a query head: it
// reads (4 + r_V) floats per partial, from L2.
struct CombineArgs {
  const UnitDesc* units;
  int layer, H, G;
  int part_stride;                    // partial slots per query head
  int nparts[kMaxHeadsPerLaunch];     // partials written for each KV head
  const float* ws;
  void* out;
  int out_bf16;
  int32_t* status;
};
constexpr int kCombThreads = 128;
constexpr int kCombWarps = kCombThreads / 32;
constexpr int kCombCols = 32;  // output columns per CTA

__global__ void __launch_bounds__(kCombThreads) decode_combine_kernel(const __grid_constant__ CombineArgs ca) {
  __shared__ __align__(16) float Ms[kD][kCombCols];       // M_V rows, this CTA's columns
  __shared__ __align__(16) float zsh[kCombWarps][kD];     // written as float4
  __shared__ float lsh[kCombWarps];
  __shared__ float mxsh[kCombWarps];
  __shared__ float y[kD];
  __shared__ float osh[kCombWarps][kCombCols];
  const int qh = blockIdx.x, s = blockIdx.y, cb = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = ca.H * ca.G, h = qh / ca.G;
  const UnitDesc dV = ca.units[(ca.layer * ca.H + h) * 2 + 1];
  const int rV = dV.r;
  // an uncompressed value unit (keys-only plans) is already in d-space: its latent is
  // the output (identity back-projection), its codes are v * 2^24
  const bool raw = dV.b == kRawBits;
  // the plan's M_V is not written by the preceding kernels: load it before the wait
  for (int i = tid; !raw && i < rV * (kCombCols / 4); i += kCombThreads) {
    const int j = i / (kCombCols / 4), c4 = i % (kCombCols / 4);
    reinterpret_cast<float4*>(Ms[j])[c4] =
        reinterpret_cast<const float4*>(dV.M + static_cast<size_t>(j) * kD + cb * kCombCols)[c4];
  }
  griddep_wait();
  griddep_launch_dependents();
  const int n_part = ca.nparts[h];
  const float* base = ca.ws + (static_cast<size_t>(s) * Hq + qh) * ca.part_stride * kPartStride;
  // One pass over the partials per warp (partials warp, warp + 4, ...) with a running
  // maximum (log2 domain); the four warps then meet at the largest of their maxima.
  float mw = -INFINITY;
  float4 zacc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  float lacc = 0.0f;
#pragma unroll 4
  for (int i = warp; i < n_part; i += kCombWarps) {
    const float* pp = base + static_cast<size_t>(i) * kPartStride;
    const float mi = pp[0];
    const float li = pp[1];
    const float4 z4 = 4 * lane < rV ? reinterpret_cast<const float4*>(pp + 4)[lane] : make_float4(0, 0, 0, 0);
    if (mi == -INFINITY) continue;  // a split without live tokens
    if (mi > mw) {
      const float sc = mw == -INFINITY ? 0.0f : exp2f(mw - mi);
      zacc.x *= sc;
      zacc.y *= sc;
      zacc.z *= sc;
      zacc.w *= sc;
      lacc *= sc;
      mw = mi;
    }
    const float wi = exp2f(mi - mw);
    lacc = fmaf(wi, li, lacc);
    zacc.x = fmaf(wi, z4.x, zacc.x);
    zacc.y = fmaf(wi, z4.y, zacc.y);
    zacc.z = fmaf(wi, z4.z, zacc.z);
    zacc.w = fmaf(wi, z4.w, zacc.w);
  }
  if (lane == 0) mxsh[warp] = mw;
  __syncthreads();
  float mx = mxsh[0];
#pragma unroll
  for (int w = 1; w < kCombWarps; ++w) mx = fmaxf(mx, mxsh[w]);
  const float sw = mw == -INFINITY ? 0.0f : exp2f(mw - mx);
  zacc.x *= sw;
  zacc.y *= sw;
  zacc.z *= sw;
  zacc.w *= sw;
  reinterpret_cast<float4*>(zsh[warp])[lane] = zacc;
  if (lane == 0) lsh[warp] = lacc * sw;
  __syncthreads();
  float L = 0.0f;
#pragma unroll
  for (int w = 0; w < kCombWarps; ++w) L += lsh[w];
  const float dlt = raw ? 0x1p-24f : dV.delta;
  for (int j = tid; j < rV; j += kCombThreads) {
    float zs = 0.0f;
#pragma unroll
    for (int w = 0; w < kCombWarps; ++w) zs += zsh[w][j];
    // z holds sum p*(c - m_V)*2^-17 (the split kernel centres it); dequantize
    y[j] = L > 0.0f ? dlt * ldexpf(zs, 17) / L : 0.0f;
  }
  __syncthreads();
  // o[k] = sum_j M_V[j][k] y[j] for this CTA's 32 columns: warp w takes j = w, w + 4, ...
  float o = 0.0f;
  for (int j = warp; !raw && j < rV; j += kCombWarps) o = fmaf(Ms[j][lane], y[j], o);
  osh[warp][lane] = o;
  __syncthreads();
  if (warp == 0) {
    const float v = raw ? y[cb * kCombCols + lane] : (osh[0][lane] + osh[1][lane]) + (osh[2][lane] + osh[3][lane]);
    const size_t off = (static_cast<size_t>(s) * Hq + qh) * kD + cb * kCombCols + lane;
    if (ca.out_bf16)
      static_cast<__nv_bfloat16*>(ca.out)[off] = __float2bfloat16_rn(v);
    else
      static_cast<float*>(ca.out)[off] = v;
  }
}

// Width class of a code: 2, 4 and 8 have specialised extraction; others share the
// run-time path (class 0); kRawBits marks an uncompressed value unit.
int width_class(int b) { return (b == 2 || b == 4 || b == 8 || b == kRawBits) ? b : 0; }

// Cost model of one page for the split allocation (warp instructions per page and warp:
// softmax, bookkeeping and the per-16-coordinate MMA rows).
constexpr double kPageCost = 320.0;
constexpr size_t kReadSlack = 2048;
constexpr double kTileCost = 56.0;

SplitFn split_fn(int bK, int bV, bool pack) {
  switch (width_class(bK)) {
    case 2: return split_fn_bk<2>(width_class(bV), pack);
    case 4: return split_fn_bk<4>(width_class(bV), pack);
    case 8: return split_fn_bk<8>(width_class(bV), pack);
    default: return split_fn_bk<0>(width_class(bV), pack);
  }
}

// Partial slots per query head: at most one context split per 8 pages (2 per warp).
int split_cap(int max_seq_len) {
  const int n_pages = std::max(1, (max_seq_len + kPage - 1) / kPage);
  return std::max(1, (n_pages + 7) / 8);
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

// Resident CTAs per SM of a kernel variant at a given dynamic shared-memory size (cached).
int occupancy(SplitFn fn, size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<const void*, size_t>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(reinterpret_cast<const void*>(fn), smem);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int n = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, smem) != cudaSuccess || n < 1) n = 1;
  cache[key] = n;
  return n;
}

// Launch with programmatic stream serialization: the kernel may start while the previous
// kernel in the stream finishes; it calls griddepcontrol.wait before reading its inputs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*fn)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
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

}  // namespace
}  // namespace dec
}  // namespace kvtc

using namespace kvtc;
using namespace kvtc::dec;

// Workspace: the partials [n_seq][Hq][cap][kPartStride] floats, then q~ [n_seq][Hq][128].
extern "C" uint64_t kvtc_decode_workspace_bytes(const kvtc_plan* plan, int n_seq, int max_seq_len) {
  if (!plan || n_seq < 1 || max_seq_len < 0) return 0;
  const uint64_t heads = static_cast<uint64_t>(n_seq) * plan->H * plan->G;
  return heads * (static_cast<uint64_t>(split_cap(max_seq_len)) * kPartStride + kD) * sizeof(float);
}

extern "C" kvtc_status kvtc_decode_attention(const kvtc_plan* plan, const kvtc_cache* cache, int layer,
                                             const void* q, kvtc_dtype q_dtype, const int32_t* seq_lens,
                                             int max_seq_len, float softmax_scale, void* out,
                                             kvtc_dtype out_dtype, void* workspace, uint64_t workspace_bytes,
                                             void* stream) {
  kvtc_status st = check_uploaded(plan);
  if (st != KVTC_OK) return st;
  if (!cache || !cache->pool || !cache->block_table) return fail(KVTC_EINVAL, "cache is incomplete");
  if (layer < 0 || layer >= plan->L) return fail(KVTC_EINVAL, "layer out of range");
  if (!q || !seq_lens || !out || !workspace) return fail(KVTC_EINVAL, "null device pointer");
  if ((q_dtype != KVTC_F32 && q_dtype != KVTC_BF16) || (out_dtype != KVTC_F32 && out_dtype != KVTC_BF16))
    return fail(KVTC_EINVAL, "dtype must be F32 or BF16");
  if (cache->n_seq < 1 || cache->max_pages < 1 || max_seq_len < 0)
    return fail(KVTC_EINVAL, "bad sizes");
  if (max_seq_len > cache->max_pages * kPage) return fail(KVTC_EINVAL, "max_seq_len exceeds the block table");
  if (reinterpret_cast<uintptr_t>(cache->pool) & 15) return fail(KVTC_EINVAL, "pool must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(workspace) & 15) return fail(KVTC_EINVAL, "workspace must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(q) & 15) return fail(KVTC_EINVAL, "q must be 16-byte aligned");
  if (plan->H > kMaxHeadsPerLaunch) return fail(KVTC_EINVAL, "at most 64 KV heads per layer");
  const int n_seq = cache->n_seq;
  const uint64_t need = kvtc_decode_workspace_bytes(plan, n_seq, max_seq_len);
  if (workspace_bytes < need) return fail(KVTC_ECAPACITY, "decode workspace too small");
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(plan->d));
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int n_hg = (plan->G + 7) / 8;
  const int cap = split_cap(max_seq_len);
  const int max_pages_seq = std::max(1, (max_seq_len + kPage - 1) / kPage);
  const int part_stride = cap;
  const int Hq = plan->H * plan->G;
  float* parts = static_cast<float*>(workspace);
  float* qt = parts + static_cast<size_t>(n_seq) * Hq * cap * kPartStride;

  // ---- kernel 0: q~ = M_K q
  {
    PrepArgs pa;
    pa.units = plan->d_units;
    pa.layer = layer;
    pa.H = plan->H;
    pa.G = plan->G;
    pa.n_hg = n_hg;
    pa.q = q;
    pa.q_bf16 = q_dtype == KVTC_BF16;
    pa.qt = qt;
    cudaError_t e = launch_pdl(decode_prep_kernel, dim3(kD / 16, plan->H * n_hg, n_seq), dim3(128), 0, cs, pa);
    if (e != cudaSuccess) return cuda_fail(e, "decode prep launch");
  }

  // ---- kernel 1: split kernels.  The layer's KV heads are grouped by kernel variant
  // (width classes of b_K and b_V).  One launch per group; the launches run side by side,
  // so each gets the share of a wave of resident CTAs that its work is of the layer's,
  // and within a group each head gets context splits in proportion to its work per page.
  // The work of a page is mostly instruction issue, not bytes: the online softmax costs
  // the same for every head, and each 16 coordinates of K or V add one MMA row of work
  // per block, so a page's cost is modelled as kPageCost + kTileCost * (k-steps + m-tiles)
  // (warp instructions, from the kernel's instruction mix).
  const bool pack = plan->G <= 4;
  std::map<int, std::vector<int>> groups;
  std::vector<double> head_bytes_pp(plan->H), head_cost(plan->H);
  double layer_cost = 0.0;
  for (int h = 0; h < plan->H; ++h) {
    const int uK = (layer * plan->H + h) * 2;
    groups[width_class(plan->b[uK]) * 32 + width_class(plan->b[uK + 1])].push_back(h);
    head_bytes_pp[h] = 16.0 * (plan->r[uK] * plan->b[uK] + plan->r[uK + 1] * plan->b[uK + 1]);
    head_cost[h] = kPageCost + kTileCost * ((plan->r[uK] + 15) / 16 + (plan->r[uK + 1] + 15) / 16);
    layer_cost += head_cost[h];
  }
  CombineArgs ca;
  ca.units = plan->d_units;
  ca.layer = layer;
  ca.H = plan->H;
  ca.G = plan->G;
  ca.part_stride = part_stride;
  ca.ws = parts;
  ca.out = out;
  ca.out_bf16 = out_dtype == KVTC_BF16;
  ca.status = cache->status;
  for (int h = 0; h < kMaxHeadsPerLaunch; ++h) ca.nparts[h] = 0;

  const size_t head_bytes = ((sizeof(SmemHead) + 8 * kWarps * 8 + 127) / 128) * 128;
  bool first = true;
  for (auto& kv : groups) {
    const int wk = kv.first >> 5, wv = kv.first & 31;
    const std::vector<int>& hs = kv.second;
    uint32_t stage_bytes = 0;
    double group_cost = 0.0;
    for (int h : hs) {
      stage_bytes = std::max(stage_bytes, (static_cast<uint32_t>(head_bytes_pp[h]) + 127u) / 128u * 128u);
      group_cost += head_cost[h];
    }
    // shared memory for kMinBlocks CTAs per SM where the pages allow it (228 KB per SM,
    // 1 KB of it reserved per CTA)
    const size_t budget = 233472 / kMinBlocks - 1024 - kReadSlack;
    int n_stage = budget > head_bytes
                      ? static_cast<int>((budget - head_bytes) / (static_cast<size_t>(kWarps) * stage_bytes))
                      : 0;
    n_stage = std::max(1, std::min(n_stage, 6));
    if (n_stage < 2) n_stage = std::min<int>(2, static_cast<int>((220 * 1024 - head_bytes) / (kWarps * stage_bytes)));
    n_stage = std::max(1, n_stage);
    // the stage region also holds the end-of-kernel merge of the four warps' partials
    const size_t merge_bytes = static_cast<size_t>(kWarps) * 8 * kPartStride * sizeof(float);
    // + slack: the kernel reads whole 16-row tiles, up to 2 KB past a page's last row
    const size_t smem = head_bytes + std::max<size_t>(static_cast<size_t>(kWarps) * n_stage * stage_bytes, merge_bytes) +
                        kReadSlack;
    SplitFn fn = split_fn(wk == 0 ? 3 : wk, wv == 0 ? 3 : wv, pack);
    if (!fn) return fail(KVTC_EINVAL, "no decode kernel for this code width");
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (decode)");
    const double share = group_cost / layer_cost;
    const int wave = static_cast<int>(occupancy(fn, smem) * sm_count() * share);
    const int columns = std::max(static_cast<int>(hs.size()), wave / std::max(1, n_hg * n_seq));
    DecodeArgs a;
    a.units = plan->d_units;
    a.layer = layer;
    a.H = plan->H;
    a.G = plan->G;
    a.n_hg = n_hg;
    a.n_heads = static_cast<int>(hs.size());
    a.part_stride = part_stride;
    // Splits per head: greedy on the modelled finishing time.  A head with s splits
    // gives each of its 4 s warps at most ceil(P / 4 s) pages, so it ends after about
    // ceil(P / 4 s) * cost; the column goes to the head that ends last, while columns
    // remain (and the head has at least 8 pages per split).
    std::vector<int> ns(hs.size(), 1);
    auto ends = [&](size_t i) {
      return std::ceil(static_cast<double>(max_pages_seq) / (kWarps * ns[i])) * head_cost[hs[i]];
    };
    for (int used = static_cast<int>(hs.size()); used < columns; ++used) {
      size_t best = hs.size();
      for (size_t i = 0; i < hs.size(); ++i)
        if (ns[i] < cap && (best == hs.size() || ends(i) > ends(best))) best = i;
      if (best == hs.size()) break;
      ++ns[best];
    }
    a.split_prefix[0] = 0;
    for (size_t i = 0; i < hs.size(); ++i) {
      a.heads[i] = hs[i];
      a.split_prefix[i + 1] = a.split_prefix[i] + ns[i];
      ca.nparts[hs[i]] = ns[i];
    }
    a.qt = qt;
    a.wait_first = first ? 1 : 0;
    a.seq_lens = seq_lens;
    a.n_seq = n_seq;
    a.pool = static_cast<const char*>(cache->pool);
    a.pages_per_unit = cache->pages_per_unit;
    a.block_table = cache->block_table;
    a.max_pages = cache->max_pages;
    a.status = cache->status;
    a.scale = scale;
    a.n_stage = n_stage;
    a.stage_bytes = stage_bytes;
    a.ws = parts;
    dim3 grid(a.split_prefix[hs.size()], n_hg, n_seq);
    e = launch_pdl(fn, grid, dim3(kThreads), smem, cs, a);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    first = false;
  }

  // ---- kernel 2: combine
  {
    cudaError_t e = launch_pdl(decode_combine_kernel, dim3(Hq, n_seq, kD / kCombCols), dim3(kCombThreads), 0, cs, ca);
    if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return KVTC_OK;
}
