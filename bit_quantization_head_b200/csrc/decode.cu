// kvtc_decode_attention: one decode step of attention over the packed code cache.
//
// KV-COBRA project page, "Efficiency": the cache is stored as packed b-bit codes with the
// rotation folded into the basis, so dequantization and the inverse rotation run in one
// fused pass.  Here the inverse key rotation is folded into the query (q~ = M_K q, the
// same algebra as NOVA-KV's query-side fold on the pith.science review page) and values
// are accumulated in their latent basis, back-projected once per query head.
//
// Kernel 1 (decode_split_kernel<BK, BV>): CTA = (context split, KV head, sequence), four
// warps, each streaming its own pages through a ring of cp.async.bulk + mbarrier stages.
// Per 16-token block a warp computes the G (<= 8) query heads' scores with m16n8k16
// tensor-core MMAs whose A operand is taken directly from the packed words: one AND
// leaves each code c in the low mantissa bits of an fp16 half, i.e. the subnormal
// c * 2^(e-24) (exact), with e the field's bit offset; e is undone per row in fp32.
// q~ is split into fp16 hi + lo (about 22 bits).  Online softmax per block; P goes to
// fp16 (scaled by 2^(7-e) so P * A = p * c * 2^-17 whatever e is), is transposed into
// the B fragment with movmatrix, and multiplies the value codes (A = V codes, rows =
// latent coordinates) into fp32 accumulators.  Each warp writes (m, l, z) partials.
// Kernel 2 (decode_combine_kernel): log-sum-exp merge of the partials, centering
// (z - m_V * l), dequantization (delta_V) and the back-projection o = M_V^T y.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <utility>
#include <vector>

#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
namespace {

// o[s][qh][:] from the partials of every split and warp.  Each warp folds a quarter of
// the partials (lane l holds latent coordinates 4l..4l+3), the warps' sums meet in shared
// memory, then every thread back-projects one output coordinate.
struct CombineArgs {
  const UnitDesc* units;
  int layer, H, G;
  int part_stride;                    // partial slots per query head
  int nparts[kMaxHeadsPerLaunch];     // partials written for each KV head
  const float* ws;
  void* out;
  int out_bf16;
};

__global__ void __launch_bounds__(128) decode_combine_kernel(const __grid_constant__ CombineArgs ca) {
  griddep_wait();
  griddep_launch_dependents();
  const UnitDesc* units = ca.units;
  const int layer = ca.layer, H = ca.H, G = ca.G;
  const float* ws = ca.ws;
  void* out = ca.out;
  const int out_bf16 = ca.out_bf16;
  __shared__ float zsh[4][128];
  __shared__ float lsh[4];
  __shared__ float mxsh[4];
  __shared__ float y[128];
  const int qh = blockIdx.x, s = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = H * G, h = qh / G;
  const UnitDesc dV = units[(layer * H + h) * 2 + 1];
  const int n_part = ca.nparts[h];
  const float* base = ws + (static_cast<size_t>(s) * Hq + qh) * ca.part_stride * kPartStride;
  // global max of the partial maxima (log2 domain)
  float mx = -INFINITY;
  for (int i = tid; i < n_part; i += 128) mx = fmaxf(mx, base[static_cast<size_t>(i) * kPartStride]);
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) mxsh[warp] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(mxsh[0], mxsh[1]), fmaxf(mxsh[2], mxsh[3]));
  const int rV = dV.r;
  float4 zacc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  float lacc = 0.0f;
#pragma unroll 4
  for (int i = warp; i < n_part; i += 4) {
    const float* pp = base + static_cast<size_t>(i) * kPartStride;
    const float mi = pp[0];
    const float wi = mi == -INFINITY ? 0.0f : exp2f(mi - mx);
    const float4 z4 = 4 * lane < rV ? reinterpret_cast<const float4*>(pp + 4)[lane] : make_float4(0, 0, 0, 0);
    lacc = fmaf(wi, pp[1], lacc);
    zacc.x = fmaf(wi, z4.x, zacc.x);
    zacc.y = fmaf(wi, z4.y, zacc.y);
    zacc.z = fmaf(wi, z4.z, zacc.z);
    zacc.w = fmaf(wi, z4.w, zacc.w);
  }
  reinterpret_cast<float4*>(zsh[warp])[lane] = zacc;
  if (lane == 0) lsh[warp] = lacc;
  __syncthreads();
  const float L = lsh[0] + lsh[1] + lsh[2] + lsh[3];
  const float mV = 0.5f * static_cast<float>((1 << dV.b) - 1);
  if (tid < rV) {
    const float zs = zsh[0][tid] + zsh[1][tid] + zsh[2][tid] + zsh[3][tid];
    // z holds sum p*c*2^-17 (uncentered codes); center and dequantize
    y[tid] = L > 0.0f ? dV.delta * (ldexpf(zs, 17) - mV * L) / L : 0.0f;
  }
  __syncthreads();
  float o0 = 0.0f, o1 = 0.0f, o2 = 0.0f, o3 = 0.0f;
  int j = 0;
  for (; j + 4 <= rV; j += 4) {
    o0 = fmaf(dV.M[static_cast<size_t>(j) * kD + tid], y[j], o0);
    o1 = fmaf(dV.M[static_cast<size_t>(j + 1) * kD + tid], y[j + 1], o1);
    o2 = fmaf(dV.M[static_cast<size_t>(j + 2) * kD + tid], y[j + 2], o2);
    o3 = fmaf(dV.M[static_cast<size_t>(j + 3) * kD + tid], y[j + 3], o3);
  }
  for (; j < rV; ++j) o0 = fmaf(dV.M[static_cast<size_t>(j) * kD + tid], y[j], o0);
  const float o = (o0 + o1) + (o2 + o3);
  const size_t off = (static_cast<size_t>(s) * Hq + qh) * kD + tid;
  if (out_bf16)
    static_cast<__nv_bfloat16*>(out)[off] = __float2bfloat16_rn(o);
  else
    static_cast<float*>(out)[off] = o;
}

// Width class of a code: 2, 4 and 8 have specialised extraction; others share the
// run-time path (class 0).
int width_class(int b) { return (b == 2 || b == 4 || b == 8) ? b : 0; }

SplitFn split_fn(int bK, int bV, bool pack, bool small) {
  switch (width_class(bK)) {
    case 2: return split_fn_bk<2>(width_class(bV), pack, small);
    case 4: return split_fn_bk<4>(width_class(bV), pack, small);
    case 8: return split_fn_bk<8>(width_class(bV), pack, small);
    default: return split_fn_bk<0>(width_class(bV), pack, small);
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
  static std::map<std::pair<const void*, size_t>, int> cache;
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

extern "C" uint64_t kvtc_decode_workspace_bytes(const kvtc_plan* plan, int n_seq, int max_seq_len) {
  if (!plan || n_seq < 1 || max_seq_len < 0) return 0;
  return static_cast<uint64_t>(n_seq) * plan->H * plan->G * split_cap(max_seq_len) * kWarps * kPartStride *
         sizeof(float);
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
  const int n_seq = cache->n_seq;
  const uint64_t need = kvtc_decode_workspace_bytes(plan, n_seq, max_seq_len);
  if (workspace_bytes < need) return fail(KVTC_ECAPACITY, "decode workspace too small");
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(plan->d));
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int n_hg = (plan->G + 7) / 8;
  const int cap = split_cap(max_seq_len);
  const int part_stride = cap * kWarps;

  // Group the layer's KV heads by kernel variant: width classes of b_K and b_V, and the
  // rank class (both ranks <= 64 use the 4-tile variant).  One launch per group, sized to
  // one wave of resident CTAs; within a group each head gets context splits in proportion
  // to its bytes per page.
  const bool pack = plan->G <= 4;
  std::map<int, std::vector<int>> groups;
  for (int h = 0; h < plan->H; ++h) {
    const int uK = (layer * plan->H + h) * 2;
    const bool small = plan->r[uK] <= 64 && plan->r[uK + 1] <= 64;
    groups[(width_class(plan->b[uK]) * 16 + width_class(plan->b[uK + 1])) * 2 + (small ? 1 : 0)].push_back(h);
  }
  CombineArgs ca;
  ca.units = plan->d_units;
  ca.layer = layer;
  ca.H = plan->H;
  ca.G = plan->G;
  ca.part_stride = part_stride;
  ca.ws = static_cast<const float*>(workspace);
  ca.out = out;
  ca.out_bf16 = out_dtype == KVTC_BF16;
  for (int h = 0; h < kMaxHeadsPerLaunch; ++h) ca.nparts[h] = 0;
  if (plan->H > kMaxHeadsPerLaunch) return fail(KVTC_EINVAL, "at most 64 KV heads per layer");

  const size_t head_bytes = ((sizeof(SmemHead) + 8 * kWarps * 8 + 127) / 128) * 128;
  for (auto& kv : groups) {
    const bool small = kv.first & 1;
    const int wk = (kv.first >> 1) >> 4, wv = (kv.first >> 1) & 15;
    const std::vector<int>& hs = kv.second;
    uint32_t stage_bytes = 0;
    std::vector<double> bytes(hs.size());
    double total_bytes = 0.0;
    for (size_t i = 0; i < hs.size(); ++i) {
      const int uK = (layer * plan->H + hs[i]) * 2;
      const uint32_t sb = static_cast<uint32_t>(16 * (plan->r[uK] * plan->b[uK] + plan->r[uK + 1] * plan->b[uK + 1]));
      stage_bytes = std::max(stage_bytes, (sb + 127u) / 128u * 128u);
      bytes[i] = sb;
      total_bytes += sb;
    }
    // shared memory for three CTAs per SM where the pages allow it
    const size_t budget = 74 * 1024;
    int n_stage = budget > head_bytes
                      ? static_cast<int>((budget - head_bytes) / (static_cast<size_t>(kWarps) * stage_bytes))
                      : 0;
    n_stage = std::max(1, std::min(n_stage, 6));
    if (n_stage < 2) n_stage = std::min<int>(2, static_cast<int>((220 * 1024 - head_bytes) / (kWarps * stage_bytes)));
    n_stage = std::max(1, n_stage);
    const size_t smem = head_bytes + static_cast<size_t>(kWarps) * n_stage * stage_bytes;
    SplitFn fn = split_fn(wk == 0 ? 3 : wk, wv == 0 ? 3 : wv, pack, small);
    if (!fn) return fail(KVTC_EINVAL, "no decode kernel for this code width");
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (decode)");
    const int wave = occupancy(fn, smem) * sm_count();
    const int columns = std::max(static_cast<int>(hs.size()), wave / std::max(1, n_hg * n_seq));
    DecodeArgs a;
    a.units = plan->d_units;
    a.layer = layer;
    a.H = plan->H;
    a.G = plan->G;
    a.n_hg = n_hg;
    a.n_heads = static_cast<int>(hs.size());
    a.part_stride = part_stride;
    a.split_prefix[0] = 0;
    for (size_t i = 0; i < hs.size(); ++i) {
      a.heads[i] = hs[i];
      int ns = static_cast<int>(std::floor(columns * bytes[i] / total_bytes));
      ns = std::max(1, std::min(ns, cap));
      a.split_prefix[i + 1] = a.split_prefix[i] + ns;
      ca.nparts[hs[i]] = ns * kWarps;
    }
    a.q = q;
    a.q_bf16 = q_dtype == KVTC_BF16;
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
    a.ws = static_cast<float*>(workspace);
    dim3 grid(a.split_prefix[hs.size()], n_hg, n_seq);
    e = launch_pdl(fn, grid, dim3(kThreads), smem, cs, a);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  }
  dim3 cgrid(plan->H * plan->G, n_seq);
  {
    cudaError_t e = launch_pdl(decode_combine_kernel, cgrid, dim3(128), 0, cs, ca);
    if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  return KVTC_OK;
}
