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
#include <vector>

#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
namespace {

// o[s][qh][:] from the partials of every split and warp.
__global__ void __launch_bounds__(128) decode_combine_kernel(const UnitDesc* units, int layer, int H, int G,
                                                             int n_part, const float* ws, void* out,
                                                             int out_bf16) {
  __shared__ float wgt[1024];
  __shared__ float y[128];
  __shared__ float red[4];
  const int qh = blockIdx.x, s = blockIdx.y, tid = threadIdx.x;
  const int Hq = H * G, h = qh / G;
  const UnitDesc dV = units[(layer * H + h) * 2 + 1];
  const float* base = ws + (static_cast<size_t>(s) * Hq + qh) * n_part * kPartStride;
  // global max of the partial maxima (log2 domain)
  float mx = -INFINITY;
  for (int i = tid; i < n_part; i += 128) mx = fmaxf(mx, base[static_cast<size_t>(i) * kPartStride]);
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float lsum = 0.0f;
  for (int i = tid; i < n_part; i += 128) {
    const float mi = base[static_cast<size_t>(i) * kPartStride];
    const float wi = mi == -INFINITY ? 0.0f : exp2f(mi - mx);
    if (i < 1024) wgt[i] = wi;
    lsum += wi * base[static_cast<size_t>(i) * kPartStride + 1];
  }
  for (int o = 16; o; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  if ((tid & 31) == 0) red[tid >> 5] = lsum;
  __syncthreads();
  const float L = red[0] + red[1] + red[2] + red[3];
  const int rV = dV.r;
  const float mV = 0.5f * static_cast<float>((1 << dV.b) - 1);
  if (tid < rV) {
    float zs = 0.0f;
    for (int i = 0; i < n_part; ++i) {
      const float mi = base[static_cast<size_t>(i) * kPartStride];
      const float wi = i < 1024 ? wgt[i] : (mi == -INFINITY ? 0.0f : exp2f(mi - mx));
      if (wi != 0.0f) zs += wi * base[static_cast<size_t>(i) * kPartStride + 2 + tid];
    }
    // z holds sum p*c*2^-17 (uncentered codes); center and dequantize
    y[tid] = L > 0.0f ? dV.delta * (ldexpf(zs, 17) - mV * L) / L : 0.0f;
  }
  __syncthreads();
  float o = 0.0f;
  for (int j = 0; j < rV; ++j) o = fmaf(dV.M[static_cast<size_t>(j) * kD + tid], y[j], o);
  const size_t off = (static_cast<size_t>(s) * Hq + qh) * kD + tid;
  if (out_bf16)
    static_cast<__nv_bfloat16*>(out)[off] = __float2bfloat16_rn(o);
  else
    static_cast<float*>(out)[off] = o;
}


SplitFn split_fn(int bK, int bV) {
  switch (bK) {
    case 2: return split_fn_bk<2>(bV);
    case 3: return split_fn_bk<3>(bV);
    case 4: return split_fn_bk<4>(bV);
    case 5: return split_fn_bk<5>(bV);
    case 6: return split_fn_bk<6>(bV);
    case 7: return split_fn_bk<7>(bV);
    default: return split_fn_bk<8>(bV);
  }
}

struct SplitPlan {
  int n_split, pages_per_split, n_hg;
};

SplitPlan split_plan(const kvtc_plan* plan, int n_seq, int max_seq_len) {
  SplitPlan sp;
  sp.n_hg = (plan->G + 7) / 8;
  const int n_pages = std::max(1, (max_seq_len + kPage - 1) / kPage);
  const long long ctas_per_split = static_cast<long long>(n_seq) * plan->H * sp.n_hg;
  int ns = static_cast<int>(std::max(1ll, (kTargetCtas + ctas_per_split - 1) / ctas_per_split));
  ns = std::min(ns, std::max(1, (n_pages + kWarps - 1) / kWarps));
  sp.pages_per_split = (n_pages + ns - 1) / ns;
  sp.n_split = (n_pages + sp.pages_per_split - 1) / sp.pages_per_split;
  return sp;
}

}  // namespace
}  // namespace dec
}  // namespace kvtc

using namespace kvtc;
using namespace kvtc::dec;

extern "C" uint64_t kvtc_decode_workspace_bytes(const kvtc_plan* plan, int n_seq, int max_seq_len) {
  if (!plan || n_seq < 1 || max_seq_len < 0) return 0;
  const SplitPlan sp = split_plan(plan, n_seq, max_seq_len);
  return static_cast<uint64_t>(n_seq) * plan->H * plan->G * sp.n_split * kWarps * kPartStride * sizeof(float);
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
  const int n_seq = cache->n_seq;
  const uint64_t need = kvtc_decode_workspace_bytes(plan, n_seq, max_seq_len);
  if (workspace_bytes < need) return fail(KVTC_ECAPACITY, "decode workspace too small");
  const SplitPlan sp = split_plan(plan, n_seq, max_seq_len);
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(plan->d));
  cudaStream_t cs = static_cast<cudaStream_t>(stream);

  // Group the layer's KV heads by (b_K, b_V): one launch per group.
  std::map<int, std::vector<int>> groups;
  uint32_t max_stage = 0;
  for (int h = 0; h < plan->H; ++h) {
    const int uK = (layer * plan->H + h) * 2;
    groups[plan->b[uK] * 16 + plan->b[uK + 1]].push_back(h);
  }
  for (auto& kv : groups) {
    uint32_t stage_bytes = 0;
    for (int h : kv.second) {
      const int uK = (layer * plan->H + h) * 2;
      const uint32_t sb = static_cast<uint32_t>(16 * (plan->r[uK] * plan->b[uK] + plan->r[uK + 1] * plan->b[uK + 1]));
      stage_bytes = std::max(stage_bytes, (sb + 127u) / 128u * 128u);
    }
    const size_t head_bytes = ((sizeof(SmemHead) + 8 * kWarps * 8 + 127) / 128) * 128;
    const size_t budget = 200 * 1024;
    int n_stage = static_cast<int>((budget - head_bytes) / (static_cast<size_t>(kWarps) * stage_bytes));
    n_stage = std::max(1, std::min(n_stage, 6));
    const size_t smem = head_bytes + static_cast<size_t>(kWarps) * n_stage * stage_bytes;
    const std::vector<int>& hs = kv.second;
    for (size_t base = 0; base < hs.size(); base += kMaxHeadsPerLaunch) {
      DecodeArgs a;
      a.units = plan->d_units;
      a.layer = layer;
      a.H = plan->H;
      a.G = plan->G;
      a.n_hg = sp.n_hg;
      a.n_heads = static_cast<int>(std::min<size_t>(kMaxHeadsPerLaunch, hs.size() - base));
      for (int i = 0; i < a.n_heads; ++i) a.heads[i] = hs[base + i];
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
      a.n_split = sp.n_split;
      a.pages_per_split = sp.pages_per_split;
      a.n_stage = n_stage;
      a.stage_bytes = stage_bytes;
      a.ws = static_cast<float*>(workspace);
      SplitFn fn = split_fn(kv.first >> 4, kv.first & 15);
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (decode)");
      dim3 grid(sp.n_split, a.n_heads * sp.n_hg, n_seq);
      fn<<<grid, kThreads, smem, cs>>>(a);
      e = cudaGetLastError();
      if (e != cudaSuccess) return cuda_fail(e, "decode launch");
      max_stage = std::max(max_stage, stage_bytes);
    }
  }
  (void)max_stage;
  dim3 cgrid(plan->H * plan->G, n_seq);
  decode_combine_kernel<<<cgrid, 128, 0, cs>>>(plan->d_units, layer, plan->H, plan->G, sp.n_split * kWarps,
                                               static_cast<const float*>(workspace), out, out_dtype == KVTC_BF16);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  return KVTC_OK;
}
