// kvtc_decode_attention: one decode step of attention over the packed code cache.
//
// KV-COBRA project page, "Efficiency": the cache is stored as packed b-bit codes with the
// rotation folded into the basis, so dequantization and the inverse rotation run in one
// fused pass.  Here the inverse key rotation is folded into the query (q~ = M_K q, the
// same algebra as NOVA-KV's query-side fold on the pith.science review page) and values
// are accumulated in their latent basis, back-projected once per query head.
//
// One kernel launch per layer and (b_K, b_V) group (decode_split_kernel<BK, BV, PACK>,
// decode_kernel.cuh): every CTA forms q~ for its heads on the tensor cores, streams its
// share of the context's pages (split-K), and writes a partial (m, l, z); the last CTAs to
// complete a (sequence, KV head, head group) merge the partials and back-project, each
// for a share of its query heads.
// The launches use programmatic dependent launch, so their set-up (plan reads, barrier
// initialisation, L2 prefetch of M_V) overlaps the tail of the preceding kernel.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <utility>
#include <vector>

#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
namespace {

// Cost model of one page for the split allocation (warp instructions per page and warp:
// softmax, bookkeeping and the per-16-coordinate MMA rows; a code width with minor parts
// adds a shift and an AND-OR per part to every A register of its rows).
constexpr double kPageCost = 320.0;
constexpr size_t kReadSlack = 2048;
constexpr double kTileCost = 56.0;
constexpr double kMinorCost = 24.0;
constexpr size_t kSmemPerSM = 233472;  // 228 KB of shared memory per SM
constexpr size_t kSmemReserved = 1024; // reserved by the system per resident CTA

// The kernel variant of a (b_K, b_V) pair: b_K in 2..8; b_V in 2..8 or kRawBits.
SplitFn split_fn(int bK, int bV, bool pack) {
  switch (bK) {
    case 2: return split_fn_bk<2>(bV, pack);
    case 3: return split_fn_bk<3>(bV, pack);
    case 4: return split_fn_bk<4>(bV, pack);
    case 5: return split_fn_bk<5>(bV, pack);
    case 6: return split_fn_bk<6>(bV, pack);
    case 7: return split_fn_bk<7>(bV, pack);
    case 8: return split_fn_bk<8>(bV, pack);
    default: return nullptr;
  }
}

double tile_cost(int b) { return kTileCost + kMinorCost * (b == kRawBits ? 0 : n_minor(b)); }

// Partial slots per query head: at most one context split per 8 pages (2 per warp), and
// at most kMaxSplits.
int split_cap(int max_seq_len) {
  const int n_pages = std::max(1, (max_seq_len + kPage - 1) / kPage);
  return std::max(1, std::min(kMaxSplits, (n_pages + 7) / 8));
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

size_t tickets_bytes(const kvtc_plan* plan, int n_seq) {
  const size_t n = static_cast<size_t>(n_seq) * plan->H * ((plan->G + 7) / 8) * kTicketInts;
  return (n * sizeof(int) + 255) / 256 * 256;
}

}  // namespace
}  // namespace dec

// The decode launches of every layer: heads grouped by the kernel variant of their
// (b_K, b_V) pair, the stage size of each group, and the stage count and
// occupancy that fit (the most CTAs per SM, up to three, that leave a stage per warp).
// Sets each variant's shared-memory attribute once, here, so decode calls do no host
// allocation and no attribute calls.
kvtc_status prepare_decode(kvtc_plan* plan) {
  using namespace dec;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "device query (decode)");
  plan->sm_count = std::max(1, sms);
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || optin <= 0)
    optin = 232448;
  plan->dec_groups.assign(plan->L, {});
  const bool pack = plan->G <= 4;
  // the epilogue's scratch: the warps' partials, then the merge
  const size_t merge_bytes = std::max<size_t>(static_cast<size_t>(kWarps) * 8 * kPartStride, kMergeFloats) * sizeof(float);
  for (int layer = 0; layer < plan->L; ++layer) {
    std::vector<DecodeGroup>& gs = plan->dec_groups[layer];
    for (int h = 0; h < plan->H; ++h) {
      const int uK = (layer * plan->H + h) * 2;
      const int wk = plan->b[uK], wv = plan->b[uK + 1];
      auto it = std::find_if(gs.begin(), gs.end(), [&](const DecodeGroup& x) { return x.wk == wk && x.wv == wv; });
      if (it == gs.end()) {
        gs.emplace_back();
        it = gs.end() - 1;
        it->wk = wk;
        it->wv = wv;
      }
      it->heads.push_back(h);
      it->cost.push_back(kPageCost + tile_cost(wk) * ((plan->r[uK] + 15) / 16) +
                         tile_cost(wv) * ((plan->r[uK + 1] + 15) / 16));
      const uint32_t pb = static_cast<uint32_t>(16 * (plan->r[uK] * plan->b[uK] + plan->r[uK + 1] * plan->b[uK + 1]));
      it->stage_bytes = std::max(it->stage_bytes, (pb + 127u) / 128u * 128u);
    }
    for (DecodeGroup& gr : gs) {
      if (static_cast<int>(gr.heads.size()) > kMaxHeadsPerLaunch) return fail(KVTC_EINVAL, "at most 64 KV heads per layer");
      SplitFn fn = split_fn(gr.wk, gr.wv, pack);
      if (!fn) return fail(KVTC_EINVAL, "no decode kernel for this code width");
      gr.fn = reinterpret_cast<const void*>(fn);
      // the most CTAs per SM that leave at least one stage per warp (more resident warps
      // beat deeper rings: with one stage a warp waits for its next page, but the other
      // warps of the SM keep the pipes and the memory system busy)
      int n_stage = 0, target = kMinBlocks;
      for (; target >= 1 && n_stage < 1; --target) {
        const size_t budget = kSmemPerSM / target - kSmemReserved - kReadSlack - kHeadBytes;
        n_stage = static_cast<int>(budget / (static_cast<size_t>(kWarps) * gr.stage_bytes));
        if (n_stage >= 1) break;
      }
      if (n_stage < 1) return fail(KVTC_EINVAL, "a page of this plan does not fit in shared memory");
      // the ring of each warp takes the whole budget (up to six of the widest stages): the
      // kernel fits as many stages of its own head's pages as the ring holds
      gr.n_stage = std::min(n_stage, 6);
      // Every launch with the same CTAs per SM asks for the same shared memory, the whole
      // share of one CTA: the next layer's CTAs start while this layer's last ones run
      // (programmatic dependent launch), and a larger request than the one before could
      // not use the holes the earlier CTAs leave, stranding a few CTAs for a second wave.
      gr.smem = kSmemPerSM / target - kSmemReserved;
      const size_t need = kHeadBytes + std::max<size_t>(static_cast<size_t>(kWarps) * gr.n_stage * gr.stage_bytes, merge_bytes) +
                          kReadSlack;  // + slack: the kernel reads whole 16-row tiles, up to 2 KB past a page's last row
      if (need > gr.smem || gr.smem > static_cast<size_t>(optin))
        return fail(KVTC_EINVAL, "a page of this plan does not fit in shared memory");
      // the attribute is per kernel, shared by every group and plan: allow the device's
      // opt-in maximum once (each launch still asks for its own size)
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (decode)");
      int occ = 1;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kThreads, gr.smem) != cudaSuccess || occ < 1) occ = 1;
      gr.per_sm = occ;
    }
  }
  return KVTC_OK;
}

}  // namespace kvtc

using namespace kvtc;
using namespace kvtc::dec;

// Workspace: the arrival tickets [n_seq][H][ceil(G/8)][kTicketInts] int32 (256-byte
// rounded), then the partials [n_seq][Hq][cap][kPartStride] floats.
extern "C" uint64_t kvtc_decode_workspace_bytes(const kvtc_plan* plan, int n_seq, int max_seq_len) {
  if (!plan || n_seq < 1 || max_seq_len < 0) return 0;
  const uint64_t heads = static_cast<uint64_t>(n_seq) * plan->H * plan->G;
  return tickets_bytes(plan, n_seq) +
         heads * static_cast<uint64_t>(split_cap(max_seq_len)) * kPartStride * sizeof(float);
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
  const int n_seq = cache->n_seq;
  const uint64_t need = kvtc_decode_workspace_bytes(plan, n_seq, max_seq_len);
  if (workspace_bytes < need) return fail(KVTC_ECAPACITY, "decode workspace too small");
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(plan->d));
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int n_hg = (plan->G + 7) / 8;
  const int cap = split_cap(max_seq_len);
  const int max_pages_seq = std::max(1, (max_seq_len + kPage - 1) / kPage);
  int* tickets = static_cast<int*>(workspace);
  float* parts = reinterpret_cast<float*>(static_cast<char*>(workspace) + tickets_bytes(plan, n_seq));

  // One launch per (b_K, b_V) group; the launches run side by side, so each gets the
  // share of a wave of resident CTAs that its work is of the layer's, and within a group
  // each head gets context splits in proportion to its work per page.  The work of a page
  // is mostly instruction issue, not bytes: the online softmax costs the same for every
  // head, and each 16 coordinates of K or V add one MMA row of work per block, so a
  // page's cost is modelled as kPageCost + kTileCost * (k-steps + m-tiles).
  const std::vector<DecodeGroup>& groups = plan->dec_groups[layer];
  double layer_cost = 0.0;
  for (const DecodeGroup& gr : groups)
    for (double c : gr.cost) layer_cost += c;
  bool first = true;
  for (const DecodeGroup& gr : groups) {
    const int nh = static_cast<int>(gr.heads.size());
    double group_cost = 0.0;
    for (double c : gr.cost) group_cost += c;
    const double share = group_cost / layer_cost;
    const int rows = std::max(1, n_hg * n_seq);
    const int wave = static_cast<int>(gr.per_sm * plan->sm_count * share);
    const int columns = std::max(nh, wave / rows);
    DecodeArgs a;
    a.units = plan->d_units;
    a.layer = layer;
    a.H = plan->H;
    a.G = plan->G;
    a.n_hg = n_hg;
    a.n_heads = nh;
    a.part_stride = cap;
    // Splits per head: greedy on the modelled finishing time.  A head with s splits
    // gives each of its 4 s warps at most ceil(P / 4 s) pages, so it ends after about
    // ceil(P / 4 s) * cost; the column goes to the head that ends last, while columns
    // remain (and the head has at least 8 pages per split).
    int ns[kMaxHeadsPerLaunch];
    for (int i = 0; i < nh; ++i) ns[i] = 1;
    auto ends = [&](int i) { return std::ceil(static_cast<double>(max_pages_seq) / (kWarps * ns[i])) * gr.cost[i]; };
    for (int used = nh; used < columns; ++used) {
      int best = -1;
      for (int i = 0; i < nh; ++i)
        if (ns[i] < cap && (best < 0 || ends(i) > ends(best))) best = i;
      if (best < 0) break;
      ++ns[best];
    }
    a.split_prefix[0] = 0;
    for (int i = 0; i < nh; ++i) {
      a.heads[i] = gr.heads[i];
      a.split_prefix[i + 1] = a.split_prefix[i] + ns[i];
    }
    a.q = q;
    a.q_bf16 = q_dtype == KVTC_BF16;
    a.out = out;
    a.out_bf16 = out_dtype == KVTC_BF16;
    a.wait_first = first ? 1 : 0;
    a.seq_lens = seq_lens;
    a.n_seq = n_seq;
    a.pool = static_cast<const char*>(cache->pool);
    a.pages_per_unit = cache->pages_per_unit;
    a.block_table = cache->block_table;
    a.max_pages = cache->max_pages;
    a.part_pages = max_pages_seq;
    a.status = cache->status;
    a.scale = scale;
    a.n_stage = gr.n_stage;
    a.stage_bytes = gr.stage_bytes;
    a.tickets = tickets;
    a.ws = parts;
    dim3 grid(a.split_prefix[nh], n_hg, n_seq);
    cudaError_t e = launch_pdl(reinterpret_cast<SplitFn>(const_cast<void*>(gr.fn)), grid, dim3(kThreads), gr.smem, cs, a);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    first = false;
  }
  return KVTC_OK;
}
