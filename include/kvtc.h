/*
 * kvtc.h -- C ABI of the KV-COBRA transform-coded KV cache for NVIDIA B200 (sm_100a).
 *
 * The method (KV-COBRA project page, "KV-COBRA: KV Cache Compression via Co-Optimized
 * Bit-Rank Allocation"):
 *   calibrate once ("How KV-COBRA Works": per-head SVD of prefill keys, a two-level
 *   C1+C2 allocator freezes the basis, rank r* and bit-width b* of every head),
 *   encode every token ("Inference": rotate and truncate with H.V^T, quantize with the
 *   head's b*-bit quantizer), and read the cache with one fused pass ("Efficiency":
 *   packed b-bit codes, dequantization and inverse rotation fused).
 *
 * Vocabulary.  A *unit* is one (layer, KV head, kind) with kind K (keys) or V (values);
 * unit index u = ((layer * n_kv_heads) + head) * 2 + kind.  d = head dimension (128).
 * G = query heads per KV head.  Unit u keeps r_u coordinates (r even, 2..d) at b_u bits
 * (2..8): R_u = r_u * b_u bits per token; in keys-only plans a value unit is stored
 * uncompressed (r = d, b = KVTC_RAW_BITS, fp16).  A *page* holds 128 tokens of one unit
 * and is exactly 16 * R_u bytes (no per-token overhead, the "0 per-token overhead"
 * figure).
 *
 * Conventions for every call:
 *   - Every call returns a kvtc_status; nothing throws or exits across the ABI.  On an
 *     error the thread-local message of kvtc_last_error() says why.
 *   - Pointers documented "device" are CUDA device pointers of the current device;
 *     "host" pointers are ordinary memory.  The library never frees caller memory.
 *   - Calls that take a stream are asynchronous on that stream (a cudaStream_t passed as
 *     void*, NULL = the legacy default stream) and allocate nothing.
 *   - Kernels never trap.  Bad page ids, positions beyond the cache capacity and
 *     timed-out waits set bits of the caller's device status word (KVTC_STATUS_*) and
 *     the affected work is skipped (decode writes zeros for that query head).
 */
#ifndef KVTC_H
#define KVTC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVTC_VERSION 1
#define KVTC_PAGE_TOKENS 128
#define KVTC_HEAD_DIM 128

typedef enum {
  KVTC_OK = 0,
  KVTC_EINVAL = 1,       /* invalid argument (null pointer, size or range)            */
  KVTC_ENOMEM = 2,       /* host or device allocation failed                           */
  KVTC_ECUDA = 3,        /* a CUDA runtime call failed                                 */
  KVTC_EINFEASIBLE = 4,  /* budget below 4 bits per unit and token (r = b = 2)        */
  KVTC_ECAPACITY = 5,    /* workspace or cache smaller than the call needs            */
  KVTC_EVERSION = 6,     /* plan file of another format version                        */
  KVTC_EIO = 7,          /* plan file could not be read or written                     */
  KVTC_ESTATE = 8        /* plan not uploaded to the device (kvtc_plan_upload)         */
} kvtc_status;

typedef enum { KVTC_F32 = 0, KVTC_BF16 = 1 } kvtc_dtype;
typedef enum { KVTC_KIND_K = 0, KVTC_KIND_V = 1 } kvtc_kind;
typedef enum { KVTC_WEIGHTS_KL = 0, KVTC_WEIGHTS_MSE = 1 } kvtc_weight_mode;
/* C2 solver: the Lagrangian water-filling (mu bisected, exact on the convex hull), or the
 * pages' iterative form ("C2, across heads": marginal distortions equalized by a damped
 * update in five rounds): every unit sits where its marginal distortion on C1's
 * distortion-versus-budget hull falls to a common level mu, and five damped Newton steps
 * in log mu bring the level to the budget. */
typedef enum { KVTC_C2_LAGRANGE = 0, KVTC_C2_DAMPED = 1 } kvtc_c2_mode;

/* b of an uncompressed value unit (keys-only mode, kvtc_calib_desc.k_only): r = d = 128
 * and every value is stored as fp16 (round to nearest even).  Its page (128 tokens,
 * 32768 bytes = 16 * r * b like every page) has one row of 64 little-endian 32-bit words
 * per coordinate j; the word of token pair k (tokens 2k in the low half, 2k + 1 in the
 * high half) sits at position k XOR 4 (j mod 8) of row j.  The decode reads such a unit
 * as the integer code c = v * 2^24 with delta = 2^-24 and no centring. */
#define KVTC_RAW_BITS 16

/* Bits of the device status word. */
#define KVTC_STATUS_BAD_PAGE 1u      /* block table entry outside [0, pages_per_unit)  */
#define KVTC_STATUS_BAD_POS 2u       /* position or length beyond max_pages * 128      */
#define KVTC_STATUS_TIMEOUT 4u       /* a bounded wait on an mbarrier gave up          */

/* Thread-local description of the last error on this thread ("" if none). */
const char* kvtc_last_error(void);

/* Library format version (KVTC_VERSION) and whether the CUDA kernels were built in. */
int kvtc_version(void);

/* ------------------------------------------------------------------ calibration -- */

typedef struct kvtc_plan kvtc_plan;  /* opaque; owned by the library */

typedef struct {
  int n_layers;        /* L >= 1                                                     */
  int n_kv_heads;      /* H_kv >= 1                                                  */
  int group;           /* G >= 1 query heads per KV head                              */
  int head_dim;        /* d; must be 128                                             */
  int n_cal;           /* calibration tokens (and queries per query head) >= 2       */
  double bpd;          /* joint budget, bits per dimension over all 2*L*H_kv units    */
  int weight_mode;     /* KVTC_WEIGHTS_KL (keys: sigma^2_Q * sigma^2_K) or _MSE       */
  int fixed_r;         /* fixed_r > 0 and fixed_b > 0: every unit gets (fixed_r,       */
  int fixed_b;         /*   fixed_b) and no allocation runs                           */
  uint64_t seed;       /* seed of the random Hadamard signs (splitmix64)              */
  int c2_mode;         /* KVTC_C2_LAGRANGE (default) or KVTC_C2_DAMPED                */
  int k_only;          /* 1: keys-only ("k-only" results): the allocation covers the  */
                       /*   key units alone (bpd * d bits per key unit and token) and */
                       /*   every value unit is stored uncompressed (KVTC_RAW_BITS)   */
} kvtc_calib_desc;

/*
 * kvtc_calibrate -- "How KV-COBRA Works" (Calibration), "C1, per head", "C2, across
 * heads", "Hadamard rotation", "Attention-KL reordering"; joint K+V per the abstract.
 *
 * For every unit: eigen-decomposition of the uncentered calibration second moment;
 * weights w_i = sigma^2_Q,i * lambda_i for keys (KL mode; sigma^2_Q,i = mean squared
 * projection of the G query heads' calibration queries on eigenvector i) or
 * w_i = lambda_i (values, and keys in MSE mode); basis sorted by w descending.  Then
 * C2 (Lagrangian water-filling over all units, C1 as the per-unit solver) allocates
 * r*b per unit within bpd * d * (2*L*H_kv) bits; M_u = H_r diag(eps_u) V_r^T with
 * eps_u the splitmix64 signs; quantizer step delta_u = g(b) * sqrt(mean retained
 * eigenvalue), g(b) the MSE-optimal step of a 2^b-level uniform quantizer on N(0,1).
 *
 * k_cal, v_cal: host fp32 [L][H_kv][n_cal][d].  q_cal: host fp32 [L][H_kv][G][n_cal][d]
 * (may be NULL in MSE mode).  Borrowed for the call.  *out receives a new plan
 * (free with kvtc_plan_destroy).  Deterministic for the same inputs and seed; uses
 * host threads.  With k_only, fixed_r/fixed_b and the budget apply to the key units
 * only and each value unit gets r = d, b = KVTC_RAW_BITS, M = identity, delta = 2^-24.
 * Errors: EINVAL (shapes, d != 128, fixed_r odd or out of [2,d], fixed_b outside
 * [2,8]), EINFEASIBLE (budget < 4 bits per unit), ENOMEM.
 */
kvtc_status kvtc_calibrate(const kvtc_calib_desc* desc, const float* k_cal, const float* v_cal,
                           const float* q_cal, kvtc_plan** out);

/*
 * kvtc_plan_create -- a plan from explicit per-unit parameters (a plan computed
 * elsewhere).  r, b: host [U]; delta: host [U] (step; inv_delta = fp32(1/delta));
 * M: host fp32, the U matrices [r_u][d] concatenated in unit order.  U = 2*L*H_kv.
 * A value unit may be uncompressed (r = 128, b = KVTC_RAW_BITS; its M and delta are
 * then not used by the kernels).
 */
kvtc_status kvtc_plan_create(int n_layers, int n_kv_heads, int group, int head_dim,
                             const int* r, const int* b, const double* delta, const float* M,
                             kvtc_plan** out);

/* Frees the plan and its device copy.  NULL is a no-op. */
void kvtc_plan_destroy(kvtc_plan* plan);

typedef struct {
  int layer, head, kind;  /* kind: KVTC_KIND_K or KVTC_KIND_V                          */
  int r, b;               /* retained coordinates, bits per code                       */
  double delta;           /* quantizer step                                            */
  float inv_delta;        /* fp32(1/delta): the multiplier the encoder applies        */
  double sigma;           /* sqrt(mean of the retained eigenvalues)                    */
  double distortion;      /* D(r, b) = sum_{i>r} w_i + 2^(-2b)/12 * sum_{i<=r} w_i       */
  uint64_t page_bytes;    /* 16 * r * b                                                */
} kvtc_unit_info;

/* Model shape of a plan.  Any output pointer may be NULL. */
kvtc_status kvtc_plan_shape(const kvtc_plan* plan, int* n_layers, int* n_kv_heads, int* group,
                            int* head_dim, int* n_units);
/* Parameters of unit u (0 <= u < n_units). */
kvtc_status kvtc_plan_unit(const kvtc_plan* plan, int unit, kvtc_unit_info* out);
/* Copies M_u (fp32 [r_u][d], row-major) into host memory M_out. */
kvtc_status kvtc_plan_matrix(const kvtc_plan* plan, int unit, float* M_out);
/* Copies the sorted weights w (fp64 [d]) and matching eigenvalues lam (fp64 [d]) of
 * unit u; either pointer may be NULL.  Plans made by kvtc_plan_create have none (EINVAL). */
kvtc_status kvtc_plan_weights(const kvtc_plan* plan, int unit, double* w_out, double* lam_out);
/* The C2 multiplier mu* (0 for fixed or imported plans) and the total bits per token. */
kvtc_status kvtc_plan_budget(const kvtc_plan* plan, double* mu, uint64_t* total_bits);
/* Wall-clock seconds kvtc_calibrate spent on the per-unit statistics (second moments,
 * eigen-decompositions, weights; host threads) and on the allocation (C1 + C2, the step
 * the project page's "per-token overhead" figure times); 0 for imported plans.  Either
 * pointer may be NULL. */
kvtc_status kvtc_plan_calib_seconds(const kvtc_plan* plan, double* stats_s, double* alloc_s);

/* Versioned binary plan file: header, then per unit r, b, delta, inv_delta and M. */
kvtc_status kvtc_plan_save(const kvtc_plan* plan, const char* path);
kvtc_status kvtc_plan_load(const char* path, kvtc_plan** out);

/*
 * kvtc_plan_upload -- one-time copy of the per-unit descriptors and matrices
 * (M fp32 for decode, M rounded to bf16 for the bf16 encoder) into library-owned device
 * memory on the current device.  Not a hot call (it allocates).  Required before any
 * encode or decode; calling it again re-uploads.
 */
kvtc_status kvtc_plan_upload(kvtc_plan* plan, void* stream);

/* ------------------------------------------------------------------ cache -------- */

/*
 * The paged code cache ("Efficiency": packed b-bit codes; paging as in PagedAttention).
 * All memory is caller-owned.  Each unit has a pool of pages_per_unit pages; unit u's
 * pool starts at pool + pages_per_unit * (sum over u' < u of page_bytes(u')) and page p
 * of it at that + p * page_bytes(u).  block_table[s * max_pages + i] is the physical
 * page id of logical page i of sequence s, shared by all units.  The pool must be
 * 16-byte aligned and zero-filled before first use (slots not yet written are 0).
 *
 * Page layout (bit-exact; chosen so the decode kernel's tensor-core fragments read it
 * directly).  A b-bit code is split into parts of width 8, 4, 2 or 1 (the binary
 * expansion of b, lowest code bits first: 3 = 2+1, 5 = 4+1, 6 = 4+2, 7 = 4+2+1).  Part
 * p (width w, code bits [lo, lo+w)) lives in its own plane starting at byte 16*r*lo of
 * the page.  A plane is rows of little-endian 32-bit words; page bit k is bit k%32 of
 * word k/32.  Token t has pair index pi = 2*(t/16) + (t/8)%2.
 *   K unit: row rho < r/2 holds coordinates 2rho, 2rho+1 of all 128 tokens, 8w words.
 *     Owner o = t%8 owns words [o*w, (o+1)*w) of the row; the pair sits in word
 *     o*w + pi/(16/w) at bit offset (pi%(16/w))*w: coordinate 2rho in bits 0-15 of the
 *     word, coordinate 2rho+1 at the same offset + 16.
 *   V unit: row j < r holds coordinate j of all 128 tokens, 4w words.  Owner
 *     o = (t%8)/2 owns words [o*w, (o+1)*w); token t sits in word o*w + pi/(16/w) at
 *     bit offset (pi%(16/w))*w + 16*(t%2).
 */
typedef struct {
  void* pool;                   /* device                                           */
  uint64_t pages_per_unit;      /* capacity of every unit's pool, in pages          */
  const int32_t* block_table;   /* device int32 [n_seq][max_pages]                  */
  int n_seq;
  int max_pages;                /* logical pages per sequence in the table          */
  int32_t* status;              /* device int32 status word (KVTC_STATUS_*) or NULL */
} kvtc_cache;

/* Bytes of the whole pool for pages_per_unit pages per unit (0 if plan is NULL). */
uint64_t kvtc_cache_bytes(const kvtc_plan* plan, uint64_t pages_per_unit);
/* Byte offset of unit u's pool inside the pool buffer. */
uint64_t kvtc_unit_pool_offset(const kvtc_plan* plan, int unit, uint64_t pages_per_unit);

/* ------------------------------------------------------------------ encode ------- */

/*
 * kvtc_encode_append -- "Inference": each new key/value is rotated and truncated with
 * M_u = H.V_r^T and quantized with the unit's b-bit uniform quantizer, then written into
 * its page slot.  Canonical arithmetic (bit-exact with the oracle): for each retained
 * coordinate j, eight fp32 chains a_e = fma(x_k, M_jk, a_e) over k = e, e+8, ... in
 * ascending order (e = 0..7, each from 0), then y_j = ((a_0 + a_1) + (a_2 + a_3)) +
 * ((a_4 + a_5) + (a_6 + a_7)); M in the input's precision (bf16-rounded M for bf16
 * input, fp32 M for fp32);
 * code = min(max(floor(fl(fl(y * inv_delta) + 2^(b-1))), 0), 2^b - 1) (NaN -> 0).
 *
 * k, v: device [n_tok][H_kv][d] of dtype.  cu_seqlens: device int32 [n_seq + 1], the new
 * tokens of sequence s are rows cu_seqlens[s] .. cu_seqlens[s+1]-1 (cu_seqlens[0] = 0,
 * cu_seqlens[n_seq] = n_tok).  pos_start: device int32 [n_seq], cache position of each
 * sequence's first new token.  The slots written are overwritten (their old bits are
 * cleared, other tokens sharing a 32-bit word are kept).  Positions beyond
 * max_pages * 128 or page ids outside the pool set status bits and are skipped.
 * Calls that write the same slot and overlap on the GPU race.  An uncompressed value unit
 * (KVTC_RAW_BITS) receives fp16(v) (round to nearest even) in its raw page layout.
 */
kvtc_status kvtc_encode_append(const kvtc_plan* plan, const kvtc_cache* cache, int layer,
                               const void* k, const void* v, kvtc_dtype dtype,
                               const int32_t* cu_seqlens, const int32_t* pos_start, int n_tok,
                               void* stream);

/*
 * kvtc_encode_prefill -- the same codes as kvtc_encode_append for one sequence's
 * page-aligned span, computed as 128-token x d by d x r_u tensor-core GEMM tiles
 * (tcgen05, TMEM accumulators) whose epilogue quantizes and packs whole pages.  Any
 * coordinate whose tensor-core sum lies within the fp32 accumulation-error bound of a
 * quantizer threshold is recomputed in the canonical order, so the codes equal the
 * canonical ones bit for bit.  bf16 input only.  Plans with uncompressed value units
 * (keys-only) are not handled here (EINVAL): use kvtc_encode_append.
 * seq: sequence index; pos_start: host, multiple of 128; n_tok: host, > 0 (a trailing
 * partial page is written with the same merge rule as append).  k, v: device
 * [n_tok][H_kv][d] bf16.
 */
kvtc_status kvtc_encode_prefill(const kvtc_plan* plan, const kvtc_cache* cache, int layer,
                                const void* k, const void* v, int seq, int pos_start, int n_tok,
                                void* stream);

/*
 * kvtc_debug_encode_latent -- test-only: the fp32 latent y = M_u x of n_tok rows of one
 * unit (layer, head, kind) in the canonical order of kvtc_encode_append (what it
 * quantizes), so a checker can quantize and pack it independently.  An uncompressed
 * value unit returns x itself.  x: device [n_tok][d] of dtype (16-byte aligned);
 * y_out: device fp32 [n_tok][r_u].  Asynchronous on the stream.
 */
kvtc_status kvtc_debug_encode_latent(const kvtc_plan* plan, int layer, int head, int kind, const void* x,
                                     kvtc_dtype dtype, int n_tok, float* y_out, void* stream);

/*
 * kvtc_plan_prefill_stats -- diagnostics of kvtc_encode_prefill since the plan was
 * uploaded (or last reset): codes produced and codes whose tensor-core sum fell within
 * the error bound of a quantizer threshold and were recomputed in canonical order.
 * Synchronous (copies two counters to the host); reset != 0 zeroes them.
 */
kvtc_status kvtc_plan_prefill_stats(const kvtc_plan* plan, uint64_t* codes, uint64_t* recomputed, int reset);

/* ------------------------------------------------------------------ decode ------- */

/* Workspace bytes kvtc_decode_attention needs for n_seq sequences of at most
 * max_seq_len tokens: arrival counters (two int32 per sequence, KV head and group of 8
 * query heads) followed by the split-K partials. */
uint64_t kvtc_decode_workspace_bytes(const kvtc_plan* plan, int n_seq, int max_seq_len);

/*
 * kvtc_decode_attention -- one decode step of attention for one layer over the
 * compressed cache ("Efficiency": dequantization and the inverse rotation in one fused
 * pass).  For query head g of KV head h:
 *   q~ = M_K q (q moved into the key basis), s_t = scale * delta_K * q~ . (c_K,t - m_K)
 *   with m = (2^b - 1)/2, p = softmax over t < seq_len, z = sum_t p_t (c_V,t - m_V),
 *   o = M_V^T (delta_V * z).
 * Equivalent to softmax(scale * q . k_hat_t) v_hat_t with k_hat = M_K^T delta_K (c - m)
 * (the oracle's d-space form).  Split-K over the context; the G query heads of a KV head
 * share every code tile; the last splits of a (sequence, KV head) to finish merge the
 * partials (log-sum-exp) and back-project, each a share of the query heads, in the same
 * kernel.  An uncompressed value
 * unit (keys-only plans) enters the value MMAs with its fp16 values as they are stored
 * (c_V = v * 2^24, delta_V = 2^-24, m_V = 0, M_V = identity), so o = sum_t p_t v_t.
 * q: device [n_seq][H_q][d] of q_dtype.  seq_lens: device int32 [n_seq] (0 gives an
 * all-zero output).  max_seq_len: host upper bound of seq_lens (sizes the split grid;
 * longer sequences set KVTC_STATUS_BAD_POS).  softmax_scale: 0 means 1/sqrt(d).
 * out: device [n_seq][H_q][d] of out_dtype.  workspace: device, at least
 * kvtc_decode_workspace_bytes(plan, n_seq, max_seq_len) bytes (else ECAPACITY), 16-byte
 * aligned and zero-filled before its first use; every call leaves its counters at zero
 * again, so one workspace serves any number of consecutive calls (of any plan and shape
 * that fits), but two calls that share a workspace and overlap on the GPU race.  After a
 * call that set KVTC_STATUS_TIMEOUT the workspace must be zero-filled again.
 * Launches one kernel per group of KV heads with the same (b_K, b_V) (each pair has its
 * own kernel variant; one launch per layer when every head has the same widths);
 * nothing is allocated.
 */
kvtc_status kvtc_decode_attention(const kvtc_plan* plan, const kvtc_cache* cache, int layer,
                                  const void* q, kvtc_dtype q_dtype, const int32_t* seq_lens,
                                  int max_seq_len, float softmax_scale, void* out,
                                  kvtc_dtype out_dtype, void* workspace, uint64_t workspace_bytes,
                                  void* stream);

/*
 * kvtc_decode_attention_rope -- kvtc_decode_attention for caches whose keys were coded
 * before the rotary position embedding (KV-COBRA project page, Results: keys compressed
 * pre-RoPE).  The rotation of a key depends on its position, so q is not moved into the
 * key basis: per 16-token block the keys are reconstructed in d-space,
 * k_t = delta_K (c_K,t - m_K) M_K (tensor cores), rotated to position t and scored:
 *   s_t = scale * q . R(t) k_t,  R(t): (x_i, x_{i+64}) -> (x_i cos a - x_{i+64} sin a,
 *   x_{i+64} cos a + x_i sin a), a = t * rope_base^(-2i/128), i < 64
 * (the rotate-half form; cached token t of a sequence sits at position t; q arrives
 * already rotated to its own position, as a model applies RoPE to q before attention).
 * Values, softmax, split merge and back-projection as kvtc_decode_attention, through the
 * same workspace (kvtc_decode_workspace_bytes, zero-filled before its first use).
 * rope_base: 0 means 500000 (the Llama-3.1 value), else > 1.  The codes are those of
 * kvtc_encode_append / kvtc_encode_prefill applied to the un-rotated keys.
 */
kvtc_status kvtc_decode_attention_rope(const kvtc_plan* plan, const kvtc_cache* cache, int layer,
                                       const void* q, kvtc_dtype q_dtype, const int32_t* seq_lens,
                                       int max_seq_len, float softmax_scale, double rope_base, void* out,
                                       kvtc_dtype out_dtype, void* workspace, uint64_t workspace_bytes,
                                       void* stream);

/*
 * kvtc_decode_attention_noalloc -- kvtc_decode_attention without a caller workspace.
 * The KV-COBRA pages have no counterpart to this call; it exists for callers that cannot
 * allocate device memory (a host runtime that owns every allocation through its own
 * pool, a plugin limited to the buffers it is handed, code running while allocation is
 * not permitted).  Its split-K scratch is a fixed 16 MiB array inside the library
 * (a file-scope __device__ array: every GPU that loads the library holds it until the
 * process exits); nothing is allocated per call.
 *   - The first call on a device looks up the array's device address (once per device,
 *     with that device current).  Make that first call before any stream capture.  The
 *     address is kept for the life of the process: after cudaDeviceReset (or anything
 *     else that destroys the device's primary context) it is stale, and this call must
 *     not be used on that device again.
 *   - Calls whose kvtc_decode_workspace_bytes(plan, n_seq, max_seq_len) exceeds 16 MiB
 *     return KVTC_ECAPACITY; use kvtc_decode_attention with a workspace for those.
 *   - Every call shares the one array and leaves its contents behind.  The array starts
 *     at zero when the library is loaded and every call returns its arrival tickets to
 *     zero, so nothing has to be cleared between calls; but two calls that run at the
 *     same time on the GPU (different streams, or overlapping graphs) race.
 * Arguments, results and error codes otherwise as kvtc_decode_attention.
 */
kvtc_status kvtc_decode_attention_noalloc(const kvtc_plan* plan, const kvtc_cache* cache, int layer,
                                          const void* q, kvtc_dtype q_dtype, const int32_t* seq_lens,
                                          int max_seq_len, float softmax_scale, void* out,
                                          kvtc_dtype out_dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KVTC_H */
