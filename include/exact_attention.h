/*
 * exact_attention.h — C ABI of the B200 (sm_100a) exact-attention library.
 *
 * What is computed (wsisp.com "FIA / FlashAttention", section 一):
 *     O = softmax(Q K^T * scale) V,   LSE = ln sum_j exp(scale * q.k_j)   per query row,
 * by tiling with an online softmax so the score matrix never reaches HBM
 * (cloud.baidu.com "FasterTransformer与FlashAttention的联系与区别", section 三,
 * tiling pseudocode; niuteng5618.github.io "Flash Attention & Paged Attention",
 * section 1).  Decode follows Flash-Decoding over a paged KV cache (same page,
 * section "FA对decode阶段的影响" and section 2): the cached context of each request
 * is split across SMs, each split emits a partial (O_i, LSE_i), and a light
 * merge kernel reduces them.  The plan/run split follows wsisp.com, sections 二
 * and 四 (plan does load balancing, run executes).
 *
 * Conventions for every entry point:
 *   - Pointers named *_host are host memory; every other pointer is device
 *     memory on the current CUDA device.  The caller owns all memory,
 *     including the decode workspace; the library never allocates device
 *     memory.  The only library-owned object is the host-side fa_plan.
 *   - bf16 tensors are IEEE bfloat16 bit patterns (2 bytes per element).
 *   - Device pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is only enqueued; nothing synchronises the host, so a run can be
 *     captured into a CUDA graph after its inputs' host-side shape data is fixed.
 *   - Every function returns an fa_status.  Arguments are validated on the host
 *     before any launch; on error nothing is enqueued.  FA_ERR_CUDA means a CUDA
 *     runtime call failed (fa_last_cuda_error() gives the cudaError_t value).
 *   - A kernel that finds bad device-side data (a page id outside the pool, a
 *     cache length beyond what its plan covers) or a wait that exceeds its
 *     bound records a code in a per-device status word; read it with
 *     fa_get_device_status().  Kernels never trap.
 *   - The same library built with FA_DEBUG (libexact_attention_debug.so) also
 *     checks every global index a kernel computes against its buffer before
 *     the access; a failed check records FA_ERR_DEBUG_INDEX and skips the
 *     access.  Its results are bit-identical to the release build's.
 */
#ifndef EXACT_ATTENTION_H_
#define EXACT_ATTENTION_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = -1,   /* null/misaligned pointer, bad size or count */
  FA_ERR_UNSUPPORTED = -2,   /* valid but not implemented (e.g. head_dim 96) */
  FA_ERR_WORKSPACE = -3,     /* decode workspace smaller than the plan needs */
  FA_ERR_CUDA = -4,          /* a CUDA runtime/driver call failed */
  FA_ERR_TIMEOUT = -5,       /* (device status) a bounded wait gave up */
  FA_ERR_PLAN_MISMATCH = -6, /* plan does not match the call's shapes, or a
                                device cache length exceeds what it covers */
  FA_ERR_BAD_PAGE = -7,      /* (device status) block_table entry outside the pool */
  FA_ERR_DEBUG_INDEX = -8    /* (device status, FA_DEBUG builds only) a computed index failed
                                its bounds check; the access was skipped */
} fa_status;

/* Opaque host-side decode plan, created by fa_decode_plan, freed by fa_plan_free. */
typedef struct fa_plan fa_plan;

/* Element type of a paged KV cache. */
typedef enum { FA_KV_BF16 = 0, FA_KV_E4M3 = 1 } fa_kv_dtype;

/* Decode split kernel a plan targets. */
typedef enum {
  FA_DECODE_AUTO = 0,          /* the planner chooses */
  FA_DECODE_CUDA_CORES = 1,    /* fp32 FMAs per element, up to 8 heads per CTA */
  FA_DECODE_TENSOR_CORES = 2   /* tcgen05 MMAs, all G heads (x q_len tokens, <= 16 rows) of a kv
                                  head per CTA; d = 128 */
} fa_decode_kernel;

/* Read-only view of a plan (for tests and tools). */
typedef struct {
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int page_size;
  int max_pages_per_seq;
  int chunk_tokens;      /* keys per split; a multiple of page_size */
  int max_splits;        /* splits of the longest planned request */
  int heads_per_cta;     /* query heads of one kv head packed into a CTA */
  int num_work_items;    /* (request, kv-head group, split) CTAs that run: each split of a
                            request, and one for an empty request (it writes O = 0, LSE = -inf) */
  int max_seqlen;        /* longest planned cache length */
  size_t workspace_bytes;
  int kv_dtype;          /* fa_kv_dtype the plan was made for */
  int tensor_cores;      /* 1 if the plan runs the tensor-core split kernel */
  int q_len;             /* query tokens per request */
} fa_plan_info;

/* Options of fa_decode_plan_ex. */
typedef struct {
  int kv_dtype;          /* fa_kv_dtype */
  int kernel;            /* fa_decode_kernel */
  int q_len;             /* query tokens per request, >= 1 (see fa_decode_plan_ex) */
} fa_decode_options;

/*
 * fa_prefill — causal or full exact attention over packed variable-length
 * sequences (FA's varlen prefill: wsisp.com "FIA / FlashAttention", sections
 * 一, 二 and 四; causal=True as in its API example).
 *
 *   q    [T, Hq,  d] bf16, row-major (token, head, dim), T = cu_seqlens[batch]
 *   k, v [T, Hkv, d] bf16, same layout
 *   cu_seqlens_dev  [batch+1] int32 device; cu_seqlens_host the same values
 *                   on the host (used to build the tile schedule)
 *   Query head h reads kv head h / (Hq/Hkv) (GQA/MQA when Hkv < Hq).
 *   causal != 0: key j is visible to query i of the same sequence iff j <= i.
 *   scale: score multiplier; NaN means 1/sqrt(d).  Must be > 0 otherwise.
 *   out  [T, Hq, d] bf16 (written); lse [T, Hq] fp32 natural-log LSE, or NULL.
 * Supported: d in {64, 128}; Hq % Hkv == 0; each sequence length >= 1;
 * T * Hq * d < 2^40 (else FA_ERR_UNSUPPORTED; the kernels index q, out and
 * lse with 64-bit offsets, and T itself is an int32 as cu_seqlens are).
 * Output rows of different sequences never mix.
 *
 * Schedule (plan-stage load balancing: wsisp.com "FIA / FlashAttention",
 * section 二).  The work is cut into items of two 128-row query tiles that read
 * the same K/V tiles, ordered heaviest first.  By default one CTA per SM takes
 * items from a device counter and keeps its pipelines running from one item to
 * the next (the persistent form).  The counter is one of 256 pairs in the
 * library's device memory, one per (device, stream) that launches the kernel,
 * reset to zero by the last CTA of each launch.  The grid form (one CTA per
 * item) runs instead when the environment variable FA_PREFILL_SCHEDULE is
 * "grid", while `stream` is being captured into a graph (a graph's replays
 * could overlap other launches on the same counter), and once 256 streams of a
 * device have taken a counter (a stream keeps its counter for the life of the
 * process).  Both forms compute bit-identical results;
 * fa_prefill_last_schedule() tells which one the calling thread's last call
 * launched.
 */
int fa_prefill(const void* q, const void* k, const void* v,
               const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host, int batch,
               int num_q_heads, int num_kv_heads, int head_dim, int causal, float scale,
               void* out, float* lse, void* stream);

/* Schedule of a prefill launch (see fa_prefill). */
typedef enum { FA_SCHEDULE_GRID = 0, FA_SCHEDULE_PERSISTENT = 1 } fa_prefill_schedule;

/*
 * fa_prefill_last_schedule — the fa_prefill_schedule that the calling thread's
 * last fa_prefill, fa_prefill_fp8 or fa_prefill_paged call launched, or -1 if
 * that call failed or there was none.  Host only; never fails.
 */
int fa_prefill_last_schedule(void);

/*
 * fa_prefill_fp8 — fa_prefill over E4M3 inputs (FP8 inference kernels:
 * wsisp.com "FIA / FlashAttention", section 三, FP8 row; the operation is
 * fa_prefill's on the dequantised tensors).
 *
 *   q [T, Hq, 128], k, v [T, Hkv, 128]: E4M3 bytes (OCP FP8 E4M3), same
 *       layouts as fa_prefill; base addresses 16-byte aligned.
 *   q_scale, k_scale, v_scale: per-tensor dequantisation scales (> 0,
 *       finite): the query is q_scale * E4M3(q8), and likewise for k and v.
 *   Other arguments as fa_prefill; head_dim must be 128 (else
 *   FA_ERR_UNSUPPORTED).
 * Q K^T multiplies the E4M3 codes exactly and accumulates in fp32; the
 * probabilities are rounded to f16 (bf16 in fa_prefill) and V is widened to f16
 * exactly, so P V also accumulates in fp32; out is bf16, lse fp32.  The NaN
 * code S.1111.111 must not occur in the inputs (a saturating quantiser never
 * writes it); it propagates as NaN into the rows that read it.
 */
int fa_prefill_fp8(const void* q, const void* k, const void* v,
                   const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host, int batch,
                   int num_q_heads, int num_kv_heads, int head_dim, int causal, float scale,
                   float q_scale, float k_scale, float v_scale, void* out, float* lse,
                   void* stream);

/*
 * fa_append_kv — write new K/V rows into a paged KV cache (the cache that
 * prefill fills for later steps: niuteng5618.github.io "Flash Attention &
 * Paged Attention", section "FA对Prefill阶段的影响"; fixed-size pages behind a
 * logical-to-physical page table: same page, section 2).
 *
 *   k_new, v_new [total_new, Hkv, d] bf16, packed by cu_seqlens_new_dev
 *       ([batch+1] int32 device; cu_seqlens_new_dev[batch] == total_new).
 *   k_pages, v_pages, num_pages, page/token/head strides: the page pool, as
 *       for fa_decode_paged (written here).
 *   block_table [batch, max_pages_per_seq] int32 device.
 *   cache_seqlens_dev [batch] int32: each request's length AFTER the append.
 *       Request b's n_b new rows take logical positions
 *       cache_seqlens[b] - n_b ... cache_seqlens[b] - 1, i.e. token t goes to
 *       page block_table[b][t / page_size], slot t % page_size.
 *   page_size: 64.
 * Only the slots of the new rows are written.  A row whose request has
 * n_b > cache_seqlens[b], or a length past max_pages_per_seq * page_size, is
 * skipped and FA_ERR_PLAN_MISMATCH recorded in the device status word; a page
 * id outside [0, num_pages) is skipped and FA_ERR_BAD_PAGE recorded.
 * total_new == 0 enqueues nothing.
 */
int fa_append_kv(const void* k_new, const void* v_new, const int32_t* cu_seqlens_new_dev,
                 int total_new, int batch, int num_kv_heads, int head_dim, void* k_pages,
                 void* v_pages, int64_t num_pages, int64_t page_stride, int64_t token_stride,
                 int64_t head_stride, int page_size, const int32_t* block_table,
                 int max_pages_per_seq, const int32_t* cache_seqlens_dev, void* stream);

/*
 * fa_prefill_paged — chunked prefill: each request's new queries attend to its
 * whole paged KV cache (the cached prefix plus the chunk's own K/V, already
 * written with fa_append_kv).  Same tiled tcgen05 kernel as fa_prefill, with
 * K/V tiles fetched page by page through block_table.
 *
 *   q [Tq, Hq, d] bf16 packed by cu_seqlens_q_dev / cu_seqlens_q_host
 *       ([batch+1] int32; q_len_b = cu[b+1] - cu[b] >= 1).
 *   k_pages, v_pages, num_pages, strides, block_table, max_pages_per_seq:
 *       the page pool and table, as for fa_decode_paged.
 *   cache_seqlens_dev / cache_seqlens_host [batch] int32: keys per request,
 *       k_len_b >= q_len_b, k_len_b <= max_pages_per_seq * page_size, and
 *       max_pages_per_seq * page_size <= 2^30 (else FA_ERR_INVALID_ARG).
 *   causal != 0: the chunk's queries are the last q_len_b positions of the
 *       request's sequence, so query i sees keys 0 .. k_len_b - q_len_b + i
 *       (with k_len_b == q_len_b this is fa_prefill's causal mask).
 *       causal == 0: every query sees all k_len_b keys.
 *   page_size: 64.  scale: NaN means 1/sqrt(d).
 *   out [Tq, Hq, d] bf16; lse [Tq, Hq] fp32 or NULL.
 * Cache slots past k_len_b in a request's last page may hold anything (NaN
 * included): they are never used.  A block_table entry outside the pool reads
 * as zeros and records FA_ERR_BAD_PAGE; device lengths that disagree with the
 * host copies record FA_ERR_PLAN_MISMATCH.  The host and device copies of
 * cu_seqlens_q and cache_seqlens must hold the same values.  Schedule: as for
 * fa_prefill (persistent by default, the grid form under FA_PREFILL_SCHEDULE=
 * grid, during graph capture or past 256 streams; bit-identical results).
 */
int fa_prefill_paged(const void* q, const int32_t* cu_seqlens_q_dev,
                     const int32_t* cu_seqlens_q_host, const void* k_pages, const void* v_pages,
                     int64_t num_pages, int64_t page_stride, int64_t token_stride,
                     int64_t head_stride, const int32_t* block_table, int max_pages_per_seq,
                     const int32_t* cache_seqlens_dev, const int32_t* cache_seqlens_host,
                     int batch, int num_q_heads, int num_kv_heads, int head_dim, int page_size,
                     int causal, float scale, void* out, float* lse, void* stream);

/*
 * fa_decode_plan — host-only split and load-balance planning for paged
 * decode (the "plan" stage: wsisp.com "FIA / FlashAttention", section 二;
 * Flash-Decoding's split along the context: niuteng5618.github.io, section
 * "FA对decode阶段的影响"; num_splits as a hardware knob: rt2005.com
 * "FlashAttention突破性架构", section 分块矩阵乘法的并行优化).
 *
 *   cache_seqlens_host [batch] int32: cached tokens per request (0 allowed).
 *   page_size: tokens per KV page (64 supported).
 *   max_pages_per_seq: columns of block_table; each cache length must be
 *                      <= max_pages_per_seq * page_size (cache overflow check,
 *                      rt2005.com section 故障诊断与性能监控).
 *   num_sms: SM count of the target GPU (148 on B200); sizes the splits.
 *   num_splits_override: 0 = automatic; S > 0 caps every request at S splits
 *                        (chunk = ceil(max_seqlen / S) rounded up to a page).
 * On success *plan_out owns a new plan and *workspace_bytes is the device
 * workspace fa_decode_paged needs (0 when no request is split).
 * The plan stays valid for later calls whose device cache lengths are not
 * longer than the planned maximum split coverage (max_splits*chunk_tokens).
 */
int fa_decode_plan(const int32_t* cache_seqlens_host, int batch, int num_q_heads,
                   int num_kv_heads, int head_dim, int page_size, int max_pages_per_seq,
                   int num_sms, int num_splits_override, fa_plan** plan_out,
                   size_t* workspace_bytes);

/*
 * fa_decode_plan_kv — fa_decode_plan for a given cache element type and split
 * kernel.  kv_dtype: FA_KV_BF16 (plans for fa_decode_paged) or FA_KV_E4M3
 * (plans for fa_decode_paged_fp8; a plan is only accepted by the entry point
 * of its type, else FA_ERR_PLAN_MISMATCH).  kernel: FA_DECODE_AUTO picks the
 * tensor-core kernel for an E4M3 cache or a group of 4 or more heads when
 * d = 128 and Hq/Hkv <= 16; FA_DECODE_TENSOR_CORES outside that range is
 * FA_ERR_UNSUPPORTED.  fa_decode_plan(...) is
 * fa_decode_plan_kv(..., FA_KV_BF16, FA_DECODE_AUTO, ...).
 */
int fa_decode_plan_kv(const int32_t* cache_seqlens_host, int batch, int num_q_heads,
                      int num_kv_heads, int head_dim, int page_size, int max_pages_per_seq,
                      int num_sms, int num_splits_override, int kv_dtype, int kernel,
                      fa_plan** plan_out, size_t* workspace_bytes);

/*
 * fa_decode_plan_ex — fa_decode_plan_kv plus multi-token decode.  With
 * options->q_len = n > 1 each request brings n query tokens (e.g. speculative
 * decoding) whose K/V are already the last n entries of its cache: q and out
 * are [batch, n, Hq, d], lse [batch, n, Hq], and token t of request b sees
 * cached keys 0 .. cache_seqlens[b] - n + t (the chunked-prefill mask).  Needs
 * the tensor-core kernel: d = 128 and n * Hq/Hkv <= 16 (else
 * FA_ERR_UNSUPPORTED); every planned length must be >= n.
 */
int fa_decode_plan_ex(const int32_t* cache_seqlens_host, int batch, int num_q_heads,
                      int num_kv_heads, int head_dim, int page_size, int max_pages_per_seq,
                      int num_sms, int num_splits_override, const fa_decode_options* options,
                      fa_plan** plan_out, size_t* workspace_bytes);

int fa_plan_get_info(const fa_plan* plan, fa_plan_info* info);
void fa_plan_free(fa_plan* plan);

/*
 * fa_decode_paged — one query token per request against its paged KV cache
 * (the "run" stage; Flash-Decoding split kernel + LSE merge kernel).
 *
 *   q [batch, Hq, d] bf16 ([batch, q_len, Hq, d] with a multi-token plan,
 *       fa_decode_plan_ex; out and lse then carry the q_len axis too).
 *   k_pages, v_pages: a pool of num_pages pages of page_size tokens; element
 *       (page p, slot t, kv head g, dim c) is at
 *       p*page_stride + t*token_stride + g*head_stride + c   (elements).
 *       NHD layout [P, page, Hkv, d]: strides (page*Hkv*d, Hkv*d, d);
 *       HND layout [P, Hkv, page, d]: strides (Hkv*page*d, d, page*d).
 *       All strides must be multiples of 8 elements.
 *   block_table [batch, max_pages_per_seq] int32: physical page of each
 *       logical page; entries past a request's last page are never read.
 *   cache_seqlens_dev [batch] int32 (device copy of the planned lengths, or
 *       shorter/equal lengths at later steps).
 *   scale: NaN means 1/sqrt(d).
 *   out [batch, Hq, d] bf16; lse [batch, Hq] fp32 (or NULL).
 *   workspace: >= the plan's workspace_bytes, 256-byte aligned (may be NULL
 *       when that is 0).  It holds the split partials; its contents need no
 *       initialisation and are dead after the call.
 * A request with cache length 0 gets O = 0 and LSE = -inf.
 * The result depends only on logical token order, never on which physical
 * pages hold them (permuting the pool and the table gives identical bits).
 */
int fa_decode_paged(const void* q, const void* k_pages, const void* v_pages, int64_t num_pages,
                    int64_t page_stride, int64_t token_stride, int64_t head_stride,
                    const int32_t* block_table, const int32_t* cache_seqlens_dev,
                    const fa_plan* plan, float scale, void* out, float* lse,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_decode_paged_fp8 — fa_decode_paged over an FP8 KV cache (FP8 inference
 * kernels: wsisp.com "FIA / FlashAttention", section 三, FP8 row).
 *
 * Same arguments, plan and workspace as fa_decode_paged, except:
 *   k_pages, v_pages: E4M3 bytes (OCP FP8 E4M3: bias 7, subnormals, max 448),
 *       same page layouts; strides are in elements (= bytes) and must be
 *       multiples of 16.
 *   k_scale, v_scale: per-tensor dequantisation scales (> 0, finite): the
 *       cached key is k_scale * E4M3(k8), the value v_scale * E4M3(v8).
 * q stays bf16; scores, softmax and P V accumulate in fp32; out is bf16.
 * The code S.1111.111 (NaN in E4M3) is read as a finite +-480; a quantiser
 * that saturates never writes it.  Slots past a request's cache length may
 * hold any byte.
 */
int fa_decode_paged_fp8(const void* q, const void* k_pages, const void* v_pages,
                        int64_t num_pages, int64_t page_stride, int64_t token_stride,
                        int64_t head_stride, const int32_t* block_table,
                        const int32_t* cache_seqlens_dev, const fa_plan* plan, float scale,
                        float k_scale, float v_scale, void* out, float* lse, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * fa_decode_paged_static — fa_decode_paged for callers that cannot allocate.
 *
 * The pages have no counterpart to this entry point; it exists for callers
 * that may not call cudaMalloc: extensions hosted inside a framework that owns
 * every byte of device memory through its own allocator and gives plugins no
 * way to allocate, serving loops that must not pay for cudaMalloc/cudaFree
 * (which can synchronise the device and stall other work), and processes
 * whose device-memory budget is fixed at start-up.
 *
 * Same arguments and results as fa_decode_paged, minus the workspace: the
 * split partials live in one file-scope static device array of
 * FA_STATIC_SCRATCH_BYTES (16 MiB) inside this library.  Every GPU that loads
 * the library holds that array until the process exits.  The caller still
 * passes all inputs and outputs.
 *   - A plan whose workspace_bytes exceeds FA_STATIC_SCRATCH_BYTES is rejected
 *     with FA_ERR_WORKSPACE before anything is enqueued.
 *   - Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.  The cached address is not looked up again, so after a
 *     cudaDeviceReset on that device this entry point must not be used again
 *     in the same process.
 *   - All calls on a device share the one array, which keeps whatever the last
 *     call left in it.  Nothing in it needs to start at zero: every partial the
 *     merge reads is written earlier in the same call.  Calls that overlap on
 *     the GPU (for example on two streams at once) race on the array; the
 *     caller must order them.
 */
#define FA_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)
int fa_decode_paged_static(const void* q, const void* k_pages, const void* v_pages,
                           int64_t num_pages, int64_t page_stride, int64_t token_stride,
                           int64_t head_stride, const int32_t* block_table,
                           const int32_t* cache_seqlens_dev, const fa_plan* plan, float scale,
                           void* out, float* lse, void* stream);

/*
 * fa_cascade_decode — decode with a prefix shared by every request of the
 * batch (prefix sharing: wsisp.com "FIA / FlashAttention", section 三, MLA/GQA
 * row), computed as two partial states merged by their LSE (niuteng5618.github.io,
 * section "FA对decode阶段的影响", steps 3-4).
 *
 *   The context of request b is the shared prefix (prefix_len tokens in the
 *   pages listed by prefix_block_table, device [ceil(prefix_len / page_size)])
 *   followed by its own suffix (cache_seqlens_dev[b] tokens through row b of
 *   block_table).  The result equals fa_decode_paged over that concatenation.
 *   plan: a bf16, single-token plan made for the suffix lengths.
 *   workspace: >= fa_cascade_workspace_bytes(plan, prefix_len), 256-byte aligned.
 * The prefix is read once for the whole batch: the requests act as the query
 * tokens of one full-attention sequence over the prefix (the paged prefill
 * kernel, its key range cut to fill the SMs); the suffixes run through the
 * paged decode; one kernel merges the states.  prefix_len == 0 is the plain
 * decode.  q, out [batch, Hq, d] bf16; lse [batch, Hq] fp32 or NULL.
 */
int fa_cascade_workspace_bytes(const fa_plan* plan, int prefix_len, size_t* bytes);
int fa_cascade_decode(const void* q, const void* k_pages, const void* v_pages, int64_t num_pages,
                      int64_t page_stride, int64_t token_stride, int64_t head_stride,
                      const int32_t* prefix_block_table, int prefix_len,
                      const int32_t* block_table, const int32_t* cache_seqlens_dev,
                      const fa_plan* plan, float scale, void* out, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * fa_merge_states — combine partial attention states by their LSE (the light
 * reduction kernel of Flash-Decoding: niuteng5618.github.io, section
 * "FA对decode阶段的影响", step 4).
 *
 *   o_parts   [num_states, rows, num_heads, d] fp32 (each state normalised)
 *   lse_parts [num_states, rows, num_heads]    fp32 natural-log LSE; -inf marks
 *             an empty state (zero weight)
 *   out [rows, num_heads, d] bf16 = sum_i w_i O_i / sum_i w_i, w_i = e^{LSE_i - max}
 *   lse [rows, num_heads] fp32 = max + ln sum_i w_i, or NULL.
 * All-empty rows give O = 0, LSE = -inf.  d in {64, 128}; num_states >= 1.
 */
int fa_merge_states(const float* o_parts, const float* lse_parts, int num_states, int rows,
                    int num_heads, int head_dim, void* out, float* lse, void* stream);

/* Human-readable text for an fa_status value (static storage). */
const char* fa_strerror(int status);

/* cudaError_t of the last failed CUDA call made by this library in this thread. */
int fa_last_cuda_error(void);

/*
 * Device status word of the current device: synchronises `stream`, copies the
 * word into *status_host (FA_OK when no kernel recorded a problem) and clears
 * it when clear != 0.
 */
int fa_get_device_status(void* stream, int* status_host, int clear);

/*
 * fa_selftest_wait_timeout — failure-detection self-test.  Launches one small
 * kernel that waits on a barrier nothing ever arrives at, with a bound of
 * limit_us microseconds (clamped to [1000, 2000000]).  When the bound runs out
 * the kernel records FA_ERR_TIMEOUT in the device status word and returns; it
 * never traps, so the CUDA context stays usable.  Read the result with
 * fa_get_device_status().  (The same bounded-wait path guards every wait in
 * the prefill and decode kernels.)
 */
int fa_selftest_wait_timeout(int64_t limit_us, void* stream);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int fa_version(void);

/*
 * fa_debug_selftest_index — check of the bounds-checked build's index checks
 * (libexact_attention_debug.so, compiled with FA_DEBUG).  No page counterpart:
 * it tests this library's failure detection.  On `stream`, one kernel sets
 * buf[0] = 1 and then tries buf[n/2 + 1], an index it checks against n/2 and
 * must refuse: the check records FA_ERR_DEBUG_INDEX in the device status
 * word and skips the store (the index lies inside buf, so even a check that
 * failed to refuse would write nothing outside it).
 *   buf: device int32 [n], n >= 4.
 * The release build launches nothing and returns FA_ERR_UNSUPPORTED.
 */
int fa_debug_selftest_index(int32_t* buf, int n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_H_ */
