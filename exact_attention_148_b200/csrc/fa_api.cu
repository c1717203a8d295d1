// C ABI of the exact-attention library: argument validation, tensor-map
// construction, tile scheduling and kernel launches (declared in
// include/exact_attention.h).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/exact_attention.h"
#include "append_sm100.cuh"
#include "decode_sm100.cuh"
#include "decode_tc_sm100.cuh"
#include "planner.h"
#include "prefill_persist_sm100.cuh"
#include "prefill_pp_sm100.cuh"

#define FA_API extern "C" __attribute__((visibility("default")))

struct fa_plan {
  fa::DecodePlan p;
};

// Work counters of the persistent prefill, {next item, CTAs finished} per
// slot; zero at load, and reset to zero by the last CTA of every launch.
__device__ uint32_t g_prefill_sched[fa::kSchedSlots][2];

namespace {

thread_local int t_last_cuda_error = 0;

int cuda_fail(int code) {
  t_last_cuda_error = code;
  return FA_ERR_CUDA;
}

#define FA_CUDA_CHECK(expr)                          \
  do {                                               \
    cudaError_t e_ = (expr);                         \
    if (e_ != cudaSuccess) return cuda_fail(e_);     \
  } while (0)

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int encode_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
               const cuuint64_t* strides_bytes, const cuuint32_t* box, CUtensorMapSwizzle swz,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto fn = encode_fn();
  if (fn == nullptr) return cuda_fail(cudaErrorNotSupported);
  const cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, dtype, rank, const_cast<void*>(base), dims,
                  strides_bytes, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(static_cast<int>(r) + 10000);
  return FA_OK;
}

// cudaFuncSetAttribute once per (kernel, device).
int ensure_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> done;
  int dev = 0;
  FA_CUDA_CHECK(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lock(mu);
  for (auto& kv : done)
    if (kv.first == kernel && kv.second == dev) return FA_OK;
  FA_CUDA_CHECK(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  done.emplace_back(kernel, dev);
  return FA_OK;
}

// SM count of the current device, queried once per device.
int sm_count(int* out) {
  constexpr int kMaxDev = 128;
  static std::mutex mu;
  static int cached[kMaxDev] = {};
  int dev = 0;
  FA_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDev) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int n = 0;
    FA_CUDA_CHECK(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev));
    cached[dev] = n;
  }
  *out = cached[dev];
  return FA_OK;
}

float resolve_scale(float scale, int head_dim) {
  return std::isnan(scale) ? 1.0f / std::sqrt(static_cast<float>(head_dim)) : scale;
}

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------- prefill
// groups: (sequence << 16 | kv head, number of CTAs) in launch order.
template <int D, bool PAGED, bool F8 = false>
int launch_prefill(fa::PrefillParams& prm, const std::vector<std::pair<uint32_t, int>>& groups,
                   cudaStream_t stream) {
  constexpr int kSmem = fa::PrefillPPCfg<D, F8>::SMEM_BYTES;
  constexpr int kThreads = fa::PrefillPPCfg<D, F8>::THREADS;
  auto kernel = fa::fa_prefill_pp_kernel<D, PAGED, F8>;
  int st = ensure_smem(reinterpret_cast<const void*>(kernel), kSmem);
  if (st != FA_OK) return st;
  for (size_t off = 0; off < groups.size(); off += fa::kPrefillMaxGroups) {
    const int n = static_cast<int>(std::min<size_t>(fa::kPrefillMaxGroups, groups.size() - off));
    int64_t total = 0;
    for (int i = 0; i < n; ++i) {
      prm.group_start[i] = static_cast<int>(total);
      prm.group_id[i] = groups[off + i].first;
      total += groups[off + i].second;
    }
    if (total > INT32_MAX) return FA_ERR_UNSUPPORTED;
    prm.group_start[n] = static_cast<int>(total);
    prm.num_groups = n;
    kernel<<<static_cast<unsigned>(total), kThreads, kSmem, stream>>>(prm);
    FA_CUDA_CHECK(cudaGetLastError());
  }
  return FA_OK;
}

// Persistent prefill (packed Q/K/V): one CTA per SM, items from a counter.
template <int D, bool F8, bool PAGED = false>
int launch_prefill_persistent(fa::PrefillParams& prm, const std::vector<std::pair<uint32_t, int>>& groups,
                              cudaStream_t stream, uint32_t* sched, int num_sms) {
  constexpr int kSmem = fa::PrefillPersistCfg<D, F8, PAGED>::SMEM_BYTES;
  constexpr int kThreads = fa::PrefillPersistCfg<D, F8, PAGED>::THREADS;
  auto kernel = fa::fa_prefill_persist_kernel<D, F8, PAGED>;
  int st = ensure_smem(reinterpret_cast<const void*>(kernel), kSmem);
  if (st != FA_OK) return st;
  for (size_t off = 0; off < groups.size(); off += fa::kPrefillMaxGroups) {
    const int n = static_cast<int>(std::min<size_t>(fa::kPrefillMaxGroups, groups.size() - off));
    int64_t total = 0;
    for (int i = 0; i < n; ++i) {
      prm.group_start[i] = static_cast<int>(total);
      prm.group_id[i] = groups[off + i].first;
      total += groups[off + i].second;
    }
    if (total > INT32_MAX) return FA_ERR_UNSUPPORTED;
    prm.group_start[n] = static_cast<int>(total);
    prm.num_groups = n;
    static thread_local fa::PrefillPersistParams pp;   // ~17 KB; kept off the stack
    pp.p = prm;
    pp.sched = sched;
    pp.total_items = static_cast<int>(total);
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(total, num_sms));
    kernel<<<grid, kThreads, kSmem, stream>>>(pp);
    FA_CUDA_CHECK(cudaGetLastError());
  }
  return FA_OK;
}

// The packed prefill runs the persistent form unless FA_PREFILL_SCHEDULE=grid.
bool prefill_persistent_requested() {
  const char* s = std::getenv("FA_PREFILL_SCHEDULE");
  return s == nullptr || std::strcmp(s, "grid") != 0;
}

// Schedule of the calling thread's last fa_prefill / fa_prefill_fp8 launch.
thread_local int t_last_prefill_schedule = -1;

// The persistent prefill's counter pair for a launch on `stream`: one pair per
// (device, stream), so launches that can overlap (other streams) never share
// one, and launches on one stream run one after the other.  Null, and the grid
// form is used, while the stream is being captured (a graph keeps the pointer,
// and its replays could overlap eager launches on the same pair), when the
// stream's id cannot be read, or once every pair of the device is taken.
uint32_t* prefill_sched_slot(cudaStream_t stream) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (cs != cudaStreamCaptureStatusNone) return nullptr;
  unsigned long long id = 0;
  int dev = 0;
  if (cudaStreamGetId(stream, &id) != cudaSuccess || cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  // The counters' address is looked up on every call (cheap once the module
  // is loaded), so it stays right after a cudaDeviceReset reloads the module.
  void* base = nullptr;
  if (cudaGetSymbolAddress(&base, g_prefill_sched) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  static std::mutex mu;
  static std::map<std::pair<int, unsigned long long>, int> slot_of;
  static std::map<int, int> taken;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev, id);
  auto it = slot_of.find(key);
  if (it == slot_of.end()) {
    int& t = taken[dev];
    if (t >= fa::kSchedSlots) return nullptr;
    it = slot_of.emplace(key, t++).first;
  }
  return static_cast<uint32_t*>(base) + 2 * it->second;
}

// Launch order of the prefill CTAs: sequences heaviest first (most query-key
// pairs; their groups carry the most work), one group of CTAs per (sequence,
// kv head).  A CTA takes two heads of the group at one q tile when the group
// is even, else two consecutive q tiles of one head, so a group has
// ceil(Lq/128) * G/2 or ceil(ceil(Lq/128)/2) * G CTAs.
// q_lens[b] >= 1 queries, k_lens[b] >= q_lens[b] keys (equal when unpaged).
int build_prefill_groups(const std::vector<int64_t>& q_lens, const std::vector<int64_t>& k_lens,
                         int num_q_heads, int num_kv_heads, bool causal,
                         std::vector<std::pair<uint32_t, int>>* groups) {
  const int batch = static_cast<int>(q_lens.size());
  std::vector<std::pair<double, int>> by_work;   // (query-key pairs, sequence)
  for (int b = 0; b < batch; ++b) {
    const double lq = static_cast<double>(q_lens[b]), lk = static_cast<double>(k_lens[b]);
    by_work.emplace_back(causal ? lq * (lk - lq) + 0.5 * lq * (lq + 1.0) : lq * lk, b);
  }
  std::stable_sort(by_work.begin(), by_work.end(),
                   [](const auto& a, const auto& b) { return a.first > b.first; });
  const int group = num_q_heads / num_kv_heads;
  groups->clear();
  groups->reserve(static_cast<size_t>(batch) * num_kv_heads);
  for (const auto& e : by_work) {
    const int ntiles = static_cast<int>((q_lens[e.second] + 127) / 128);
    const int ctas = (group % 2 == 0) ? ntiles * (group / 2) : ((ntiles + 1) / 2) * group;
    for (int g = 0; g < num_kv_heads; ++g)
      groups->emplace_back((static_cast<uint32_t>(e.second) << 16) | static_cast<uint32_t>(g), ctas);
  }
  return FA_OK;
}

// 4-D tensor map over a K or V page pool: dim 0 = the d contiguous columns,
// dims 1..3 = token slot, kv head and page ordered by increasing stride.  The
// box is `box_cols` columns x a whole page of tokens x 1 head x 1 page.
// Reports which dimension holds the kv head and which the page.
int encode_page_pool_map(CUtensorMap* map, const void* pool, int64_t num_pages, int64_t page_stride,
                         int64_t token_stride, int64_t head_stride, int page_size, int num_kv_heads,
                         int head_dim, int box_cols, CUtensorMapSwizzle swz, int* head_coord,
                         int* page_coord, int elem_bytes = 2) {
  struct Dim { int64_t stride; int64_t extent; int role; };   // role 0 token, 1 head, 2 page
  Dim dd[3] = {{token_stride, page_size, 0}, {head_stride, num_kv_heads, 1},
               {page_stride, num_pages, 2}};
  std::sort(dd, dd + 3, [](const Dim& a, const Dim& b) { return a.stride < b.stride; });
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_dim), 0, 0, 0};
  cuuint64_t strides[3];
  cuuint32_t box[4] = {static_cast<cuuint32_t>(box_cols), 1, 1, 1};
  for (int i = 0; i < 3; ++i) {
    dims[i + 1] = static_cast<cuuint64_t>(dd[i].extent);
    strides[i] = static_cast<cuuint64_t>(dd[i].stride) * elem_bytes;
    if (dd[i].role == 0) box[i + 1] = static_cast<cuuint32_t>(page_size);
    if (dd[i].role == 1) *head_coord = i + 1;
    if (dd[i].role == 2) *page_coord = i + 1;
  }
  return encode_map(map, pool, 4, dims, strides, box, swz,
                    elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

// Shared checks of a page pool's description (element strides; every stride
// must be a multiple of 16 bytes).
bool valid_pool(const void* k_pages, const void* v_pages, int64_t num_pages, int64_t page_stride,
                int64_t token_stride, int64_t head_stride, int elem_bytes = 2) {
  if (!k_pages || !v_pages || !aligned(k_pages, 16) || !aligned(v_pages, 16)) return false;
  if (num_pages < 1 || num_pages > INT32_MAX) return false;
  const int64_t m = 16 / elem_bytes;
  if (page_stride <= 0 || token_stride <= 0 || head_stride <= 0 || page_stride % m ||
      token_stride % m || head_stride % m)
    return false;
  return true;
}

// ---------------------------------------------------------------------------- decode
template <int D, int GC, bool KV8>
int launch_decode_split(const fa::DecodeParams& prm, dim3 grid, cudaStream_t stream) {
  using C = fa::DecodeCfg<D, GC, KV8>;
  auto kernel = fa::fa_decode_split_kernel<D, GC, KV8>;
  int st = ensure_smem(reinterpret_cast<const void*>(kernel), C::SMEM_BYTES);
  if (st != FA_OK) return st;
  kernel<<<grid, fa::kDecodeThreads, C::SMEM_BYTES, stream>>>(prm);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}

template <int D, bool KV8>
int dispatch_decode_gc(int gc, const fa::DecodeParams& prm, dim3 grid, cudaStream_t stream) {
  switch (gc) {
    case 1: return launch_decode_split<D, 1, KV8>(prm, grid, stream);
    case 2: return launch_decode_split<D, 2, KV8>(prm, grid, stream);
    case 4: return launch_decode_split<D, 4, KV8>(prm, grid, stream);
    case 8: return launch_decode_split<D, 8, KV8>(prm, grid, stream);
  }
  return FA_ERR_UNSUPPORTED;
}

template <bool KV8, int NPAD>
int launch_decode_tc(const fa::DecodeParams& prm, dim3 grid, cudaStream_t stream) {
  using C = fa::DecodeTcCfg<KV8, NPAD>;
  auto kernel = fa::fa_decode_tc_kernel<KV8, NPAD>;
  int st = ensure_smem(reinterpret_cast<const void*>(kernel), C::SMEM_BYTES);
  if (st != FA_OK) return st;
  kernel<<<grid, fa::kDecodeTcThreads, C::SMEM_BYTES, stream>>>(prm);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}

int launch_merge(const fa::MergeParams& mp, int head_dim, cudaStream_t stream) {
  const int rows = mp.rows * mp.num_heads;
  dim3 grid((rows + 3) / 4);
  if (head_dim == 128)
    fa::fa_merge_kernel<128><<<grid, 128, 0, stream>>>(mp);
  else
    fa::fa_merge_kernel<64><<<grid, 128, 0, stream>>>(mp);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}

}  // namespace

// ============================================================================ API

namespace {

// fa_prefill and fa_prefill_fp8 (f8: E4M3 Q/K/V with per-tensor scales).
int prefill_impl(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_dev,
                 const int32_t* cu_seqlens_host, int batch, int num_q_heads, int num_kv_heads,
                 int head_dim, int causal, float scale, bool f8, float q_scale, float k_scale,
                 float v_scale, void* out, float* lse, void* stream) {
  if (!q || !k || !v || !cu_seqlens_dev || !cu_seqlens_host || !out) return FA_ERR_INVALID_ARG;
  if (f8 && head_dim != 128) return FA_ERR_UNSUPPORTED;
  for (float sc : {q_scale, k_scale, v_scale})
    if (!(sc > 0.0f) || std::isinf(sc)) return FA_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || num_q_heads < 1 || num_kv_heads < 1 ||
      num_q_heads > 65535 || num_q_heads % num_kv_heads != 0)
    return FA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(lse, 4) || !aligned(cu_seqlens_dev, 4))
    return FA_ERR_INVALID_ARG;
  scale = resolve_scale(scale, head_dim);
  if (!(scale > 0.0f) || std::isinf(scale)) return FA_ERR_INVALID_ARG;
  if (cu_seqlens_host[0] != 0) return FA_ERR_INVALID_ARG;
  if (num_kv_heads > 65535) return FA_ERR_UNSUPPORTED;
  std::vector<int64_t> lens;
  for (int b = 0; b < batch; ++b) {
    const int64_t L = static_cast<int64_t>(cu_seqlens_host[b + 1]) - cu_seqlens_host[b];
    if (L < 1) return FA_ERR_INVALID_ARG;
    if ((L + 127) / 128 > 65535) return FA_ERR_UNSUPPORTED;
    lens.push_back(L);
  }
  const int64_t T = cu_seqlens_host[batch];
  if (T * num_q_heads * head_dim >= (int64_t{1} << 40)) return FA_ERR_UNSUPPORTED;
  const int group = num_q_heads / num_kv_heads;
  std::vector<std::pair<uint32_t, int>> groups;
  build_prefill_groups(lens, lens, num_q_heads, num_kv_heads, causal != 0, &groups);

  static thread_local fa::PrefillParams prm;   // ~17 KB; kept off the stack
  std::memset(&prm, 0, sizeof(prm));
  // 128-byte boxes: 64 bf16 columns, or all 128 E4M3 columns, of 128 rows
  const int eb = f8 ? 1 : 2;
  const CUtensorMapDataType dt = f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), 1, 128};
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                                static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * eb,
                                   static_cast<cuuint64_t>(num_q_heads) * head_dim * eb};
    int st = encode_map(&prm.tm_q, q, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, dt);
    if (st != FA_OK) return st;
  }
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_kv_heads),
                                static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * eb,
                                   static_cast<cuuint64_t>(num_kv_heads) * head_dim * eb};
    int st = encode_map(&prm.tm_k, k, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, dt);
    if (st != FA_OK) return st;
    st = encode_map(&prm.tm_v, v, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, dt);
    if (st != FA_OK) return st;
  }
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.out_v8 = aligned(out, 32) ? 1 : 0;
  prm.lse = lse;
  prm.cu_seqlens = cu_seqlens_dev;
  prm.total_q = static_cast<int>(T);
  prm.batch = batch;
  prm.num_q_heads = num_q_heads;
  prm.group = group;
  prm.causal = causal ? 1 : 0;
  prm.scale_log2 = scale * kLog2e * q_scale * k_scale;
  prm.v_scale = v_scale;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  t_last_prefill_schedule = -1;
  int st = FA_OK;
  if (prefill_persistent_requested()) {
    uint32_t* sched = prefill_sched_slot(s);
    int sms = 0;
    if (sched != nullptr && sm_count(&sms) == FA_OK) {
      if (f8) st = launch_prefill_persistent<128, true>(prm, groups, s, sched, sms);
      else if (head_dim == 128) st = launch_prefill_persistent<128, false>(prm, groups, s, sched, sms);
      else st = launch_prefill_persistent<64, false>(prm, groups, s, sched, sms);
      if (st == FA_OK) t_last_prefill_schedule = FA_SCHEDULE_PERSISTENT;
      return st;
    }
  }
  if (f8) st = launch_prefill<128, false, true>(prm, groups, s);
  else if (head_dim == 128) st = launch_prefill<128, false>(prm, groups, s);
  else st = launch_prefill<64, false>(prm, groups, s);
  if (st == FA_OK) t_last_prefill_schedule = FA_SCHEDULE_GRID;
  return st;
}

}  // namespace

FA_API int fa_prefill(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_dev,
                      const int32_t* cu_seqlens_host, int batch, int num_q_heads, int num_kv_heads,
                      int head_dim, int causal, float scale, void* out, float* lse, void* stream) {
  return prefill_impl(q, k, v, cu_seqlens_dev, cu_seqlens_host, batch, num_q_heads, num_kv_heads,
                      head_dim, causal, scale, false, 1.0f, 1.0f, 1.0f, out, lse, stream);
}

FA_API int fa_prefill_last_schedule(void) { return t_last_prefill_schedule; }

FA_API int fa_prefill_fp8(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_dev,
                          const int32_t* cu_seqlens_host, int batch, int num_q_heads,
                          int num_kv_heads, int head_dim, int causal, float scale, float q_scale,
                          float k_scale, float v_scale, void* out, float* lse, void* stream) {
  return prefill_impl(q, k, v, cu_seqlens_dev, cu_seqlens_host, batch, num_q_heads, num_kv_heads,
                      head_dim, causal, scale, true, q_scale, k_scale, v_scale, out, lse, stream);
}

FA_API int fa_prefill_paged(const void* q, const int32_t* cu_seqlens_q_dev,
                            const int32_t* cu_seqlens_q_host, const void* k_pages,
                            const void* v_pages, int64_t num_pages, int64_t page_stride,
                            int64_t token_stride, int64_t head_stride, const int32_t* block_table,
                            int max_pages_per_seq, const int32_t* cache_seqlens_dev,
                            const int32_t* cache_seqlens_host, int batch, int num_q_heads,
                            int num_kv_heads, int head_dim, int page_size, int causal, float scale,
                            void* out, float* lse, void* stream) {
  if (!q || !cu_seqlens_q_dev || !cu_seqlens_q_host || !block_table || !cache_seqlens_dev ||
      !cache_seqlens_host || !out)
    return FA_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || num_q_heads < 1 || num_kv_heads < 1 ||
      num_q_heads > 65535 || num_q_heads % num_kv_heads != 0 || max_pages_per_seq < 1)
    return FA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return FA_ERR_UNSUPPORTED;
  if (page_size != fa::kPrefillPage) return FA_ERR_UNSUPPORTED;
  if (num_kv_heads > 65535) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(cu_seqlens_q_dev, 4) ||
      !aligned(block_table, 4) || !aligned(cache_seqlens_dev, 4))
    return FA_ERR_INVALID_ARG;
  if (!valid_pool(k_pages, v_pages, num_pages, page_stride, token_stride, head_stride))
    return FA_ERR_INVALID_ARG;
  scale = resolve_scale(scale, head_dim);
  if (!(scale > 0.0f) || std::isinf(scale)) return FA_ERR_INVALID_ARG;
  if (cu_seqlens_q_host[0] != 0) return FA_ERR_INVALID_ARG;
  const int64_t capacity = static_cast<int64_t>(max_pages_per_seq) * page_size;
  if (capacity > (int64_t{1} << 30)) return FA_ERR_INVALID_ARG;   // as for fa_decode_plan
  std::vector<int64_t> q_lens, k_lens;
  for (int b = 0; b < batch; ++b) {
    const int64_t lq = static_cast<int64_t>(cu_seqlens_q_host[b + 1]) - cu_seqlens_q_host[b];
    const int64_t lk = cache_seqlens_host[b];
    if (lq < 1 || lk < lq || lk > capacity) return FA_ERR_INVALID_ARG;
    if ((lq + 127) / 128 > 65535) return FA_ERR_UNSUPPORTED;
    q_lens.push_back(lq);
    k_lens.push_back(lk);
  }
  const int64_t T = cu_seqlens_q_host[batch];
  if (T * num_q_heads * head_dim >= (int64_t{1} << 40)) return FA_ERR_UNSUPPORTED;
  std::vector<std::pair<uint32_t, int>> groups;
  build_prefill_groups(q_lens, k_lens, num_q_heads, num_kv_heads, causal != 0, &groups);

  static thread_local fa::PrefillParams prm;
  std::memset(&prm, 0, sizeof(prm));
  {
    const cuuint32_t box[3] = {64, 1, 128};
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                                static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                                   static_cast<cuuint64_t>(num_q_heads) * head_dim * 2};
    int st = encode_map(&prm.tm_q, q, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != FA_OK) return st;
  }
  int st = encode_page_pool_map(&prm.tm_k, k_pages, num_pages, page_stride, token_stride, head_stride,
                                page_size, num_kv_heads, head_dim, 64, CU_TENSOR_MAP_SWIZZLE_128B,
                                &prm.head_coord, &prm.page_coord);
  if (st != FA_OK) return st;
  st = encode_page_pool_map(&prm.tm_v, v_pages, num_pages, page_stride, token_stride, head_stride,
                            page_size, num_kv_heads, head_dim, 64, CU_TENSOR_MAP_SWIZZLE_128B,
                            &prm.head_coord, &prm.page_coord);
  if (st != FA_OK) return st;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.out_v8 = aligned(out, 32) ? 1 : 0;
  prm.lse = lse;
  prm.cu_seqlens = cu_seqlens_q_dev;
  prm.total_q = static_cast<int>(T);
  prm.batch = batch;
  prm.block_table = block_table;
  prm.cache_seqlens = cache_seqlens_dev;
  prm.max_pages = max_pages_per_seq;
  prm.num_pages = static_cast<int>(num_pages);
  prm.num_q_heads = num_q_heads;
  prm.group = num_q_heads / num_kv_heads;
  prm.causal = causal ? 1 : 0;
  prm.scale_log2 = scale * kLog2e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  t_last_prefill_schedule = -1;
  if (prefill_persistent_requested()) {
    uint32_t* sched = prefill_sched_slot(s);
    int sms = 0;
    if (sched != nullptr && sm_count(&sms) == FA_OK) {
      st = head_dim == 128 ? launch_prefill_persistent<128, false, true>(prm, groups, s, sched, sms)
                           : launch_prefill_persistent<64, false, true>(prm, groups, s, sched, sms);
      if (st == FA_OK) t_last_prefill_schedule = FA_SCHEDULE_PERSISTENT;
      return st;
    }
  }
  st = head_dim == 128 ? launch_prefill<128, true>(prm, groups, s) : launch_prefill<64, true>(prm, groups, s);
  if (st == FA_OK) t_last_prefill_schedule = FA_SCHEDULE_GRID;
  return st;
}

FA_API int fa_append_kv(const void* k_new, const void* v_new, const int32_t* cu_seqlens_new_dev,
                        int total_new, int batch, int num_kv_heads, int head_dim, void* k_pages,
                        void* v_pages, int64_t num_pages, int64_t page_stride,
                        int64_t token_stride, int64_t head_stride, int page_size,
                        const int32_t* block_table, int max_pages_per_seq,
                        const int32_t* cache_seqlens_dev, void* stream) {
  if (!k_new || !v_new || !cu_seqlens_new_dev || !block_table || !cache_seqlens_dev)
    return FA_ERR_INVALID_ARG;
  if (total_new < 0 || batch < 1 || num_kv_heads < 1 || max_pages_per_seq < 1)
    return FA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return FA_ERR_UNSUPPORTED;
  if (page_size != fa::kAppendPage) return FA_ERR_UNSUPPORTED;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(cu_seqlens_new_dev, 4) ||
      !aligned(block_table, 4) || !aligned(cache_seqlens_dev, 4))
    return FA_ERR_INVALID_ARG;
  if (!valid_pool(k_pages, v_pages, num_pages, page_stride, token_stride, head_stride))
    return FA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_pages_per_seq) * page_size > INT32_MAX) return FA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(total_new) * num_kv_heads * head_dim >= (int64_t{1} << 40))
    return FA_ERR_UNSUPPORTED;
  if (total_new == 0) return FA_OK;
  fa::AppendParams ap;
  ap.k_new = static_cast<const uint4*>(k_new);
  ap.v_new = static_cast<const uint4*>(v_new);
  ap.cu_seqlens = cu_seqlens_new_dev;
  ap.cache_seqlens = cache_seqlens_dev;
  ap.block_table = block_table;
  ap.k_pages = static_cast<__nv_bfloat16*>(k_pages);
  ap.v_pages = static_cast<__nv_bfloat16*>(v_pages);
  ap.page_stride = page_stride;
  ap.token_stride = token_stride;
  ap.head_stride = head_stride;
  ap.pool_elems = (num_pages - 1) * page_stride + (page_size - 1) * token_stride +
                  (num_kv_heads - 1) * head_stride + head_dim;
  ap.total_new = total_new;
  ap.batch = batch;
  ap.num_kv_heads = num_kv_heads;
  ap.max_pages = max_pages_per_seq;
  ap.num_pages = static_cast<int>(num_pages);
  // One warp per token; a grid of at most 8 blocks per SM loops over the rest.
  int sms = 0;
  const int st = sm_count(&sms);
  if (st != FA_OK) return st;
  const int64_t want = (static_cast<int64_t>(total_new) + 7) / 8;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(want, static_cast<int64_t>(sms) * 8));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (head_dim == 128)
    fa::fa_append_kv_kernel<128><<<grid, fa::kAppendThreads, 0, s>>>(ap);
  else
    fa::fa_append_kv_kernel<64><<<grid, fa::kAppendThreads, 0, s>>>(ap);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}

FA_API int fa_decode_plan_ex(const int32_t* cache_seqlens_host, int batch, int num_q_heads,
                             int num_kv_heads, int head_dim, int page_size, int max_pages_per_seq,
                             int num_sms, int num_splits_override, const fa_decode_options* options,
                             fa_plan** plan_out, size_t* workspace_bytes) {
  if (plan_out == nullptr || options == nullptr) return FA_ERR_INVALID_ARG;
  *plan_out = nullptr;
  const int kv_dtype = options->kv_dtype;
  if (kv_dtype != FA_KV_BF16 && kv_dtype != FA_KV_E4M3) return FA_ERR_INVALID_ARG;
  fa::DecodePlan p;
  int st = fa::make_decode_plan(cache_seqlens_host, batch, num_q_heads, num_kv_heads, head_dim,
                                page_size, max_pages_per_seq, num_sms, num_splits_override,
                                kv_dtype == FA_KV_E4M3 ? 1 : 2, options->kernel, options->q_len, &p);
  if (st != FA_OK) return st;
  fa_plan* plan = new (std::nothrow) fa_plan;
  if (plan == nullptr) return FA_ERR_INVALID_ARG;
  plan->p = std::move(p);
  *plan_out = plan;
  if (workspace_bytes) *workspace_bytes = plan->p.workspace_bytes;
  return FA_OK;
}

FA_API int fa_decode_plan_kv(const int32_t* cache_seqlens_host, int batch, int num_q_heads,
                             int num_kv_heads, int head_dim, int page_size, int max_pages_per_seq,
                             int num_sms, int num_splits_override, int kv_dtype, int kernel,
                             fa_plan** plan_out, size_t* workspace_bytes) {
  const fa_decode_options o = {kv_dtype, kernel, 1};
  return fa_decode_plan_ex(cache_seqlens_host, batch, num_q_heads, num_kv_heads, head_dim, page_size,
                           max_pages_per_seq, num_sms, num_splits_override, &o, plan_out,
                           workspace_bytes);
}

FA_API int fa_decode_plan(const int32_t* cache_seqlens_host, int batch, int num_q_heads,
                          int num_kv_heads, int head_dim, int page_size, int max_pages_per_seq,
                          int num_sms, int num_splits_override, fa_plan** plan_out,
                          size_t* workspace_bytes) {
  return fa_decode_plan_kv(cache_seqlens_host, batch, num_q_heads, num_kv_heads, head_dim, page_size,
                           max_pages_per_seq, num_sms, num_splits_override, FA_KV_BF16,
                           FA_DECODE_AUTO, plan_out, workspace_bytes);
}

FA_API int fa_plan_get_info(const fa_plan* plan, fa_plan_info* info) {
  if (plan == nullptr || info == nullptr || plan->p.magic != fa::kPlanMagic) return FA_ERR_INVALID_ARG;
  const auto& p = plan->p;
  info->batch = p.batch;
  info->num_q_heads = p.num_q_heads;
  info->num_kv_heads = p.num_kv_heads;
  info->head_dim = p.head_dim;
  info->page_size = p.page_size;
  info->max_pages_per_seq = p.max_pages_per_seq;
  info->chunk_tokens = p.chunk_tokens;
  info->max_splits = p.max_splits;
  info->heads_per_cta = p.heads_per_cta;
  info->num_work_items = p.num_work_items;
  info->max_seqlen = p.max_seqlen;
  info->workspace_bytes = p.workspace_bytes;
  info->kv_dtype = p.kv_elem_bytes == 1 ? FA_KV_E4M3 : FA_KV_BF16;
  info->tensor_cores = p.tensor_cores ? 1 : 0;
  info->q_len = p.q_len;
  return FA_OK;
}

FA_API void fa_plan_free(fa_plan* plan) {
  if (plan != nullptr) {
    plan->p.magic = 0;
    delete plan;
  }
}

namespace {

// fa_decode_paged and fa_decode_paged_fp8: kv8 selects E4M3 pages with
// per-tensor scales (k_scale, v_scale); both are 1 for a bf16 cache.
int decode_paged_impl(const void* q, const void* k_pages, const void* v_pages, int64_t num_pages,
                      int64_t page_stride, int64_t token_stride, int64_t head_stride,
                      const int32_t* block_table, const int32_t* cache_seqlens_dev,
                      const fa_plan* plan, float scale, bool kv8, float k_scale, float v_scale,
                      void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (plan == nullptr || plan->p.magic != fa::kPlanMagic) return FA_ERR_INVALID_ARG;
  const fa::DecodePlan& pl = plan->p;
  if (!q || !k_pages || !v_pages || !block_table || !cache_seqlens_dev || !out)
    return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(out, 16) ||
      !aligned(lse, 4) || !aligned(block_table, 4) || !aligned(cache_seqlens_dev, 4))
    return FA_ERR_INVALID_ARG;
  const int elem_bytes = kv8 ? 1 : 2;
  if (pl.kv_elem_bytes != elem_bytes) return FA_ERR_PLAN_MISMATCH;
  if (!valid_pool(k_pages, v_pages, num_pages, page_stride, token_stride, head_stride, elem_bytes))
    return FA_ERR_INVALID_ARG;
  if (!(k_scale > 0.0f) || std::isinf(k_scale) || !(v_scale > 0.0f) || std::isinf(v_scale))
    return FA_ERR_INVALID_ARG;
  if (pl.workspace_bytes > 0) {
    if (workspace == nullptr || !aligned(workspace, 256)) return FA_ERR_INVALID_ARG;
    if (workspace_bytes < pl.workspace_bytes) return FA_ERR_WORKSPACE;
  }
  scale = resolve_scale(scale, pl.head_dim);
  if (!(scale > 0.0f) || std::isinf(scale)) return FA_ERR_INVALID_ARG;

  static thread_local fa::DecodeParams prm;
  std::memset(&prm, 0, sizeof(prm));
  // CUDA-core kernel: whole rows (d columns) of one 64-token page per box, no
  // swizzle.  Tensor-core kernel: 128-byte column chunks with the 128-byte
  // swizzle the MMA operand descriptors expect.
  const int box_cols = pl.tensor_cores ? 128 / elem_bytes : pl.head_dim;
  const CUtensorMapSwizzle swz = pl.tensor_cores ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  int st = encode_page_pool_map(&prm.tm_k, k_pages, num_pages, page_stride, token_stride, head_stride,
                                pl.page_size, pl.num_kv_heads, pl.head_dim, box_cols, swz,
                                &prm.head_coord, &prm.page_coord, elem_bytes);
  if (st != FA_OK) return st;
  st = encode_page_pool_map(&prm.tm_v, v_pages, num_pages, page_stride, token_stride, head_stride,
                            pl.page_size, pl.num_kv_heads, pl.head_dim, box_cols, swz,
                            &prm.head_coord, &prm.page_coord, elem_bytes);
  if (st != FA_OK) return st;
  const int npad = pl.q_len * pl.group <= 8 ? 8 : 16;
  if (pl.tensor_cores && !kv8) {
    // q [B, q_len, Hq, d]: a box is the G heads of one kv head for every token
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(pl.head_dim),
                                static_cast<cuuint64_t>(pl.num_q_heads),
                                static_cast<cuuint64_t>(pl.q_len), static_cast<cuuint64_t>(pl.batch)};
    const cuuint64_t strides[3] = {
        static_cast<cuuint64_t>(pl.head_dim) * 2,
        static_cast<cuuint64_t>(pl.num_q_heads) * pl.head_dim * 2,
        static_cast<cuuint64_t>(pl.q_len) * pl.num_q_heads * pl.head_dim * 2};
    const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(pl.group), static_cast<cuuint32_t>(pl.q_len), 1};
    st = encode_map(&prm.tm_q, q, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != FA_OK) return st;
  }

  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.block_table = block_table;
  prm.cache_seqlens = cache_seqlens_dev;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.ws_o = pl.workspace_bytes ? reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.ws_o_offset)
                                : nullptr;
  prm.ws_lse = pl.workspace_bytes
                   ? reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.ws_lse_offset)
                   : nullptr;
  prm.batch = pl.batch;
  prm.q_len = pl.q_len;
  prm.num_q_heads = pl.num_q_heads;
  prm.group = pl.group;
  prm.subgroups = pl.subgroups;
  prm.max_pages = pl.max_pages_per_seq;
  prm.num_pages = static_cast<int>(num_pages);
  prm.chunk_tokens = pl.chunk_tokens;
  prm.max_splits = pl.max_splits;
  prm.scale_log2 = scale * kLog2e * k_scale;
  prm.v_scale = v_scale;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dim3 grid(pl.max_splits, pl.num_kv_heads * pl.subgroups, pl.batch);
  if (pl.tensor_cores) {
    if (kv8)
      st = npad == 8 ? launch_decode_tc<true, 8>(prm, grid, s) : launch_decode_tc<true, 16>(prm, grid, s);
    else
      st = npad == 8 ? launch_decode_tc<false, 8>(prm, grid, s) : launch_decode_tc<false, 16>(prm, grid, s);
  } else if (kv8)
    st = pl.head_dim == 128 ? dispatch_decode_gc<128, true>(pl.heads_per_cta, prm, grid, s)
                            : dispatch_decode_gc<64, true>(pl.heads_per_cta, prm, grid, s);
  else
    st = pl.head_dim == 128 ? dispatch_decode_gc<128, false>(pl.heads_per_cta, prm, grid, s)
                            : dispatch_decode_gc<64, false>(pl.heads_per_cta, prm, grid, s);
  if (st != FA_OK) return st;
  if (pl.max_splits > 1) {
    fa::MergeParams mp;
    mp.o_parts = prm.ws_o;
    mp.lse_parts = prm.ws_lse;
    mp.out = prm.out;
    mp.lse = lse;
    mp.cache_seqlens = cache_seqlens_dev;
    mp.q_len = pl.q_len;
    mp.num_states = pl.max_splits;
    mp.rows = pl.batch * pl.q_len;
    mp.num_heads = pl.num_q_heads;
    mp.chunk_tokens = pl.chunk_tokens;
    mp.max_pages = pl.max_pages_per_seq;
    st = launch_merge(mp, pl.head_dim, s);
  }
  return st;
}

}  // namespace

FA_API int fa_decode_paged(const void* q, const void* k_pages, const void* v_pages, int64_t num_pages,
                           int64_t page_stride, int64_t token_stride, int64_t head_stride,
                           const int32_t* block_table, const int32_t* cache_seqlens_dev,
                           const fa_plan* plan, float scale, void* out, float* lse, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return decode_paged_impl(q, k_pages, v_pages, num_pages, page_stride, token_stride, head_stride,
                           block_table, cache_seqlens_dev, plan, scale, false, 1.0f, 1.0f, out, lse,
                           workspace, workspace_bytes, stream);
}

FA_API int fa_decode_paged_fp8(const void* q, const void* k_pages, const void* v_pages,
                               int64_t num_pages, int64_t page_stride, int64_t token_stride,
                               int64_t head_stride, const int32_t* block_table,
                               const int32_t* cache_seqlens_dev, const fa_plan* plan, float scale,
                               float k_scale, float v_scale, void* out, float* lse, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return decode_paged_impl(q, k_pages, v_pages, num_pages, page_stride, token_stride, head_stride,
                           block_table, cache_seqlens_dev, plan, scale, true, k_scale, v_scale, out,
                           lse, workspace, workspace_bytes, stream);
}

FA_API int fa_merge_states(const float* o_parts, const float* lse_parts, int num_states, int rows,
                           int num_heads, int head_dim, void* out, float* lse, void* stream) {
  if (!o_parts || !lse_parts || !out) return FA_ERR_INVALID_ARG;
  if (num_states < 1 || rows < 1 || num_heads < 1) return FA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(o_parts, 16) || !aligned(lse_parts, 4) || !aligned(out, 16) || !aligned(lse, 4))
    return FA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(rows) * num_heads > INT32_MAX / 4) return FA_ERR_UNSUPPORTED;
  fa::MergeParams mp;
  mp.o_parts = o_parts;
  mp.lse_parts = lse_parts;
  mp.out = static_cast<__nv_bfloat16*>(out);
  mp.lse = lse;
  mp.cache_seqlens = nullptr;
  mp.q_len = 1;
  mp.num_states = num_states;
  mp.rows = rows;
  mp.num_heads = num_heads;
  mp.chunk_tokens = 1;
  mp.max_pages = 0;
  return launch_merge(mp, head_dim, static_cast<cudaStream_t>(stream));
}

FA_API const char* fa_strerror(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_WORKSPACE: return "workspace too small";
    case FA_ERR_CUDA: return "CUDA call failed";
    case FA_ERR_TIMEOUT: return "device wait timed out";
    case FA_ERR_PLAN_MISMATCH: return "plan does not cover the call";
    case FA_ERR_BAD_PAGE: return "block_table entry outside the page pool";
    case FA_ERR_DEBUG_INDEX: return "index outside its buffer (bounds-checked build)";
  }
  return "unknown status";
}

FA_API int fa_last_cuda_error(void) { return t_last_cuda_error; }

FA_API int fa_get_device_status(void* stream, int* status_host, int clear) {
  if (status_host == nullptr) return FA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FA_CUDA_CHECK(cudaStreamSynchronize(s));
  int v = 0;
  FA_CUDA_CHECK(cudaMemcpyFromSymbol(&v, fa::g_device_status, sizeof(int)));
  if (clear) {
    const int zero = 0;
    FA_CUDA_CHECK(cudaMemcpyToSymbol(fa::g_device_status, &zero, sizeof(int)));
  }
  *status_host = v;
  return FA_OK;
}

FA_API int fa_selftest_wait_timeout(int64_t limit_us, void* stream) {
  const int64_t us = std::min<int64_t>(std::max<int64_t>(limit_us, 1000), 2000000);
  fa::fa_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(us) * 1000ull);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}

FA_API int fa_version(void) { return 100; }

#ifdef FA_DEBUG
namespace fa {
// buf[0] = 1, then a store at n/2 + 1 checked against a logical extent of n/2.
__global__ void fa_debug_selftest_index_kernel(int32_t* buf, int n) {
  const int half = n / 2;
  if (FA_DBG_OK(0 < half)) buf[0] = 1;
  if (FA_DBG_OK(half + 1 < half)) buf[half + 1] = 1;
}
}  // namespace fa
#endif

FA_API int fa_debug_selftest_index(int32_t* buf, int n, void* stream) {
  if (buf == nullptr || n < 4 || !aligned(buf, 4)) return FA_ERR_INVALID_ARG;
#ifdef FA_DEBUG
  fa::fa_debug_selftest_index_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(buf, n);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
#else
  (void)stream;
  return FA_ERR_UNSUPPORTED;
#endif
}

// ============================================================================
// Scratch-free decode (fa_decode_paged_static): the split partials go to a
// fixed static device array instead of a caller workspace, for callers that
// cannot allocate device memory.  Host code must not use the array's name as a
// device address; its address is looked up once per device below.
namespace {

constexpr size_t kStaticScratchBytes = FA_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 128;

// Device address of g_static_scratch on the current device, looked up with
// cudaGetSymbolAddress the first time each device asks and cached after that.
int static_scratch_address(void** addr_out) {
  int dev = 0;
  FA_CUDA_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    addr[dev] = ptr;
  }
  *addr_out = addr[dev];
  return FA_OK;
}

}  // namespace

FA_API int fa_decode_paged_static(const void* q, const void* k_pages, const void* v_pages,
                                  int64_t num_pages, int64_t page_stride, int64_t token_stride,
                                  int64_t head_stride, const int32_t* block_table,
                                  const int32_t* cache_seqlens_dev, const fa_plan* plan, float scale,
                                  void* out, float* lse, void* stream) {
  if (plan == nullptr || plan->p.magic != fa::kPlanMagic) return FA_ERR_INVALID_ARG;
  if (plan->p.workspace_bytes > kStaticScratchBytes) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (plan->p.workspace_bytes > 0) {
    const int st = static_scratch_address(&scratch);
    if (st != FA_OK) return st;
  }
  return fa_decode_paged(q, k_pages, v_pages, num_pages, page_stride, token_stride, head_stride,
                         block_table, cache_seqlens_dev, plan, scale, out, lse, scratch,
                         kStaticScratchBytes, stream);
}

// ============================================================================
// Cascade (prefix-sharing) decode: every request's query attends to one shared
// prefix (read once for the whole batch by the paged prefill kernel, the
// requests acting as the query tokens of one full-attention sequence, cut into
// key ranges to fill the SMs) and to its own suffix (the paged decode); the
// two states are merged by LSE.
namespace {

struct CascadeLayout {
  int splits = 0, split_tiles = 0;
  size_t off_so = 0, off_sl = 0, off_po = 0, off_pl = 0, total = 0;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

CascadeLayout cascade_layout(const fa::DecodePlan& pl, int prefix_len) {
  CascadeLayout c;
  const size_t rows = static_cast<size_t>(pl.batch) * pl.num_q_heads;
  c.off_so = align256(pl.workspace_bytes);
  c.off_sl = align256(c.off_so + rows * pl.head_dim * 2);
  c.off_po = align256(c.off_sl + rows * 4);
  if (prefix_len > 0) {
    const int n_ktiles = (prefix_len + 127) / 128;
    const int n_qtiles = (pl.batch + 127) / 128;
    const int g = pl.group;
    const int per_head = (g % 2 == 0) ? n_qtiles * (g / 2) : ((n_qtiles + 1) / 2) * g;
    const int base = per_head * pl.num_kv_heads;             // CTAs per key range
    const int want = std::max(1, pl.num_sms / base);     // one wave of CTAs
    c.splits = std::min(want, n_ktiles);
    c.split_tiles = (n_ktiles + c.splits - 1) / c.splits;
    c.splits = (n_ktiles + c.split_tiles - 1) / c.split_tiles;
  }
  c.off_pl = align256(c.off_po + static_cast<size_t>(c.splits) * rows * pl.head_dim * 4);
  c.total = align256(c.off_pl + static_cast<size_t>(c.splits) * rows * 4);
  return c;
}

}  // namespace

FA_API int fa_cascade_workspace_bytes(const fa_plan* plan, int prefix_len, size_t* bytes) {
  if (plan == nullptr || plan->p.magic != fa::kPlanMagic || bytes == nullptr || prefix_len < 0)
    return FA_ERR_INVALID_ARG;
  *bytes = cascade_layout(plan->p, prefix_len).total;
  return FA_OK;
}

FA_API int fa_cascade_decode(const void* q, const void* k_pages, const void* v_pages,
                             int64_t num_pages, int64_t page_stride, int64_t token_stride,
                             int64_t head_stride, const int32_t* prefix_block_table,
                             int prefix_len, const int32_t* block_table,
                             const int32_t* cache_seqlens_dev, const fa_plan* plan, float scale,
                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (plan == nullptr || plan->p.magic != fa::kPlanMagic) return FA_ERR_INVALID_ARG;
  const fa::DecodePlan& pl = plan->p;
  if (pl.kv_elem_bytes != 2 || pl.q_len != 1) return FA_ERR_PLAN_MISMATCH;
  if (!q || !out || !workspace || prefix_len < 0 || (prefix_len > 0 && !prefix_block_table))
    return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(workspace, 256) ||
      !aligned(prefix_block_table, 4))
    return FA_ERR_INVALID_ARG;
  if (!valid_pool(k_pages, v_pages, num_pages, page_stride, token_stride, head_stride))
    return FA_ERR_INVALID_ARG;
  const CascadeLayout c = cascade_layout(pl, prefix_len);
  if (workspace_bytes < c.total) return FA_ERR_WORKSPACE;
  scale = resolve_scale(scale, pl.head_dim);
  if (!(scale > 0.0f) || std::isinf(scale)) return FA_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (prefix_len == 0)   // nothing shared: the plain decode
    return decode_paged_impl(q, k_pages, v_pages, num_pages, page_stride, token_stride, head_stride,
                             block_table, cache_seqlens_dev, plan, scale, false, 1.0f, 1.0f, out,
                             lse, workspace, pl.workspace_bytes, stream);

  // 1. shared prefix: B "tokens" (one per request) x Hq heads, full attention
  static thread_local fa::PrefillParams prm;
  std::memset(&prm, 0, sizeof(prm));
  {
    const cuuint32_t box[3] = {64, 1, 128};
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(pl.head_dim), static_cast<cuuint64_t>(pl.num_q_heads),
                                static_cast<cuuint64_t>(pl.batch)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(pl.head_dim) * 2,
                                   static_cast<cuuint64_t>(pl.num_q_heads) * pl.head_dim * 2};
    int st = encode_map(&prm.tm_q, q, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != FA_OK) return st;
  }
  int st = encode_page_pool_map(&prm.tm_k, k_pages, num_pages, page_stride, token_stride, head_stride,
                                pl.page_size, pl.num_kv_heads, pl.head_dim, 64,
                                CU_TENSOR_MAP_SWIZZLE_128B, &prm.head_coord, &prm.page_coord);
  if (st != FA_OK) return st;
  st = encode_page_pool_map(&prm.tm_v, v_pages, num_pages, page_stride, token_stride, head_stride,
                            pl.page_size, pl.num_kv_heads, pl.head_dim, 64, CU_TENSOR_MAP_SWIZZLE_128B,
                            &prm.head_coord, &prm.page_coord);
  if (st != FA_OK) return st;
  prm.cu_seqlens = nullptr;
  prm.batch = 1;                     // one sequence: the batch's queries over the prefix
  prm.uniform_q_len = pl.batch;
  prm.cache_seqlens = nullptr;
  prm.uniform_k_len = prefix_len;
  prm.block_table = prefix_block_table;
  prm.max_pages = (prefix_len + pl.page_size - 1) / pl.page_size;
  prm.num_pages = static_cast<int>(num_pages);
  prm.num_q_heads = pl.num_q_heads;
  prm.group = pl.group;
  prm.causal = 0;
  prm.scale_log2 = scale * kLog2e;
  prm.kv_splits = c.splits;
  prm.kv_split_tiles = c.split_tiles;
  prm.total_q = pl.batch;
  prm.part_o = reinterpret_cast<float*>(ws + c.off_po);
  prm.part_lse = reinterpret_cast<float*>(ws + c.off_pl);
  std::vector<std::pair<uint32_t, int>> groups;
  build_prefill_groups({static_cast<int64_t>(pl.batch)}, {static_cast<int64_t>(prefix_len)},
                       pl.num_q_heads, pl.num_kv_heads, false, &groups);
  for (auto& g : groups) g.second *= c.splits;
  st = pl.head_dim == 128 ? launch_prefill<128, true>(prm, groups, s) : launch_prefill<64, true>(prm, groups, s);
  if (st != FA_OK) return st;

  // 2. each request's own suffix
  __nv_bfloat16* so = reinterpret_cast<__nv_bfloat16*>(ws + c.off_so);
  float* sl = reinterpret_cast<float*>(ws + c.off_sl);
  st = decode_paged_impl(q, k_pages, v_pages, num_pages, page_stride, token_stride, head_stride,
                         block_table, cache_seqlens_dev, plan, scale, false, 1.0f, 1.0f, so, sl,
                         workspace, pl.workspace_bytes, stream);
  if (st != FA_OK) return st;

  // 3. LSE merge of the prefix ranges and the suffix
  fa::CascadeMergeParams mp;
  mp.prefix_o = prm.part_o;
  mp.prefix_lse = prm.part_lse;
  mp.suffix_o = so;
  mp.suffix_lse = sl;
  mp.out = static_cast<__nv_bfloat16*>(out);
  mp.lse = lse;
  mp.num_prefix = c.splits;
  mp.rows = pl.batch;
  mp.num_heads = pl.num_q_heads;
  dim3 grid((pl.batch * pl.num_q_heads + 3) / 4);
  if (pl.head_dim == 128)
    fa::fa_cascade_merge_kernel<128><<<grid, 128, 0, s>>>(mp);
  else
    fa::fa_cascade_merge_kernel<64><<<grid, 128, 0, s>>>(mp);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}
