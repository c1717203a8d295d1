#include "planner.h"

#include <algorithm>
#include <functional>
#include <limits>
#include <vector>

#include "../../include/exact_attention.h"

namespace fa {

namespace {
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Decode-time model used to choose the split size (fitted to B200 timings,
// 148 SMs): all resident split CTAs share the HBM bandwidth, one CTA alone
// cannot pull more than its ceiling, each CTA costs a fixed fill/drain time,
// and a second (merge) launch costs ~5 us.  Per kernel (CTA ceiling, fill,
// CTAs per SM): CUDA cores 44 GB/s, 0.5 us, 2 (1 with 8 packed heads; its
// E4M3 ring holds as many bytes as the bf16 one); tensor cores with 8 padded
// rows (96 KB ring of K and V tiles) 30 GB/s, 2 us, 2; with 16 padded rows
// (192 KB ring) 50 GB/s, 10 us, 1 for bf16 and 30 GB/s, 7 us, 1 for E4M3.
constexpr double kHbmBytesPerUs148 = 6.9e6;       // bytes per microsecond, 148 SMs
constexpr double kMergeLaunchUs = 5.0;

struct CtaModel {
  double bytes_per_us;   // one CTA's ceiling
  double overhead_us;    // fill and drain of one CTA
  int ctas_per_sm;
};

CtaModel cta_model(bool tensor_cores, int kv_elem_bytes, int heads_per_cta) {
  if (tensor_cores) {
    // 8 padded rows: 96 KB ring, two CTAs per SM; 16: 192 KB ring, one
    const bool wide = heads_per_cta > 8;
    if (!wide) return CtaModel{3.0e4, 2.0, 2};
    return kv_elem_bytes == 1 ? CtaModel{3.0e4, 7.0, 1} : CtaModel{5.0e4, 10.0, 1};
  }
  return {4.36e4, 0.5, heads_per_cta == 8 ? 1 : 2};
}

// Estimated duration (us) of the split kernel (+ merge) for one chunk size:
// CTAs enter the resident slots in grid order (split fastest, then kv-head
// group, then request) and every running CTA moves at min(one CTA's limit,
// HBM bandwidth / running CTAs).  Event simulation over a min-heap of finish
// points measured in "bytes done by every running CTA" (all running CTAs
// advance at the same rate, so that scale is shared).  The elapsed time only
// grows as events are processed, so the simulation stops, returning a value
// above `cutoff`, as soon as it passes `cutoff` (a candidate that cannot win).
// Buffers of one simulation, kept across the candidates of a plan.
struct SimScratch {
  std::vector<double> ring, lastq, heap;
  std::vector<int32_t> qhead, qtail;
  std::vector<std::pair<double, int32_t>> fronts;
};

double estimate_decode_us(const std::vector<int32_t>& lens, int64_t units, int64_t chunk, int slots,
                          int head_dim, int kv_elem_bytes, const CtaModel& cm, int num_sms,
                          int max_len, double cutoff, SimScratch& sc) {
  const double bytes_per_token = 2.0 * head_dim * kv_elem_bytes;   // K and V rows of one kv head
  const double hbm = kHbmBytesPerUs148 * num_sms / 148.0;
  const double cta_bytes_per_us = cm.bytes_per_us;
  const double overhead_bytes = cm.overhead_us * cta_bytes_per_us;
  const double full = static_cast<double>(chunk) * bytes_per_token + overhead_bytes;
  // Running CTAs' finish points (bytes done by every running CTA).  Full-chunk
  // CTAs start in non-decreasing order and all have the same size, so their
  // finish points come in order: a FIFO ring holds them.  The other CTAs
  // (each request's last split, one per unit) have the request's own size,
  // so a request's finish in the order they start: each request's wait in a
  // queue of their own (lastq, units entries per request) and a min-heap
  // holds the first of every request with some running, a handful of requests
  // rather than every running CTA.  (Past kMaxQueuedLast entries one heap of
  // all running last splits is used instead.)  The next event is the smaller
  // of the two fronts, so events come in the same order as from one heap of
  // all running CTAs.
  std::vector<double>& ring = sc.ring;
  ring.resize(static_cast<size_t>(std::max(slots, 1)));
  size_t head = 0, count = 0;
  const bool queued = static_cast<int64_t>(lens.size()) * units <= kMaxQueuedLast;
  std::vector<double>& lastq = sc.lastq;
  std::vector<int32_t>& qhead = sc.qhead;
  std::vector<int32_t>& qtail = sc.qtail;
  if (queued) {
    lastq.resize(lens.size() * static_cast<size_t>(units));
    qhead.assign(lens.size(), 0);
    qtail.assign(lens.size(), 0);
  }
  using Front = std::pair<double, int32_t>;   // (finish point, request)
  std::vector<Front>& fronts = sc.fronts;     // min-heap of each request's first
  std::vector<double>& heap = sc.heap;        // min-heap of all (past kMaxQueuedLast)
  fronts.clear();
  heap.clear();
  size_t running_last = 0;
  const auto later = std::greater<double>();
  const auto later_front = [](const Front& x, const Front& y) { return x.first > y.first; };
  auto start_cta = [&](double finish, bool full_chunk, size_t req) {
    if (full_chunk) {
      size_t at = head + count;
      if (at >= ring.size()) at -= ring.size();
      ring[at] = finish;
      ++count;
      return;
    }
    ++running_last;
    if (queued) {
      lastq[req * static_cast<size_t>(units) + static_cast<size_t>(qtail[req])] = finish;
      if (qtail[req]++ == qhead[req]) {
        fronts.emplace_back(finish, static_cast<int32_t>(req));
        std::push_heap(fronts.begin(), fronts.end(), later_front);
      }
    } else {
      heap.push_back(finish);
      std::push_heap(heap.begin(), heap.end(), later);
    }
  };
  auto last_front = [&]() { return queued ? fronts.front().first : heap.front(); };
  auto pop_last = [&]() {
    --running_last;
    if (queued) {
      const int32_t r = fronts.front().second;
      std::pop_heap(fronts.begin(), fronts.end(), later_front);
      fronts.pop_back();
      if (++qhead[r] < qtail[r]) {
        fronts.emplace_back(lastq[static_cast<size_t>(r) * static_cast<size_t>(units) + static_cast<size_t>(qhead[r])], r);
        std::push_heap(fronts.begin(), fronts.end(), later_front);
      }
    } else {
      std::pop_heap(heap.begin(), heap.end(), later);
      heap.pop_back();
    }
  };
  // CTAs in grid order: request b's n splits (every one a full chunk but the
  // last), repeated for each of the units, then request b + 1.
  size_t b = 0;
  int64_t u = 0, sidx = 0, n = 1;
  double last = 0.0;
  auto load = [&]() {
    const int64_t L = lens[b];
    n = std::max<int64_t>(1, ceil_div(L, chunk));
    last = static_cast<double>(std::max<int64_t>(0, L - (n - 1) * chunk)) * bytes_per_token + overhead_bytes;
  };
  if (!lens.empty()) load();
  // start the next CTA at v, if any is left
  auto next_cta = [&](double v) -> bool {
    if (b >= lens.size()) return false;
    const bool is_full = sidx != n - 1;
    start_cta(v + (is_full ? full : last), is_full, b);
    if (++sidx == n) {
      sidx = 0;
      if (++u == units) {
        u = 0;
        if (++b < lens.size()) load();
      }
    }
    return true;
  };
  for (int i = 0; i < slots; ++i)
    if (!next_cta(0.0)) break;
  const double merge = ceil_div(std::max(max_len, 1), chunk) > 1 ? kMergeLaunchUs : 0.0;
  const double limit = cutoff - merge;
  double v = 0.0, t = 0.0;
  size_t rate_for = 0;   // running count the rate below was computed for
  double inv_rate = 0.0;
  while (count + running_last > 0) {
    if (count + running_last != rate_for) {
      rate_for = count + running_last;
      inv_rate = 1.0 / std::min(cta_bytes_per_us, hbm / static_cast<double>(rate_for));
    }
    if (t > limit) return t + merge;
    double nxt;
    if (count > 0 && (running_last == 0 || ring[head] <= last_front())) {
      nxt = ring[head];
      if (++head == ring.size()) head = 0;
      --count;
    } else {
      nxt = last_front();
      pop_last();
    }
    t += (nxt - v) * inv_rate;
    v = nxt;
    next_cta(v);
  }
  return t + merge;
}

// A lower bound of estimate_decode_us for the same arguments, in O(batch):
// the running CTAs never move more than the HBM bandwidth in total, nor more
// than their slots' ceilings, and no CTA finishes faster than its own ceiling.
double lower_bound_decode_us(const std::vector<int32_t>& lens, int64_t units, int64_t chunk,
                             int slots, int head_dim, int kv_elem_bytes, const CtaModel& cm,
                             int num_sms) {
  const double bytes_per_token = 2.0 * head_dim * kv_elem_bytes;
  const double hbm = kHbmBytesPerUs148 * num_sms / 148.0;
  const double overhead_bytes = cm.overhead_us * cm.bytes_per_us;
  double total = 0.0, largest = 0.0;
  int64_t max_splits = 1;
  for (const int32_t L : lens) {
    const int64_t n = std::max<int64_t>(1, ceil_div(L, chunk));
    max_splits = std::max(max_splits, n);
    total += static_cast<double>(units) * (static_cast<double>(L) * bytes_per_token +
                                           static_cast<double>(n) * overhead_bytes);
    largest = std::max(largest, static_cast<double>(std::min<int64_t>(chunk, L)) * bytes_per_token +
                                    overhead_bytes);
  }
  const double t = std::max({total / hbm, total / (static_cast<double>(slots) * cm.bytes_per_us),
                             largest / cm.bytes_per_us});
  return t + (max_splits > 1 ? kMergeLaunchUs : 0.0);
}
}  // namespace

int make_decode_plan(const int32_t* cache_seqlens_host, int batch, int num_q_heads,
                     int num_kv_heads, int head_dim, int page_size, int max_pages_per_seq,
                     int num_sms, int num_splits_override, int kv_elem_bytes, int kernel,
                     int q_len, DecodePlan* plan) {
  if (plan == nullptr || cache_seqlens_host == nullptr) return FA_ERR_INVALID_ARG;
  if (q_len < 1 || q_len > kTensorCoreMaxGroup) return FA_ERR_INVALID_ARG;
  if (kv_elem_bytes != 1 && kv_elem_bytes != 2) return FA_ERR_INVALID_ARG;
  if (kernel < kDecodeKernelAuto || kernel > kDecodeKernelTensorCores) return FA_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || num_q_heads < 1 || num_kv_heads < 1 ||
      max_pages_per_seq < 1 || num_sms < 1 || num_splits_override < 0)
    return FA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads != 0) return FA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return FA_ERR_UNSUPPORTED;
  if (page_size != 64) return FA_ERR_UNSUPPORTED;
  const int64_t capacity = static_cast<int64_t>(max_pages_per_seq) * page_size;
  if (capacity > (int64_t{1} << 30)) return FA_ERR_INVALID_ARG;

  DecodePlan pl;
  pl.batch = batch;
  pl.num_q_heads = num_q_heads;
  pl.num_kv_heads = num_kv_heads;
  pl.head_dim = head_dim;
  pl.page_size = page_size;
  pl.max_pages_per_seq = max_pages_per_seq;
  pl.num_sms = num_sms;
  pl.group = num_q_heads / num_kv_heads;
  pl.kv_elem_bytes = kv_elem_bytes;
  pl.q_len = q_len;
  const bool tc_ok = head_dim == 128 && q_len * pl.group <= kTensorCoreMaxGroup;
  if ((kernel == kDecodeKernelTensorCores || q_len > 1) && !tc_ok) return FA_ERR_UNSUPPORTED;
  if (q_len > 1 && kernel == kDecodeKernelCudaCores) return FA_ERR_UNSUPPORTED;
  // Tensor cores by default for an E4M3 cache (the CUDA-core loop spends an
  // integer widening and G FMAs on every byte) and for groups of 4 or more
  // (measured on B200: CUDA cores ahead at G = 1 and 2, tensor cores from 4).
  // Several query tokens per request (multi-token decode) only run on tensor cores.
  pl.tensor_cores = kernel == kDecodeKernelTensorCores || q_len > 1 ||
                    (kernel == kDecodeKernelAuto && tc_ok && (kv_elem_bytes == 1 || pl.group >= 4));
  if (pl.tensor_cores) {
    pl.heads_per_cta = pl.group;
  } else {
    for (int gc : {8, 4, 2, 1})
      if (pl.group % gc == 0) {
        pl.heads_per_cta = gc;
        break;
      }
  }
  pl.subgroups = pl.group / pl.heads_per_cta;
  if (static_cast<int64_t>(num_kv_heads) * pl.subgroups > 65535) return FA_ERR_UNSUPPORTED;

  pl.seqlens.assign(cache_seqlens_host, cache_seqlens_host + batch);
  int64_t total = 0;
  int max_len = 0;
  for (int b = 0; b < batch; ++b) {
    const int32_t L = pl.seqlens[b];
    // Cache-overflow check: a length the block table cannot address is an error.
    if (L < 0 || L > capacity) return FA_ERR_INVALID_ARG;
    // The chunk's own tokens are in the cache already.
    if (q_len > 1 && L < q_len) return FA_ERR_INVALID_ARG;
    total += L;
    max_len = std::max(max_len, static_cast<int>(L));
  }
  pl.max_seqlen = max_len;
  const int64_t units = static_cast<int64_t>(num_kv_heads) * pl.subgroups;   // CTAs per split

  int64_t chunk;
  if (num_splits_override > 0) {
    chunk = round_up(std::max<int64_t>(1, ceil_div(max_len, num_splits_override)), page_size);
  } else if (max_len <= kMinChunkTokens) {
    chunk = round_up(std::max(max_len, 1), page_size);
  } else {
    // Try split counts s (chunk = ceil(max_len / s) rounded to a page, at
    // least kMinChunkTokens keys) plus the many-small-items rule, and keep the
    // one the decode-time model estimates fastest (ties: fewer splits).
    const CtaModel cm = cta_model(pl.tensor_cores, kv_elem_bytes, q_len * pl.heads_per_cta);
    const int slots = num_sms * cm.ctas_per_sm;
    std::vector<int64_t> cands;
    for (int s : {1, 2, 3, 4, 5, 6, 8, 10, 12, 16, 20, 24, 32, 48, 64, 96, 128})
      cands.push_back(round_up(ceil_div(max_len, s), page_size));
    const int64_t target = ceil_div(total * units, static_cast<int64_t>(slots) * kItemsPerSlot);
    cands.push_back(round_up(target, page_size));
    // Simulate the candidates in increasing order of their lower bound and
    // skip any whose bound already exceeds the best estimate: the choice is
    // the exhaustive search's, at a fraction of the simulations (the many-CTA
    // candidates, the costly ones to simulate, have the highest bounds).
    for (int64_t& c : cands) c = std::max<int64_t>(c, kMinChunkTokens);
    std::sort(cands.begin(), cands.end());
    cands.erase(std::unique(cands.begin(), cands.end()), cands.end());   // one simulation per chunk
    std::vector<std::pair<double, int64_t>> order;
    for (const int64_t c : cands) {
      if (ceil_div(max_len, c) > kMaxSplits) continue;
      order.emplace_back(lower_bound_decode_us(pl.seqlens, units, c, slots, head_dim, kv_elem_bytes,
                                               cm, num_sms), c);
    }
    std::sort(order.begin(), order.end());
    // Candidates in increasing order of their lower bound; none whose bound
    // exceeds the best estimate can win (its estimate is at least its bound),
    // and a simulation stops once it passes the best estimate.
    double best_t = 0.0;
    chunk = 0;
    SimScratch scratch;
    for (const auto& [lb, c] : order) {
      if (chunk != 0 && lb > best_t * (1.0 + 1e-9)) break;
      const double cutoff = chunk == 0 ? std::numeric_limits<double>::infinity() : best_t * (1.0 + 1e-9);
      const double t = estimate_decode_us(pl.seqlens, units, c, slots, head_dim, kv_elem_bytes, cm, num_sms,
                                          max_len, cutoff, scratch);
      if (chunk == 0 || t < best_t * (1.0 - 1e-9) || (t <= best_t * (1.0 + 1e-9) && c > chunk)) {
        best_t = t;
        chunk = c;
      }
    }
  }
  if (max_len > 0 && ceil_div(max_len, chunk) > kMaxSplits)
    chunk = round_up(ceil_div(max_len, kMaxSplits), page_size);
  chunk = std::max<int64_t>(chunk, page_size);
  pl.chunk_tokens = static_cast<int>(chunk);
  pl.max_splits = static_cast<int>(std::max<int64_t>(1, ceil_div(max_len, chunk)));

  int64_t items = 0;
  for (int b = 0; b < batch; ++b) items += std::max<int64_t>(1, ceil_div(pl.seqlens[b], chunk));
  pl.num_work_items = static_cast<int>(items * units);

  if (pl.max_splits > 1) {
    const size_t rows = static_cast<size_t>(batch) * q_len * num_q_heads;
    pl.ws_o_offset = 0;
    pl.ws_lse_offset = align256(static_cast<size_t>(pl.max_splits) * rows * head_dim * 4);
    pl.workspace_bytes = align256(pl.ws_lse_offset + static_cast<size_t>(pl.max_splits) * rows * 4);
  } else {
    pl.workspace_bytes = 0;
  }
  *plan = std::move(pl);
  return FA_OK;
}

}  // namespace fa
