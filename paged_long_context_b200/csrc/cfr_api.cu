// cfr_api.cu -- the C ABI: host-side argument checks, workspace layout, kernel
// selection and launches.  Nothing here allocates memory or synchronises.
#include <climits>
#include <cstring>

#include "cfr_common.cuh"
#include "cfr_sched.cuh"

namespace cfr {

void launch_schedule(const int32_t *seq_lens, int batch, int P, int max_pages, int target,
                     int sink, int window, int nq, int unit, int32_t *split_off, int32_t *splits,
                     int max_splits, int32_t *num_splits, uint32_t *item_ctr, uint32_t *err,
                     cudaStream_t stream);
void launch_merge(const float *part_acc, const float *part_m, const float *part_l,
                  const int32_t *split_off, int batch, int Hq, int D, int max_splits, float *out,
                  float *lse, uint32_t *err, cudaStream_t stream);
void launch_gather(const DecodeParams &p, int b, int g, int n_tokens, void *k_out, void *v_out,
                   long long pitch, cudaStream_t stream);
cudaError_t launch_decode_cc(const DecodeParams &p, int grid, cudaStream_t stream);
int cc_stages(int D, int gt, int pitch, size_t smem_limit);
int cc_group_tile(int gmax);
cudaError_t launch_decode_tc(const DecodeParams &p, int grid, cudaStream_t stream,
                             const SchedArgs *sched);
bool tc_supported(const DecodeParams &p, bool page_fmt_given);
cudaError_t launch_decode_f32(const DecodeParams &p, int grid, cudaStream_t stream);
bool f32_supported(const DecodeParams &p, bool page_fmt_given);

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int sms = 0;
  size_t smem_optin = 0;
};

// SM count and opt-in shared memory of the current device (cached per device).
bool device_info(DeviceInfo *out) {
  static DeviceInfo cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
  if (dev < kMaxDevices && cache[dev].sms > 0) {
    *out = cache[dev];
    return true;
  }
  DeviceInfo di;
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
  di.sms = v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return false;
  di.smem_optin = static_cast<size_t>(v);
  if (dev < kMaxDevices) cache[dev] = di;
  *out = di;
  return true;
}

bool mul_ok(size_t a, size_t b, size_t *r) {
  if (a != 0 && b > SIZE_MAX / a) return false;
  *r = a * b;
  return true;
}

bool add_ok(size_t a, size_t b, size_t *r) {
  if (b > SIZE_MAX - a) return false;
  *r = a + b;
  return true;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Target number of splits over the whole batch: about `per_sm` work items
// (split x kv head) per SM, so that a persistent grid of one CTA per SM gets
// an even share.  Every item pays one pipeline drain at its end and one more
// partial for the merge.
//  - The tcgen05 path over bf16-only pools, and over uniform int8 / int4 pools
//    in its int8-MMA variant, balances at run time (its CTAs claim items from a
//    counter), so it takes the fewest, longest items: 4 per SM measured faster
//    than 8 or 16, and 2 per SM for sink + window subsets and for groups of
//    more than 8 rows (the 32-column variants), whose tiles cost more.
//  - Other uniform caches are shared out in a fixed pattern: 8 per SM.
//  - A cache of mixed storage formats has items of unequal cost (a page of
//    int4 codes is a quarter of the bytes of a bf16 page, but takes longer to
//    expand), so its fixed share is cut finer: 16 per SM.
constexpr int kItemsPerSmClaimed = 4, kItemsPerSmClaimedLong = 2, kItemsPerSm = 8, kItemsPerSmMixed = 16;

// true when a decode over these pools expands quantised codes on chip
bool quantised_pools(const DecodeParams &p, bool page_fmt_given) {
  if (page_fmt_given)
    return p.k_pool[CFR_FMT_I8] || p.k_pool[CFR_FMT_I4] || p.k_pool[CFR_FMT_FP8];
  return is_quantised(p.uniform_fmt);
}

int target_splits(int sms, int hkv, int per_sm = kItemsPerSmMixed) {
  const long long items = static_cast<long long>(per_sm) * sms;
  long long t = (items + hkv - 1) / hkv;
  if (t < 1) t = 1;
  if (t > (1 << 20)) t = 1 << 20;
  return static_cast<int>(t);
}

// The decode schedule's unit (tokens): the page, or 128 tokens (every kernel's
// tile divides 128) when pages are a larger multiple of 128 and the page tables
// hold fewer pages than the GPU has SMs, so that a short batch of long pages
// still spreads over the SMs.  (Splitting pages of larger batches measured
// slower: the mixed-format cache took 27 % longer.)
int schedule_unit(int page_tokens, int batch, int max_pages, int sms) {
  const bool few_pages = static_cast<long long>(batch) * max_pages < sms;
  return page_tokens > 128 && page_tokens % 128 == 0 && few_pages ? 128 : page_tokens;
}

// workspace header: [0] split count, [1] split length in schedule units; at byte
// kItemCtrOffset the decode kernel's work-item claim counter and finished-CTA count
constexpr size_t kItemCtrOffset = 64;

struct WsLayout {
  size_t header, split_off, splits, part_m, part_l, part_acc, qimg, qscale, total;
  int max_splits;
};

bool ws_layout(int batch, int hq, int hkv, int d, int max_pages, int page_tokens, int unit,
               int target, WsLayout *w) {
  // ceil(len / chunk) summed over at most two unit ranges per sequence
  long long ms = static_cast<long long>(target) + 2LL * batch;
  const long long cap = static_cast<long long>(batch) * max_pages * (page_tokens / unit);
  if (cap < ms) ms = cap;
  if (ms < 1) ms = 1;
  if (ms > INT_MAX / 4) return false;
  w->max_splits = static_cast<int>(ms);
  size_t o = 0, t = 0;
  w->header = 0;
  o = 256;
  w->split_off = o;
  if (!mul_ok(static_cast<size_t>(batch) + 1, 4, &t) || !add_ok(o, t, &o)) return false;
  o = align_up(o, 256);
  w->splits = o;
  if (!mul_ok(static_cast<size_t>(ms), 12, &t) || !add_ok(o, t, &o)) return false;
  o = align_up(o, 256);
  size_t mh = 0;
  if (!mul_ok(static_cast<size_t>(ms), static_cast<size_t>(hq), &mh)) return false;
  w->part_m = o;
  if (!mul_ok(mh, 4, &t) || !add_ok(o, t, &o)) return false;
  o = align_up(o, 256);
  w->part_l = o;
  if (!add_ok(o, t, &o)) return false;
  o = align_up(o, 256);
  w->part_acc = o;
  if (!mul_ok(mh, static_cast<size_t>(d) * 4, &t) || !add_ok(o, t, &o)) return false;
  // query operand images of the tensor-core decode, one per (sequence, row
  // group); a kv head's rows make at most count / kMaxGroup + 1 groups
  size_t groups = 0;
  const size_t ngmax = static_cast<size_t>(hkv) + (static_cast<size_t>(hq) + kMaxGroup - 1) / kMaxGroup;
  if (!mul_ok(static_cast<size_t>(batch), ngmax, &groups)) return false;
  o = align_up(o, 1024);
  w->qimg = o;
  if (!mul_ok(groups, static_cast<size_t>(kQImgBytes), &t) || !add_ok(o, t, &o)) return false;
  o = align_up(o, 256);
  w->qscale = o;
  if (!mul_ok(groups, 16, &t) || !add_ok(o, t, &o)) return false;
  w->total = align_up(o, 256);
  return true;
}

bool valid_fmt(int f) { return f >= 0 && f < kFmtCount; }

// Checks of the pool description shared by decode, gather and path queries.
cfr_status check_pool(const cfr_kv_pool *kv) {
  if (!kv) return CFR_ERR_INVALID_ARG;
  if (kv->num_kv_heads <= 0 || kv->head_dim <= 0 || kv->page_tokens <= 0) return CFR_ERR_INVALID_ARG;
  if (kv->head_dim != 64 && kv->head_dim != 128) return CFR_ERR_UNSUPPORTED;
  if (kv->page_tokens < 8) return CFR_ERR_UNSUPPORTED;
  bool any = false;
  for (int f = 0; f < kFmtCount; ++f) {
    const bool has = kv->k_pool[f] || kv->v_pool[f];
    if (!has) continue;
    if (!kv->k_pool[f] || !kv->v_pool[f]) return CFR_ERR_INVALID_ARG;
    if (!aligned(kv->k_pool[f], 16) || !aligned(kv->v_pool[f], 16)) return CFR_ERR_INVALID_ARG;
    if (kv->pool_pages[f] < 0) return CFR_ERR_INVALID_ARG;
    if (is_quantised(f) && kv->pool_pages[f] > 0) {
      if (!kv->scales[f] || !aligned(kv->scales[f], 8)) return CFR_ERR_INVALID_ARG;
    }
    // byte offsets of the last row must fit in 64 bits
    size_t t = 0;
    if (!mul_ok(static_cast<size_t>(kv->pool_pages[f]), static_cast<size_t>(kv->num_kv_heads), &t) ||
        !mul_ok(t, static_cast<size_t>(kv->page_tokens), &t) ||
        !mul_ok(t, static_cast<size_t>(row_bytes(f, kv->head_dim)), &t) || t > (size_t)LLONG_MAX)
      return CFR_ERR_OVERFLOW;
    any = true;
  }
  if (!any) return CFR_ERR_INVALID_ARG;
  return CFR_OK;
}

// Query-row groups per kv head, from a host head map (or the contiguous rule).
// With nq queries per sequence the rows are vh = qi * hq + h (qi < nq); row vh
// belongs to the kv head of query head h.
cfr_status build_groups(int hq, int hkv, const int32_t *head_map, DecodeParams *p, int nq = 1) {
  if (hq <= 0 || hkv <= 0 || hkv > kMaxQHeads || nq <= 0) return CFR_ERR_UNSUPPORTED;
  if (static_cast<long long>(hq) * nq > kMaxQHeads) return CFR_ERR_UNSUPPORTED;
  if (!head_map && hq % hkv != 0) return CFR_ERR_INVALID_ARG;
  const int rows = hq * nq;
  int count[kMaxQHeads + 1];
  std::memset(count, 0, sizeof(count));
  for (int h = 0; h < hq; ++h) {
    const int g = head_map ? head_map[h] : h / (hq / hkv);
    if (g < 0 || g >= hkv) return CFR_ERR_INVALID_ARG;
    count[g] += nq;
  }
  // the rows of each kv head in order; a kv head with more than kMaxGroup rows
  // (MQA, wide GQA, many query tokens) is cut into ceil(count / kMaxGroup)
  // groups of near-equal size
  int start[kMaxQHeads + 1];
  int off = 0;
  for (int g = 0; g < hkv; ++g) {
    start[g] = off;
    off += count[g];
  }
  int gmax = 0, ng = 0, nblk0 = -1;
  bool uniform = true;  // every kv head cut into the same number of groups
  for (int g = 0; g < hkv; ++g) {
    const int nblk = count[g] <= kMaxGroup ? 1 : (count[g] + kMaxGroup - 1) / kMaxGroup;
    if (nblk0 < 0) nblk0 = nblk;
    uniform = uniform && nblk == nblk0;
    for (int j = 0; j < nblk; ++j) {
      const int lo = start[g] + count[g] * j / nblk, hi = start[g] + count[g] * (j + 1) / nblk;
      if (ng >= kMaxGroups) return CFR_ERR_UNSUPPORTED;
      p->grp_off[ng] = static_cast<int16_t>(lo);
      p->grp_kv[ng] = static_cast<int16_t>(g);
      if (hi - lo > gmax) gmax = hi - lo;
      ++ng;
    }
  }
  p->grp_off[ng] = static_cast<int16_t>(off);
  p->ngroups = ng;
  p->gsub = uniform && nblk0 > 1 ? nblk0 : 1;
  int fill[kMaxQHeads];
  for (int g = 0; g < hkv; ++g) fill[g] = start[g];
  for (int vh = 0; vh < rows; ++vh) {
    const int h = vh % hq;
    const int g = head_map ? head_map[h] : h / (hq / hkv);
    p->grp_heads[fill[g]++] = static_cast<int16_t>(vh);
  }
  p->gmax = gmax < 1 ? 1 : gmax;
  p->nq = nq;
  p->hq_real = hq;
  return CFR_OK;
}

void fill_pool(const cfr_kv_pool *kv, DecodeParams *p) {
  for (int f = 0; f < kFmtCount; ++f) {
    p->k_pool[f] = static_cast<const uint8_t *>(kv->k_pool[f]);
    p->v_pool[f] = static_cast<const uint8_t *>(kv->v_pool[f]);
    p->scales[f] = kv->scales[f];
    p->pool_pages[f] = kv->k_pool[f] ? kv->pool_pages[f] : 0;
  }
  p->Hkv = kv->num_kv_heads;
  p->D = kv->head_dim;
  p->P = kv->page_tokens;
}

int widest_row(const cfr_kv_pool *kv, const uint8_t *page_fmt, int uniform_fmt) {
  if (!page_fmt) return row_bytes(uniform_fmt, kv->head_dim);
  int w = 0;
  for (int f = 0; f < kFmtCount; ++f)
    if (kv->k_pool[f] && row_bytes(f, kv->head_dim) > w) w = row_bytes(f, kv->head_dim);
  return w;
}

cfr_status common_checks(int32_t q_fmt, const cfr_kv_pool *kv, int32_t max_pages,
                         const uint8_t *page_fmt, int32_t uniform_fmt) {
  cfr_status st = check_pool(kv);
  if (st != CFR_OK) return st;
  if (q_fmt != CFR_FMT_F32 && q_fmt != CFR_FMT_BF16) return CFR_ERR_INVALID_ARG;
  if (max_pages <= 0) return CFR_ERR_INVALID_ARG;
  if (static_cast<long long>(max_pages) * kv->page_tokens > INT_MAX) return CFR_ERR_OVERFLOW;
  if (!page_fmt) {
    if (!valid_fmt(uniform_fmt)) return CFR_ERR_INVALID_ARG;
    if (!kv->k_pool[uniform_fmt]) return CFR_ERR_INVALID_ARG;
  }
  return CFR_OK;
}

}  // namespace
}  // namespace cfr

using namespace cfr;

extern "C" {

size_t cfr_paged_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t max_pages, int32_t page_tokens) {
  if (batch <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_pages <= 0 ||
      page_tokens <= 0)
    return 0;
  DeviceInfo di;
  if (!device_info(&di)) return 0;
  WsLayout w;
  if (!ws_layout(batch, num_q_heads, num_kv_heads, head_dim, max_pages, page_tokens,
                 schedule_unit(page_tokens, batch, max_pages, di.sms),
                 target_splits(di.sms, num_kv_heads), &w))
    return 0;
  return w.total;
}

int32_t cfr_paged_decode_path(int32_t q_fmt, const cfr_kv_pool *kv, int32_t max_pages,
                              const uint8_t *page_fmt, int32_t uniform_fmt, int32_t num_q_heads,
                              const int32_t *head_map) {
  if (common_checks(q_fmt, kv, max_pages, page_fmt, uniform_fmt) != CFR_OK) return 0;
  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  if (build_groups(num_q_heads, kv->num_kv_heads, head_map, &p) != CFR_OK) return 0;
  fill_pool(kv, &p);
  p.q_fmt = q_fmt;
  p.uniform_fmt = uniform_fmt;
  p.Hq = num_q_heads;
  p.max_pages = max_pages;
  if (tc_supported(p, page_fmt != nullptr)) return 2;
  if (f32_supported(p, page_fmt != nullptr)) return 3;
  return 1;
}

cfr_status cfr_paged_decode(const void *q, int32_t q_fmt, const cfr_kv_pool *kv,
                            const int32_t *page_table, int32_t max_pages,
                            const int32_t *seq_lens, int32_t batch, const uint8_t *page_fmt,
                            int32_t uniform_fmt, int32_t num_q_heads, const int32_t *head_map,
                            const float *alibi_slopes, float softmax_scale, float *out,
                            float *lse, void *workspace, size_t workspace_bytes,
                            uint32_t *err_word, void *stream) {
  return cfr_paged_decode_phases(q, q_fmt, kv, page_table, max_pages, seq_lens, batch, page_fmt,
                                 uniform_fmt, num_q_heads, head_map, alibi_slopes, softmax_scale,
                                 out, lse, workspace, workspace_bytes, err_word, stream,
                                 CFR_PHASE_ALL);
}

}  // extern "C"

namespace cfr {
namespace {

// Every decode entry point: checks, schedule, decode and merge launches.
// window > 0 restricts each softmax to the first `sink` and last `window` tokens.
cfr_status decode_impl(const void *q, int32_t q_fmt, const cfr_kv_pool *kv,
                       const int32_t *page_table, int32_t max_pages, const int32_t *seq_lens,
                       int32_t batch, const uint8_t *page_fmt, int32_t uniform_fmt,
                       int32_t num_q_heads, const int32_t *head_map, const float *alibi_slopes,
                       float softmax_scale, float *out, float *lse, void *workspace,
                       size_t workspace_bytes, uint32_t *err_word, void *stream, uint32_t phases,
                       int32_t sink, int32_t window, int32_t nq) {
  if (phases == 0 || (phases & ~CFR_PHASE_ALL)) return CFR_ERR_INVALID_ARG;
  cfr_status st = common_checks(q_fmt, kv, max_pages, page_fmt, uniform_fmt);
  if (st != CFR_OK) return st;
  if (!q || !page_table || !seq_lens || !out || batch <= 0) return CFR_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16)) return CFR_ERR_INVALID_ARG;
  if (!(softmax_scale >= 0.f) || softmax_scale == INFINITY) return CFR_ERR_INVALID_ARG;
  if (static_cast<long long>(batch) * max_pages > INT_MAX) return CFR_ERR_OVERFLOW;

  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  st = build_groups(num_q_heads, kv->num_kv_heads, head_map, &p, nq);
  if (st != CFR_OK) return st;
  fill_pool(kv, &p);
  const int rows = num_q_heads * nq;  // query rows per sequence

  DeviceInfo di;
  if (!device_info(&di)) return CFR_ERR_CUDA;
  p.q = q;
  p.q_fmt = q_fmt;
  p.page_fmt = page_fmt;
  p.uniform_fmt = uniform_fmt;
  const bool use_tc = tc_supported(p, page_fmt != nullptr);
  const bool use_f32 = !use_tc && f32_supported(p, page_fmt != nullptr);
  // the tcgen05 path claims its items at run time over bf16 pools and over
  // uniform int8 / int4 pools of up to 4 rows per group (the int8-MMA variant)
  const bool claimed =
      use_tc && (!quantised_pools(p, page_fmt != nullptr) ||
                 (!page_fmt && p.gmax <= 4 && kv->head_dim == 128 &&
                  (uniform_fmt == CFR_FMT_I8 || uniform_fmt == CFR_FMT_I4)));
  const int per_sm = claimed ? ((window > 0 || p.gmax > 8) ? kItemsPerSmClaimedLong : kItemsPerSmClaimed)
                     : page_fmt ? kItemsPerSmMixed : kItemsPerSm;
  const int target = target_splits(di.sms, p.ngroups, per_sm);
  WsLayout w;
  const int unit = schedule_unit(kv->page_tokens, batch, max_pages, di.sms);
  if (!ws_layout(batch, rows, kv->num_kv_heads, kv->head_dim, max_pages, kv->page_tokens, unit,
                 target, &w))
    return CFR_ERR_OVERFLOW;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.total) return CFR_ERR_WORKSPACE;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int32_t *num_splits = reinterpret_cast<int32_t *>(ws + w.header);
  uint32_t *item_ctr = reinterpret_cast<uint32_t *>(ws + w.header + kItemCtrOffset);
  int32_t *split_off = reinterpret_cast<int32_t *>(ws + w.split_off);
  int32_t *splits = reinterpret_cast<int32_t *>(ws + w.splits);
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.slopes = alibi_slopes;
  p.part_acc = reinterpret_cast<float *>(ws + w.part_acc);
  p.part_m = reinterpret_cast<float *>(ws + w.part_m);
  p.part_l = reinterpret_cast<float *>(ws + w.part_l);
  p.splits = splits;
  p.num_splits = num_splits;
  p.max_splits = w.max_splits;
  p.split_unit = unit;
  p.max_units = static_cast<int>(static_cast<long long>(max_pages) * kv->page_tokens / p.split_unit);
  // mixed-format caches with quantised pages share their items out in a fixed
  // pattern (no claim counter); see tc_claimed_items
  p.item_ctr = (page_fmt && quantised_pools(p, true)) ? nullptr : item_ctr;
  p.qimg = ws + w.qimg;
  p.qscale = reinterpret_cast<float *>(ws + w.qscale);
  p.err = err_word;
  p.batch = batch;
  p.max_pages = max_pages;
  p.Hq = rows;
  const float sigma = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf(static_cast<float>(kv->head_dim));
  p.sigma_log2e = sigma * kLog2e;
  p.sink = sink;
  p.window = window;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!use_tc && !use_f32) {
    p.pitch = widest_row(kv, page_fmt, uniform_fmt);
    p.stages = cc_stages(p.D, cc_group_tile(p.gmax), p.pitch, di.smem_optin);
    if (p.stages < 2) return CFR_ERR_UNSUPPORTED;
  }
  const SchedArgs sched{seq_lens, batch, kv->page_tokens, max_pages, target, sink, window, nq,
                        p.split_unit, split_off, splits, w.max_splits, num_splits, item_ctr,
                        err_word};
  // the tensor-core path runs a call's schedule inside its own first launch
  const bool sched_in_decode = use_tc && (phases & CFR_PHASE_SCHEDULE) && (phases & CFR_PHASE_DECODE);
  if ((phases & CFR_PHASE_SCHEDULE) && !sched_in_decode) {
    launch_schedule(seq_lens, batch, kv->page_tokens, max_pages, target, sink, window, nq,
                    p.split_unit, split_off, splits, w.max_splits, num_splits, item_ctr, err_word, s);
    if (cudaGetLastError() != cudaSuccess) return CFR_ERR_CUDA;
  }
  if (phases & CFR_PHASE_DECODE) {
    const cudaError_t e = use_tc    ? launch_decode_tc(p, di.sms, s, sched_in_decode ? &sched : nullptr)
                          : use_f32 ? launch_decode_f32(p, di.sms, s)
                                    : launch_decode_cc(p, di.sms, s);
    if (e != cudaSuccess) return CFR_ERR_CUDA;
  }
  if (phases & CFR_PHASE_MERGE) {
    launch_merge(p.part_acc, p.part_m, p.part_l, split_off, batch, rows, kv->head_dim,
                 w.max_splits, out, lse, err_word, s);
    if (cudaGetLastError() != cudaSuccess) return CFR_ERR_CUDA;
  }
  return CFR_OK;
}

}  // namespace
}  // namespace cfr

extern "C" {

cfr_status cfr_paged_decode_phases(const void *q, int32_t q_fmt, const cfr_kv_pool *kv,
                                   const int32_t *page_table, int32_t max_pages,
                                   const int32_t *seq_lens, int32_t batch,
                                   const uint8_t *page_fmt, int32_t uniform_fmt,
                                   int32_t num_q_heads, const int32_t *head_map,
                                   const float *alibi_slopes, float softmax_scale, float *out,
                                   float *lse, void *workspace, size_t workspace_bytes,
                                   uint32_t *err_word, void *stream, uint32_t phases) {
  return decode_impl(q, q_fmt, kv, page_table, max_pages, seq_lens, batch, page_fmt, uniform_fmt,
                     num_q_heads, head_map, alibi_slopes, softmax_scale, out, lse, workspace,
                     workspace_bytes, err_word, stream, phases, 0, 0, 1);
}

cfr_status cfr_paged_decode_sink_window(const void *q, int32_t q_fmt, const cfr_kv_pool *kv,
                                        const int32_t *page_table, int32_t max_pages,
                                        const int32_t *seq_lens, int32_t batch,
                                        const uint8_t *page_fmt, int32_t uniform_fmt,
                                        int32_t num_q_heads, const int32_t *head_map,
                                        const float *alibi_slopes, float softmax_scale,
                                        float *out, float *lse, void *workspace,
                                        size_t workspace_bytes, uint32_t *err_word, void *stream,
                                        int32_t sink_tokens, int32_t window_tokens,
                                        uint32_t phases) {
  if (sink_tokens < 0 || window_tokens < 1) return CFR_ERR_INVALID_ARG;
  return decode_impl(q, q_fmt, kv, page_table, max_pages, seq_lens, batch, page_fmt, uniform_fmt,
                     num_q_heads, head_map, alibi_slopes, softmax_scale, out, lse, workspace,
                     workspace_bytes, err_word, stream, phases, sink_tokens, window_tokens, 1);
}

cfr_status cfr_paged_decode_multi(const void *q, int32_t q_fmt, const cfr_kv_pool *kv,
                                  const int32_t *page_table, int32_t max_pages,
                                  const int32_t *seq_lens, int32_t batch, const uint8_t *page_fmt,
                                  int32_t uniform_fmt, int32_t num_q_heads, int32_t num_queries,
                                  const int32_t *head_map, const float *alibi_slopes,
                                  float softmax_scale, float *out, float *lse, void *workspace,
                                  size_t workspace_bytes, uint32_t *err_word, void *stream,
                                  uint32_t phases) {
  if (num_queries < 1 || num_queries > 16) return num_queries < 1 ? CFR_ERR_INVALID_ARG
                                                                 : CFR_ERR_UNSUPPORTED;
  return decode_impl(q, q_fmt, kv, page_table, max_pages, seq_lens, batch, page_fmt, uniform_fmt,
                     num_q_heads, head_map, alibi_slopes, softmax_scale, out, lse, workspace,
                     workspace_bytes, err_word, stream, phases, 0, 0, num_queries);
}

cfr_status cfr_merge_partials(const float *part_acc, const float *part_m, const float *part_l,
                              const int32_t *split_off, int32_t batch, int32_t num_q_heads,
                              int32_t head_dim, float *out, float *lse, void *stream) {
  if (!part_acc || !part_m || !part_l || !split_off || !out) return CFR_ERR_INVALID_ARG;
  if (batch <= 0 || num_q_heads <= 0) return CFR_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return CFR_ERR_UNSUPPORTED;
  if (!aligned(part_acc, 16) || !aligned(out, 16)) return CFR_ERR_INVALID_ARG;
  if (static_cast<long long>(batch) * num_q_heads > INT_MAX) return CFR_ERR_OVERFLOW;
  launch_merge(part_acc, part_m, part_l, split_off, batch, num_q_heads, head_dim, INT_MAX, out,
               lse, nullptr, static_cast<cudaStream_t>(stream));
  return cudaGetLastError() == cudaSuccess ? CFR_OK : CFR_ERR_CUDA;
}

cfr_status cfr_schedule_splits(const int32_t *seq_lens, int32_t batch, int32_t page_tokens,
                               int32_t max_pages, int32_t target_splits, int32_t *split_off,
                               int32_t *splits, int32_t max_splits, int32_t *num_splits,
                               uint32_t *err_word, void *stream) {
  if (!seq_lens || !split_off || !splits || !num_splits) return CFR_ERR_INVALID_ARG;
  if (batch <= 0 || page_tokens <= 0 || max_pages <= 0 || target_splits <= 0 || max_splits <= 0)
    return CFR_ERR_INVALID_ARG;
  if (static_cast<long long>(max_pages) * page_tokens > INT_MAX) return CFR_ERR_OVERFLOW;
  // (in pages: the schedule unit of this entry point is the page)
  launch_schedule(seq_lens, batch, page_tokens, max_pages, target_splits, 0, 0, 1, page_tokens,
                  split_off, splits, max_splits, num_splits, nullptr, err_word,
                  static_cast<cudaStream_t>(stream));
  return cudaGetLastError() == cudaSuccess ? CFR_OK : CFR_ERR_CUDA;
}

cfr_status cfr_gather_pages(const cfr_kv_pool *kv, const int32_t *page_table,
                            const uint8_t *page_fmt, int32_t uniform_fmt, int32_t batch,
                            int32_t max_pages, int32_t b, int32_t kv_head, int32_t n_tokens,
                            void *k_raw_out,
                            void *v_raw_out, int64_t out_row_pitch, uint32_t *err_word,
                            void *stream) {
  cfr_status st = common_checks(CFR_FMT_F32, kv, max_pages, page_fmt, uniform_fmt);
  if (st != CFR_OK) return st;
  if (!page_table || !k_raw_out || !v_raw_out) return CFR_ERR_INVALID_ARG;
  if (batch <= 0 || b < 0 || b >= batch || kv_head < 0 || kv_head >= kv->num_kv_heads || n_tokens < 0) return CFR_ERR_INVALID_ARG;
  if (static_cast<long long>(n_tokens) > static_cast<long long>(max_pages) * kv->page_tokens)
    return CFR_ERR_INVALID_ARG;
  if (static_cast<long long>(batch) * max_pages > INT_MAX) return CFR_ERR_OVERFLOW;
  if (out_row_pitch % 16 != 0 || out_row_pitch < widest_row(kv, page_fmt, uniform_fmt))
    return CFR_ERR_INVALID_ARG;
  if (!aligned(k_raw_out, 16) || !aligned(v_raw_out, 16)) return CFR_ERR_INVALID_ARG;
  if (n_tokens == 0) return CFR_OK;
  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  fill_pool(kv, &p);
  p.page_table = page_table;
  p.page_fmt = page_fmt;
  p.uniform_fmt = uniform_fmt;
  p.max_pages = max_pages;
  p.err = err_word;
  launch_gather(p, b, kv_head, n_tokens, k_raw_out, v_raw_out, out_row_pitch,
                static_cast<cudaStream_t>(stream));
  return cudaGetLastError() == cudaSuccess ? CFR_OK : CFR_ERR_CUDA;
}

const char *cfr_status_str(cfr_status status) {
  switch (status) {
    case CFR_OK: return "ok";
    case CFR_ERR_INVALID_ARG: return "invalid argument";
    case CFR_ERR_UNSUPPORTED: return "unsupported configuration";
    case CFR_ERR_OVERFLOW: return "size overflow";
    case CFR_ERR_PAGE_INDEX: return "page index out of range";
    case CFR_ERR_CUDA: return "CUDA error";
    case CFR_ERR_TIMEOUT: return "device wait timed out";
    case CFR_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

}  // extern "C"
