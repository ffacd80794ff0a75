// cfr_sched.cuh -- the ragged-batch split scheduler as a block-level device
// function, shared by the schedule kernel and by the tensor-core path's
// query-image kernel (which runs it in one extra block, saving a launch).
//
// From seq_lens alone, cuts every sequence into contiguous ranges of `chunk`
// pages, chunk = ceil(total pages / target_splits), so that splits carry about
// equal numbers of tokens whatever the length mix (the split-K decoding of the
// CMF page, "split-K flash-decoding so throughput holds at depth", sized here by
// the sequence lengths).  With a sink + recent window subset (window > 0) only
// the pages holding tokens of the subset are scheduled: the pages of the first
// `sink` tokens and those of the last `window` tokens, two page ranges when a
// gap separates them.  A sequence shorter than its number of query tokens (or
// empty, or longer than its page table) gets no split and sets
// CFR_DEVERR_SEQ_LEN.  Writes split_off[B+1], the (b, first page, end page)
// triple of every split, and (total splits, chunk).  Deterministic.
#pragma once

#include "cfr_common.cuh"

namespace cfr {

// arguments of one schedule (see schedule_block)
struct SchedArgs {
  const int32_t *seq_lens;
  int batch, P, max_pages, target, sink, window, nq;
  // tokens per schedule unit: splits are ranges of whole units (P, i.e. pages,
  // or a divisor of P that is a multiple of every kernel's tile, so that a
  // short sequence of long pages still spreads over many splits)
  int unit;
  int32_t *split_off;   // [batch + 1]
  int32_t *splits;      // [max_splits][3]
  int max_splits;
  int32_t *num_splits;  // [0] split count, [1] split length in pages
  uint32_t *item_ctr;   // the decode kernel's claim counter and finished-CTA count, or null
  uint32_t *err;
};

__device__ __forceinline__ long long block_sum_ll(long long v, long long *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  long long t = 0;
  if (threadIdx.x < 32) {
    t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (threadIdx.x == 0) red[32] = t;
  }
  __syncthreads();
  t = red[32];
  __syncthreads();
  return t;
}

// exclusive prefix sum over the block; *total receives the block sum
__device__ __forceinline__ int block_exclusive_scan(int v, int *red, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  if (threadIdx.x < 32) {
    int w = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0;
    int s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    red[threadIdx.x] = s - w;  // exclusive prefix of warp sums
    if (threadIdx.x == 31) red[32] = s;
  }
  __syncthreads();
  const int r = red[warp] + x - v;
  *total = red[32];
  __syncthreads();
  return r;
}

// units of P tokens (pages, or the schedule's smaller unit) of a sequence of n
// tokens; -1 when n is outside [min_len, max_pages * P]
__device__ __forceinline__ int valid_pages(int n, int P, int max_pages, int min_len) {
  if (n <= 0 || n < min_len || n > max_pages * P) return -1;
  return (n + P - 1) / P;
}

// Page ranges [0, *a_end) and [*b_begin, np) of a sequence of n tokens and np
// pages that hold the tokens taking part (the second range is empty when the
// first covers everything).
__device__ __forceinline__ void page_ranges(int n, int np, int P, int sink, int window, int *a_end,
                                            int *b_begin) {
  *a_end = np;
  *b_begin = np;
  if (window <= 0 || np <= 0 || static_cast<long long>(sink) + window >= n) return;
  const int ps = (sink + P - 1) / P;       // pages of the sink tokens
  const int pw = (n - window) / P;         // first page of the window
  if (pw <= ps) return;
  *a_end = ps;
  *b_begin = pw;
}

// The whole schedule, computed by every thread of one CTA (any size that is a
// multiple of 32, up to 1024 threads).
__device__ __forceinline__ void schedule_block(const SchedArgs &a) {
  const int32_t *__restrict__ seq_lens = a.seq_lens;
  const int batch = a.batch, max_pages = a.max_pages, target = a.target;
  // units of U tokens: a sequence of n tokens is valid when 1 <= n <= max_pages * P
  // (and n >= nq), and spans ceil(n / U) units
  const int U = a.unit, max_units = static_cast<int>(static_cast<long long>(max_pages) * a.P / U);
  const int sink = a.sink, window = a.window, nq = a.nq, max_splits = a.max_splits;
  int32_t *__restrict__ split_off = a.split_off;
  int32_t *__restrict__ splits = a.splits;
  int32_t *__restrict__ num_splits = a.num_splits;
  uint32_t *__restrict__ item_ctr = a.item_ctr;
  uint32_t *err = a.err;
  // the decode kernel's work-item claim counter and finished-CTA count start at 0
  if (threadIdx.x == 0 && item_ctr) {
    item_ctr[0] = 0u;
    item_ctr[1] = 0u;
  }
  __shared__ long long red_ll[33];
  __shared__ int red_i[33];
  long long local = 0;
  for (int b = threadIdx.x; b < batch; b += blockDim.x) {
    const int n = seq_lens[b];
    const int np = valid_pages(n, U, max_units, nq);
    if (np < 0) {
      set_err(err, CFR_DEVERR_SEQ_LEN);
    } else {
      int a_end, b_begin;
      page_ranges(n, np, U, sink, window, &a_end, &b_begin);
      local += a_end + (np - b_begin);
    }
  }
  const long long total = block_sum_ll(local, red_ll);
  const long long tgt = target > 0 ? target : 1;
  int chunk = static_cast<int>((total + tgt - 1) / tgt);
  if (chunk < 1) chunk = 1;

  int running = 0;
  bool overflow = false;
  for (int base = 0; base < batch; base += blockDim.x) {
    const int b = base + threadIdx.x;
    const int n = b < batch ? seq_lens[b] : 0;
    int np = b < batch ? valid_pages(n, U, max_units, nq) : -1;
    if (np < 0) np = 0;
    int a_end, b_begin;
    page_ranges(n, np, U, sink, window, &a_end, &b_begin);
    const int cnt_a = (a_end + chunk - 1) / chunk;
    const int cnt = cnt_a + (np - b_begin + chunk - 1) / chunk;
    int tot = 0;
    const int excl = block_exclusive_scan(cnt, red_i, &tot) + running;
    if (b < batch) {
      split_off[b] = excl < max_splits ? excl : max_splits;
      for (int s = 0; s < cnt; ++s) {
        const int idx = excl + s;
        if (idx >= max_splits) {
          overflow = true;
          break;
        }
        // splits of the first range, then of the second
        const int r0 = s < cnt_a ? 0 : b_begin, r1 = s < cnt_a ? a_end : np;
        const int pb = r0 + (s < cnt_a ? s : s - cnt_a) * chunk;
        const int pe = pb + chunk < r1 ? pb + chunk : r1;
        splits[3 * idx + 0] = b;
        splits[3 * idx + 1] = pb;
        splits[3 * idx + 2] = pe;
      }
    }
    running += tot;
  }
  if (overflow) set_err(err, CFR_DEVERR_SEQ_LEN);
  if (threadIdx.x == 0) {
    const int S = running < max_splits ? running : max_splits;
    split_off[batch] = S;
    num_splits[0] = S;
    num_splits[1] = chunk;
  }
}

}  // namespace cfr
