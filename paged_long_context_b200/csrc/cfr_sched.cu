// cfr_sched.cu -- ragged-batch split scheduler (one CTA).
//
// From seq_lens alone, cuts every sequence into contiguous ranges of `chunk`
// pages, chunk = ceil(total pages / target_splits), so that splits carry about
// equal numbers of tokens whatever the length mix (the split-K decoding of the
// CMF page, "split-K flash-decoding so throughput holds at depth", sized here by
// the sequence lengths).  Writes split_off[B+1], the (b, first page, end page)
// triple of every split, and (total splits, chunk).  Deterministic.
#include "cfr_common.cuh"

namespace cfr {

constexpr int kSchedThreads = 1024;

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

__device__ __forceinline__ int valid_pages(int n, int P, int max_pages) {
  if (n <= 0 || n > max_pages * P) return -1;
  return (n + P - 1) / P;
}

__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(
    const int32_t *__restrict__ seq_lens, int batch, int P, int max_pages, int target,
    int32_t *__restrict__ split_off, int32_t *__restrict__ splits, int max_splits,
    int32_t *__restrict__ num_splits, uint32_t *err) {
  griddep_launch_dependents();
  __shared__ long long red_ll[33];
  __shared__ int red_i[33];
  long long local = 0;
  for (int b = threadIdx.x; b < batch; b += blockDim.x) {
    const int np = valid_pages(seq_lens[b], P, max_pages);
    if (np < 0) set_err(err, CFR_DEVERR_SEQ_LEN);
    else local += np;
  }
  const long long total = block_sum_ll(local, red_ll);
  const long long tgt = target > 0 ? target : 1;
  int chunk = static_cast<int>((total + tgt - 1) / tgt);
  if (chunk < 1) chunk = 1;

  int running = 0;
  bool overflow = false;
  for (int base = 0; base < batch; base += blockDim.x) {
    const int b = base + threadIdx.x;
    int np = b < batch ? valid_pages(seq_lens[b], P, max_pages) : -1;
    if (np < 0) np = 0;
    const int cnt = (np + chunk - 1) / chunk;
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
        const int pb = s * chunk;
        const int pe = pb + chunk < np ? pb + chunk : np;
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

void launch_schedule(const int32_t *seq_lens, int batch, int P, int max_pages, int target,
                     int32_t *split_off, int32_t *splits, int max_splits, int32_t *num_splits,
                     uint32_t *err, cudaStream_t stream) {
  schedule_kernel<<<1, kSchedThreads, 0, stream>>>(seq_lens, batch, P, max_pages, target,
                                                   split_off, splits, max_splits, num_splits, err);
}

}  // namespace cfr
