// cfr_merge.cu -- log-sum-exp merge of split partials (one CTA per (b, h)).
//
// For sequence b and query head h the splits s in [split_off[b], split_off[b+1])
// hold (m_s, l_s, a_s): base-2 running maximum, normaliser and unnormalised
// weighted-V accumulator.  The merge rescales every split to the common
// maximum M and normalises once:
//   out = sum_s 2^(m_s - M) a_s / sum_s 2^(m_s - M) l_s,   lse = (M + log2 L) ln 2
// (the combine rule of online softmax; the merge step of the CMF page's
// split-K flash-decoding).  Splits with l_s = 0 carry no token and are skipped.
// The weights 2^(m_s - M) are computed once per split by all threads together;
// then four groups of 128 threads each sum a quarter of the splits (thread i of a
// group owns dim i) with independent loads in flight, and the four group sums
// are added in a fixed order.
// Work per sequence grows with its number of splits, i.e. with its length.
// Every sum runs in a fixed order, so the result is deterministic.
#include "cfr_common.cuh"

namespace cfr {

constexpr int kMergeThreads = 512;  // four groups of 128 threads
constexpr int kMergeGroups = 4;
constexpr int kMergeChunk = 512;  // splits whose weights are staged in shared memory at once

template <int D>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(
    const float *__restrict__ part_acc, const float *__restrict__ part_m,
    const float *__restrict__ part_l, const int32_t *__restrict__ split_off, int batch, int Hq,
    int max_splits, float *__restrict__ out, float *__restrict__ lse, uint32_t *err) {
  __shared__ float w_s[kMergeChunk];
  __shared__ float red[kMergeThreads / 32];
  __shared__ float gsum[kMergeGroups][D];
  __shared__ float shared_M, shared_L;
  griddep_wait();
  const long long pair = blockIdx.x;
  if (pair >= static_cast<long long>(batch) * Hq) return;
  const int b = static_cast<int>(pair / Hq), h = static_cast<int>(pair % Hq);
  int s0 = split_off[b], s1 = split_off[b + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (s0 < 0 || s1 < s0 || s1 > max_splits) {
    // offsets that do not index this call's partial arrays (a merge-only call on
    // a workspace scheduled with other arguments): merge only what is in range
    if (tid == 0) set_err(err, CFR_DEVERR_SCHEDULE);
    s0 = min(max(s0, 0), max_splits);
    s1 = min(max(s1, s0), max_splits);
  }

  // M = max over non-empty splits
  float M = -INFINITY;
  for (int s = s0 + tid; s < s1; s += kMergeThreads) {
    const long long c = static_cast<long long>(s) * Hq + h;
    if (part_l[c] > 0.f) M = fmaxf(M, part_m[c]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  if (tid == 0) {
    float m = red[0];
    for (int w = 1; w < kMergeThreads / 32; ++w) m = fmaxf(m, red[w]);
    shared_M = m;
  }
  __syncthreads();
  M = shared_M;

  float acc = 0.f, L = 0.f;
  if (M != -INFINITY) {
    for (int c0 = s0; c0 < s1; c0 += kMergeChunk) {
      const int c1 = min(s1, c0 + kMergeChunk);
      // weights of this chunk of splits (0 for empty splits) and their normaliser share
      float lsum = 0.f;
      for (int s = c0 + tid; s < c1; s += kMergeThreads) {
        const long long c = static_cast<long long>(s) * Hq + h;
        const float l = part_l[c];
        const float w = l > 0.f ? exp2_approx(part_m[c] - M) : 0.f;
        w_s[s - c0] = w;
        lsum = fmaf(l > 0.f ? l : 0.f, w, lsum);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
      __syncthreads();
      if (lane == 0) red[warp] = lsum;
      __syncthreads();
      if (tid == 0) {
        float t = 0.f;
        for (int w = 0; w < kMergeThreads / 32; ++w) t += red[w];
        shared_L = t;
      }
      // group grp sums the splits c0 + grp, c0 + grp + 4, ...; thread dim owns dim `dim`
      const int grp = tid >> 7, dim = tid & 127;
      if (dim < D) {
        const long long stride = static_cast<long long>(Hq) * D;
        const float *ap = part_acc + (static_cast<long long>(c0) * Hq + h) * D + dim;
        const int n = c1 - c0;
        int s = grp;
        for (; s + 4 * 7 < n; s += 4 * 8) {
          float a[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) a[u] = ap[(s + 4 * u) * stride];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (w_s[s + 4 * u] != 0.f) acc = fmaf(w_s[s + 4 * u], a[u], acc);
        }
        for (; s < n; s += 4) {
          const float a = ap[s * stride];
          if (w_s[s] != 0.f) acc = fmaf(w_s[s], a, acc);
        }
      }
      __syncthreads();
      L += shared_L;
    }
  }
  // add the four groups' sums in a fixed order
  const int grp = tid >> 7, dim = tid & 127;
  if (dim < D) gsum[grp][dim] = acc;
  __syncthreads();
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (tid < D) out[pair * D + tid] = ((gsum[0][tid] + gsum[1][tid]) + (gsum[2][tid] + gsum[3][tid])) * inv;
  if (lse && tid == 0) lse[pair] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

void launch_merge(const float *part_acc, const float *part_m, const float *part_l,
                  const int32_t *split_off, int batch, int Hq, int D, int max_splits, float *out,
                  float *lse, uint32_t *err, cudaStream_t stream) {
  const long long pairs = static_cast<long long>(batch) * Hq;
  if (pairs <= 0) return;
  const unsigned blocks = static_cast<unsigned>(pairs);
  if (D == 64)
    (void)launch_after_previous(merge_kernel<64>, dim3(blocks), dim3(kMergeThreads), 0, stream,
                                part_acc, part_m, part_l, split_off, batch, Hq, max_splits, out, lse, err);
  else
    (void)launch_after_previous(merge_kernel<128>, dim3(blocks), dim3(kMergeThreads), 0, stream,
                                part_acc, part_m, part_l, split_off, batch, Hq, max_splits, out, lse, err);
}

}  // namespace cfr
