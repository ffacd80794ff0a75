// cfr_merge.cu -- log-sum-exp merge of split partials (one warp per (b, h)).
//
// For sequence b and query head h the splits s in [split_off[b], split_off[b+1])
// hold (m_s, l_s, a_s): base-2 running maximum, normaliser and unnormalised
// weighted-V accumulator.  The merge rescales every split to the common
// maximum M and normalises once:
//   out = sum_s 2^(m_s - M) a_s / sum_s 2^(m_s - M) l_s,   lse = (M + log2 L) ln 2
// (the combine rule of online softmax; the merge step of the CMF page's
// split-K flash-decoding).  Splits with l_s = 0 carry no token and are skipped.
// Work per sequence grows with its number of splits, i.e. with its length.
// The summation order is fixed, so the result is deterministic.
#include "cfr_common.cuh"

namespace cfr {

constexpr int kMergeWarps = 8;

template <int D>
__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(
    const float *__restrict__ part_acc, const float *__restrict__ part_m,
    const float *__restrict__ part_l, const int32_t *__restrict__ split_off, int batch, int Hq,
    float *__restrict__ out, float *__restrict__ lse) {
  constexpr int DPL = D / 32;
  const int lane = threadIdx.x & 31;
  const long long pair = static_cast<long long>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
  if (pair >= static_cast<long long>(batch) * Hq) return;
  const int b = static_cast<int>(pair / Hq), h = static_cast<int>(pair % Hq);
  const int s0 = split_off[b], s1 = split_off[b + 1];

  // M = max over non-empty splits (lanes stride the splits, then a fixed tree)
  float M = -INFINITY;
  for (int s = s0 + lane; s < s1; s += 32) {
    const long long c = static_cast<long long>(s) * Hq + h;
    if (part_l[c] > 0.f) M = fmaxf(M, part_m[c]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));

  float o_acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) o_acc[i] = 0.f;
  float L = 0.f;
  if (M != -INFINITY) {
    // normaliser: lane-strided partial sums, then a fixed tree
    for (int s = s0 + lane; s < s1; s += 32) {
      const long long c = static_cast<long long>(s) * Hq + h;
      const float l = part_l[c];
      if (l > 0.f) L = fmaf(l, exp2_approx(part_m[c] - M), L);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    // accumulators: four splits per step with independent loads; empty splits
    // contribute nothing whatever their accumulator holds
    for (int s = s0; s < s1; s += 4) {
      float w[4], a[4][DPL];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        w[u] = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) a[u][i] = 0.f;
        if (s + u < s1) {
          const long long c = static_cast<long long>(s + u) * Hq + h;
          const float l = part_l[c];
          const float m = part_m[c];
          const float *ap = part_acc + c * D + lane * DPL;
          if constexpr (DPL == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(ap);
            a[u][0] = v.x; a[u][1] = v.y; a[u][2] = v.z; a[u][3] = v.w;
          } else {
            const float2 v = *reinterpret_cast<const float2 *>(ap);
            a[u][0] = v.x; a[u][1] = v.y;
          }
          w[u] = l > 0.f ? exp2_approx(m - M) : 0.f;
          if (!(l > 0.f)) {
#pragma unroll
            for (int i = 0; i < DPL; ++i) a[u][i] = 0.f;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < DPL; ++i) o_acc[i] = fmaf(w[u], a[u][i], o_acc[i]);
    }
  }
  float *o = out + pair * D + lane * DPL;
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if constexpr (DPL == 4) {
    *reinterpret_cast<float4 *>(o) =
        make_float4(o_acc[0] * inv, o_acc[1] * inv, o_acc[2] * inv, o_acc[3] * inv);
  } else {
    *reinterpret_cast<float2 *>(o) = make_float2(o_acc[0] * inv, o_acc[1] * inv);
  }
  if (lse && lane == 0) lse[pair] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

void launch_merge(const float *part_acc, const float *part_m, const float *part_l,
                  const int32_t *split_off, int batch, int Hq, int D, float *out, float *lse,
                  cudaStream_t stream) {
  const long long pairs = static_cast<long long>(batch) * Hq;
  const unsigned blocks = static_cast<unsigned>((pairs + kMergeWarps - 1) / kMergeWarps);
  if (blocks == 0) return;
  if (D == 64)
    merge_kernel<64><<<blocks, kMergeWarps * 32, 0, stream>>>(part_acc, part_m, part_l,
                                                             split_off, batch, Hq, out, lse);
  else
    merge_kernel<128><<<blocks, kMergeWarps * 32, 0, stream>>>(part_acc, part_m, part_l,
                                                              split_off, batch, Hq, out, lse);
}

}  // namespace cfr
