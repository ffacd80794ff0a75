// cfr_demote.cu -- page demotion down the compression cascade, and KV append.
//
// Demotion re-encodes whole pages from one storage format into another: the
// compression cascade of the ARGUS page ("Visual Architecture": hot pages in
// full precision, cold pages FP8 -> INT8 -> INT4).  Per (page, kv head,
// K-or-V) block of P rows x d, over its first `valid` rows:
//   x      = stored value as fp32 (quantised sources: code * scale in fp32);
//   scale  = max|x| / Q in fp32 (Q = 127 int8, 7 int4, 448 FP8 E4M3);
//   int    code = clamp(round_half_even(x / scale), -Q, Q), IEEE fp32 division;
//   FP8    code = E4M3 nearest to x / scale, saturating at 448;
//   BF16   x rounded to nearest even; F32: x.
// An all-zero block gets scale 0 and zero codes; rows past `valid` are
// written as zero bytes.  One CTA per block: pass 1 reduces max|x| over the
// valid rows with every load of a thread in flight at once, pass 2 encodes and
// writes the codes with coalesced vector stores.  A block of up to 4096
// vectors of 8 elements (bf16 / int / FP8 sources; 2048 for fp32, e.g. 256
// tokens x 128 dims) stays in registers between the passes; a larger one is
// read again in pass 2, from L2.  The kernel is bound by HBM: it reads the
// source block once from DRAM and writes the destination block once.
//
// Append writes the new K and V rows of one decode step into the hot tier:
// token j = positions[b] of sequence b goes to row j % P of logical page j / P
// (ARGUS page, "The One-Minute Explanation": recent tokens stay in
// high-fidelity memory), widened to fp32 or rounded to bf16.
#include <climits>

#include <cuda_bf16.h>

#include "cfr_common.cuh"

namespace cfr {

namespace {

constexpr int kDemoteThreads = 512;
constexpr int kVec = 8;  // elements per vector access

struct DemoteParams {
  const uint8_t *src_k, *src_v;
  const float *src_scales;
  long long src_pages;
  uint8_t *dst_k, *dst_v;
  float *dst_scales;
  long long dst_pages;
  const int32_t *src_slots, *dst_slots, *valid_tokens;
  uint32_t *err;
  int src_fmt, dst_fmt, Hkv, D, P;
};

// Raw stored bytes of kVec consecutive elements of a source format, loaded with
// one or two vector accesses and decoded later (so that every load of a thread
// is in flight before the first one is used).
template <int SRC>
struct RawVec {
  uint2 w;  // CFR_FMT_I8 and CFR_FMT_FP8: 8 one-byte codes
};
template <>
struct RawVec<CFR_FMT_F32> {
  uint4 a, b;
};
template <>
struct RawVec<CFR_FMT_BF16> {
  uint4 a;
};
template <>
struct RawVec<CFR_FMT_I4> {
  uint32_t w;
};

template <int SRC>
__device__ __forceinline__ RawVec<SRC> load_raw(const uint8_t *blk, long long v) {
  RawVec<SRC> r;
  if constexpr (SRC == CFR_FMT_F32) {
    const uint4 *p = reinterpret_cast<const uint4 *>(blk + 32 * v);
    r.a = p[0];
    r.b = p[1];
  } else if constexpr (SRC == CFR_FMT_BF16) {
    r.a = *reinterpret_cast<const uint4 *>(blk + 16 * v);
  } else if constexpr (SRC == CFR_FMT_I4) {
    r.w = *reinterpret_cast<const uint32_t *>(blk + 4 * v);
  } else {
    r.w = *reinterpret_cast<const uint2 *>(blk + 8 * v);
  }
  return r;
}

// the eight values of a raw vector as fp32 (quantised: code * scale, fp32 product)
template <int SRC>
__device__ __forceinline__ void decode_raw(const RawVec<SRC> &r, float scale, float (&x)[kVec]) {
  if constexpr (SRC == CFR_FMT_F32) {
    const uint32_t a[8] = {r.a.x, r.a.y, r.a.z, r.a.w, r.b.x, r.b.y, r.b.z, r.b.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = __uint_as_float(a[k]);
  } else if constexpr (SRC == CFR_FMT_BF16) {
    const uint32_t a[4] = {r.a.x, r.a.y, r.a.z, r.a.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = bf16_lo(a[k]);
      x[2 * k + 1] = bf16_hi(a[k]);
    }
  } else if constexpr (SRC == CFR_FMT_I8) {
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = __fmul_rn(i8_at(k < 4 ? r.w.x : r.w.y, k & 3), scale);
  } else if constexpr (SRC == CFR_FMT_FP8) {
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = __fmul_rn(e4m3_at(k < 4 ? r.w.x : r.w.y, k & 3), scale);
  } else {  // CFR_FMT_I4
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = __fmul_rn(i4_at(r.w, k), scale);
  }
}

// vectors a thread holds in registers: a block of up to kDemoteThreads * R
// vectors is read from DRAM once and encoded from registers
template <int SRC>
constexpr int resident_vectors() {
  return SRC == CFR_FMT_F32 ? 4 : 8;
}

__device__ __forceinline__ int int_code(float x, float scale, int q) {
  if (!(scale > 0.f)) return 0;
  const int c = __float2int_rn(__fdiv_rn(x, scale));  // NaN -> 0
  return min(max(c, -q), q);
}

__device__ __forceinline__ uint32_t fp8_code(float x, float scale) {
  if (!(scale > 0.f)) return 0u;
  const float q = __fdiv_rn(x, scale);
  if (q != q) return 0x7Fu;  // NaN: the positive E4M3 NaN code
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3));
}

// encodes eight values and stores them at element e of the destination block
__device__ __forceinline__ void store8(int fmt, uint8_t *blk, long long e, float scale,
                                       const float (&x)[kVec]) {
  if (fmt == CFR_FMT_F32) {
    float4 *p = reinterpret_cast<float4 *>(blk + 4 * e);
    p[0] = make_float4(x[0], x[1], x[2], x[3]);
    p[1] = make_float4(x[4], x[5], x[6], x[7]);
  } else if (fmt == CFR_FMT_BF16) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(x[2 * k]));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(x[2 * k + 1]));
      w[k] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4 *>(blk + 2 * e) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if (fmt == CFR_FMT_I8) {
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 8; ++k)
      w[k >> 2] |= (static_cast<uint32_t>(int_code(x[k], scale, 127)) & 0xFFu) << (8 * (k & 3));
    *reinterpret_cast<uint2 *>(blk + e) = make_uint2(w[0], w[1]);
  } else if (fmt == CFR_FMT_FP8) {
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 8; ++k) w[k >> 2] |= fp8_code(x[k], scale) << (8 * (k & 3));
    *reinterpret_cast<uint2 *>(blk + e) = make_uint2(w[0], w[1]);
  } else {  // CFR_FMT_I4: element 2i in the low nibble of byte i
    uint32_t w = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) w |= (static_cast<uint32_t>(int_code(x[k], scale, 7)) & 0xFu) << (4 * k);
    *reinterpret_cast<uint32_t *>(blk + e / 2) = w;
  }
}

__device__ __forceinline__ void store_zero8(int fmt, uint8_t *blk, long long e) {
  if (fmt == CFR_FMT_F32) {
    float4 *p = reinterpret_cast<float4 *>(blk + 4 * e);
    p[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    p[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else if (fmt == CFR_FMT_BF16) {
    *reinterpret_cast<uint4 *>(blk + 2 * e) = make_uint4(0u, 0u, 0u, 0u);
  } else if (fmt == CFR_FMT_I4) {
    *reinterpret_cast<uint32_t *>(blk + e / 2) = 0u;
  } else {
    *reinterpret_cast<uint2 *>(blk + e) = make_uint2(0u, 0u);
  }
}

__device__ __forceinline__ float qmax_of(int fmt) {
  return fmt == CFR_FMT_I8 ? 127.f : fmt == CFR_FMT_I4 ? 7.f : 448.f;
}

// One (page k, kv head g, K or V) block, resolved from blockIdx.x.
struct DemoteBlock {
  const uint8_t *src;
  uint8_t *dst;
  float *dst_scale;      // null for unquantised destinations
  float src_scale;       // 1 for unquantised sources
  long long nvec_valid;  // vectors of kVec elements in the valid rows
  long long nvec;        // vectors in the whole block
};

// resolves the CTA's block; false (after reporting) when its slots or valid
// count are out of range, in which case nothing is written
__device__ __forceinline__ bool resolve_block(const DemoteParams &p, int src_fmt, DemoteBlock &b) {
  const long long blk_id = blockIdx.x;
  const int kv = static_cast<int>(blk_id & 1);
  const int g = static_cast<int>((blk_id >> 1) % p.Hkv);
  const long long k = (blk_id >> 1) / p.Hkv;
  const long long s = p.src_slots[k], t = p.dst_slots[k];
  const int valid = p.valid_tokens ? p.valid_tokens[k] : p.P;
  if (s < 0 || s >= p.src_pages || t < 0 || t >= p.dst_pages) {
    if (threadIdx.x == 0) set_err(p.err, CFR_DEVERR_PAGE_ID);
    return false;
  }
  if (valid < 1 || valid > p.P) {
    if (threadIdx.x == 0) set_err(p.err, CFR_DEVERR_SEQ_LEN);
    return false;
  }
  b.src = (kv ? p.src_v : p.src_k) + (s * p.Hkv + g) * p.P * row_bytes(src_fmt, p.D);
  b.dst = (kv ? p.dst_v : p.dst_k) + (t * p.Hkv + g) * p.P * row_bytes(p.dst_fmt, p.D);
  b.dst_scale = is_quantised(p.dst_fmt) ? p.dst_scales + (t * p.Hkv + g) * 2 + kv : nullptr;
  b.src_scale = is_quantised(src_fmt) ? p.src_scales[(s * p.Hkv + g) * 2 + kv] : 1.f;
  b.nvec_valid = static_cast<long long>(valid) * p.D / kVec;
  b.nvec = static_cast<long long>(p.P) * p.D / kVec;
  return true;
}

// The block with every decision taken as written above (IEEE division per
// element).  Called by all CTAs of the block together (it holds __syncthreads).
template <int SRC>
__device__ __forceinline__ void demote_block_exact(const DemoteParams &p, const DemoteBlock &b,
                                                   float *red) {
  constexpr int R = resident_vectors<SRC>();
  constexpr int T = kDemoteThreads;
  const uint8_t *src = b.src;
  uint8_t *dst = b.dst;
  const float src_scale = b.src_scale;
  const long long nvec_valid = b.nvec_valid;
  const int tid = threadIdx.x;
  // the whole valid part of the block fits the registers of the CTA
  const bool resident = nvec_valid <= static_cast<long long>(R) * T;
  RawVec<SRC> buf[R];

  float scale = 1.f;
  if (is_quantised(p.dst_fmt)) {
    // pass 1: max |x| over the valid rows, R independent loads in flight per thread
    float amax = 0.f;
    for (long long c0 = 0; c0 < nvec_valid; c0 += static_cast<long long>(R) * T) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const long long v = c0 + static_cast<long long>(r) * T + tid;
        if (v < nvec_valid) buf[r] = load_raw<SRC>(src, v);
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const long long v = c0 + static_cast<long long>(r) * T + tid;
        if (v < nvec_valid) {
          float x[kVec];
          decode_raw<SRC>(buf[r], src_scale, x);
#pragma unroll
          for (int i = 0; i < kVec; ++i) amax = fmaxf(amax, fabsf(x[i]));
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < T / 32; ++w) amax = fmaxf(amax, red[w]);
    scale = __fdiv_rn(amax, qmax_of(p.dst_fmt));
    if (tid == 0) *b.dst_scale = scale;
  } else if (resident) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const long long v = static_cast<long long>(r) * T + tid;
      if (v < nvec_valid) buf[r] = load_raw<SRC>(src, v);
    }
  }
  // pass 2: encode and store (from registers when resident, else chunk by chunk
  // again, the re-read hitting L2)
  if (resident) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const long long v = static_cast<long long>(r) * T + tid;
      if (v < nvec_valid) {
        float x[kVec];
        decode_raw<SRC>(buf[r], src_scale, x);
        store8(p.dst_fmt, dst, v * kVec, scale, x);
      }
    }
  } else {
    for (long long c0 = 0; c0 < nvec_valid; c0 += static_cast<long long>(R) * T) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const long long v = c0 + static_cast<long long>(r) * T + tid;
        if (v < nvec_valid) buf[r] = load_raw<SRC>(src, v);
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const long long v = c0 + static_cast<long long>(r) * T + tid;
        if (v < nvec_valid) {
          float x[kVec];
          decode_raw<SRC>(buf[r], src_scale, x);
          store8(p.dst_fmt, dst, v * kVec, scale, x);
        }
      }
    }
  }
  for (long long v = nvec_valid + tid; v < b.nvec; v += T) store_zero8(p.dst_fmt, dst, v * kVec);
}

template <int SRC>
__global__ void __launch_bounds__(kDemoteThreads) demote_kernel(DemoteParams p) {
  __shared__ float red[kDemoteThreads / 32];
  DemoteBlock b;
  if (!resolve_block(p, SRC, b)) return;
  demote_block_exact<SRC>(p, b, red);
}

// ---------------------------------------------------------------------------
// The cascade's steps (bf16 -> E4M3 / int8 / int4, int8 -> int4 or E4M3,
// E4M3 -> int8 or int4) on blocks staged in shared memory.
//
// The codes are the ones defined above, code = rint(fl(x / scale)) (or the
// E4M3 code of fl(x / scale)), reached without a division per element.  Let q = x / scale (exact) and f = fl(q).
// With a normal, finite scale and r = fl(1 / scale) (one correctly rounded
// reciprocal per block), take r- = fl(r * (1 - 2^-20)) and r+ = fl(r * (1 + 2^-20)).
// Each of r, r-, r+ and f carries a relative rounding error of at most 2^-24,
// so x*r- and x*r+ (exact products) lie on either side of f:
//   |x*r-| <= |q| (1 - 2^-20 + 2^-23) < |f|,   |x*r+| >= |q| (1 + 2^-20 - 2^-23) > |f|
// (for tiny |q| all three round to 0).  One fused multiply-add of each into
// the magic constant 1.5 * 2^23, whose unit in the last place is 1, rounds
// the exact product to the nearest integer (ties to even) and leaves it in
// the low bits of the sum.  Rounding to nearest is monotone, so when both
// sums agree they equal rint(f): that is the code, and |code| <= Q (the clamp
// cannot bind: |x| <= max|x| and scale >= max|x| / Q to within 2^-24).  When
// they differ (a half-integer within about |q| * 2^-20 of the product, and
// every NaN), the eight elements of the vector are encoded again with the
// IEEE division.  On bf16 blocks of N(0,1) values that is about one element in
// 600: a value that is a simple fraction of max|x| (max|x| / 2, say) puts
// x / scale within an ulp of a half-integer.  E4M3 destinations
// round the two products to fp32 and then to E4M3, both monotone, so equal
// codes of the two are the code of f.  A block whose maximum is infinite or
// whose scale is zero or subnormal (where the bounds above fail) is encoded
// with the division throughout.
// max|x| is taken on the codes (src_absmax_acc), equal to the fp32 maximum of
// the decoded values.
// ---------------------------------------------------------------------------

constexpr float kRintMagic = 12582912.0f;         // 1.5 * 2^23
constexpr uint32_t kRintMagicBits = 0x4B400000u;  // its bit pattern

// Running max|x| of bf16 pairs: per half, max(|m|, |w|) (its sign bit left
// arbitrary).  The bf16 max returns the other operand when one is NaN, as
// fmaxf does.
__device__ __forceinline__ uint32_t absmax_acc(uint32_t m, uint32_t w) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(m), "r"(w));
  return d;
}

__device__ __forceinline__ float absmax_value(uint32_t m) {
  return fmaxf(bf16_lo(m & 0x7FFF7FFFu), bf16_hi(m & 0x7FFF7FFFu));
}

// stores eight codes (the low byte, or for int4 the low nibble, of each tb)
// as vector v of the block
template <int DST>
__device__ __forceinline__ void store_codes8(uint8_t *dst, int v, const uint32_t (&tb)[kVec]) {
  if constexpr (DST == CFR_FMT_I4) {  // element 2i in the low nibble of byte i
    uint32_t n[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) n[k] = (tb[2 * k] & 0x0Fu) | (tb[2 * k + 1] << 4);
    reinterpret_cast<uint32_t *>(dst)[v] =
        __byte_perm(__byte_perm(n[0], n[1], 0x0040), __byte_perm(n[2], n[3], 0x0040), 0x5410);
  } else {  // int8 and E4M3: one byte each
    const uint32_t lo = __byte_perm(__byte_perm(tb[0], tb[1], 0x0040), __byte_perm(tb[2], tb[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(tb[4], tb[5], 0x0040), __byte_perm(tb[6], tb[7], 0x0040), 0x5410);
    reinterpret_cast<uint2 *>(dst)[v] = make_uint2(lo, hi);
  }
}

// The eight codes of one vector of decoded values x, from the two bracketing
// products x * r_lo and x * r_hi; true when they disagree somewhere (or a
// value is NaN), and the vector must be encoded again with the division.
//  - int8 / int4: each as 0x4B400000 + code (the rounded sum with 1.5 * 2^23);
//  - E4M3: the code of each rounded product (rounding to fp32 and then to E4M3
//    are both monotone, so equal codes of the two products are the code of
//    fl(x / scale), which lies between them).
template <int DST>
__device__ __forceinline__ bool codes8_fast(const float (&x)[kVec], float r_lo, float r_hi,
                                            uint32_t (&tb)[kVec]) {
  bool near = false;
#pragma unroll
  for (int k = 0; k < kVec; ++k) {
    if constexpr (DST == CFR_FMT_FP8) {
      const uint32_t lo = __nv_cvt_float_to_fp8(__fmul_rn(x[k], r_lo), __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float_to_fp8(__fmul_rn(x[k], r_hi), __NV_SATFINITE, __NV_E4M3);
      near |= (lo != hi) || (x[k] != x[k]);
      tb[k] = lo;
    } else {
      const float lo = __fmaf_rn(x[k], r_lo, kRintMagic);
      const float hi = __fmaf_rn(x[k], r_hi, kRintMagic);
      near |= lo != hi;
      tb[k] = __float_as_uint(lo);
    }
  }
  return near;
}

// the same codes with the IEEE division
template <int DST>
__device__ __forceinline__ void codes8_exact(const float (&x)[kVec], float scale, uint32_t (&tb)[kVec]) {
#pragma unroll
  for (int k = 0; k < kVec; ++k) {
    if constexpr (DST == CFR_FMT_FP8)
      tb[k] = fp8_code(x[k], scale);
    else
      tb[k] = kRintMagicBits + static_cast<uint32_t>(int_code(x[k], scale, DST == CFR_FMT_I8 ? 127 : 7));
  }
}

// Running max|code| of one source vector, in the source's own terms:
//  - bf16: per half of m, max(|m|, |w|) of the bf16 pairs (NaN left out);
//  - int8: the largest |code| (0..128);
//  - E4M3: the largest magnitude byte (0..0x7E), NaN codes (0x7F) left out.
// For quantised sources max|x| = fl(max value * scale) for a non-negative
// finite scale, since x = fl(code * scale) is monotone in |code|.
template <int SRC>
__device__ __forceinline__ uint32_t src_absmax_acc(uint32_t m, const RawVec<SRC> &r) {
  if constexpr (SRC == CFR_FMT_BF16) {
    return absmax_acc(absmax_acc(absmax_acc(absmax_acc(m, r.a.x), r.a.y), r.a.z), r.a.w);
  } else {
    const uint32_t w[2] = {r.w.x, r.w.y};
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if constexpr (SRC == CFR_FMT_I8) {
          const int c = static_cast<int8_t>((w[i] >> (8 * k)) & 0xFFu);
          m = max(m, static_cast<uint32_t>(abs(c)));
        } else {  // CFR_FMT_FP8
          const uint32_t mag = (w[i] >> (8 * k)) & 0x7Fu;
          m = mag == 0x7Fu ? m : max(m, mag);
        }
      }
    return m;
  }
}

template <int SRC>
__device__ __forceinline__ uint32_t src_absmax_combine(uint32_t a, uint32_t b) {
  if constexpr (SRC == CFR_FMT_BF16)
    return absmax_acc(a, b);
  else
    return max(a, b);
}

template <int SRC>
__device__ __forceinline__ float src_absmax_value(uint32_t m, float src_scale) {
  if constexpr (SRC == CFR_FMT_BF16)
    return absmax_value(m);
  else if constexpr (SRC == CFR_FMT_I8)
    return __fmul_rn(static_cast<float>(m), src_scale);
  else
    return __fmul_rn(e4m3_at(m, 0), src_scale);
}

// The block is staged in shared memory by one bulk copy (all of it in flight
// at once), with three 256-thread CTAs per SM; the max pass and the encode
// pass read it there.  Blocks of up to 64 KiB and 8192 vectors of 8 elements.
// Pairs: bf16 -> int8 / int4 / E4M3, int8 -> int4 / E4M3, E4M3 -> int8 (E4M3
// -> int4 measured faster on the general kernel).
constexpr int kSmemThreads = 256;
constexpr int kSmemBlockBytes = 65536;
constexpr int kSmemMaxVecs = 32 * kSmemThreads;  // one bit per vector of a thread in `redo`

template <int SRC, int DST>
__global__ void __launch_bounds__(kSmemThreads, 3) demote_staged_kernel(DemoteParams p) {
  constexpr int T = kSmemThreads;
  // vectors of a thread: as many as a 64 KiB block holds, at most 32
  constexpr int ITERS = kSmemBlockBytes / static_cast<int>(sizeof(RawVec<SRC>)) / T < kSmemMaxVecs / T
                            ? kSmemBlockBytes / static_cast<int>(sizeof(RawVec<SRC>)) / T
                            : kSmemMaxVecs / T;
  extern __shared__ __align__(128) uint8_t stage_bytes[];
  const RawVec<SRC> *stage = reinterpret_cast<const RawVec<SRC> *>(stage_bytes);
  __shared__ uint64_t bar;
  __shared__ uint32_t redw[T / 32];
  __shared__ float redf[T / 32];
  DemoteBlock b;
  if (!resolve_block(p, SRC, b)) return;
  const int tid = threadIdx.x;
  const int nv = static_cast<int>(b.nvec_valid);
  const float s_src = b.src_scale;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(nv * sizeof(RawVec<SRC>)));
    bulk_g2s(stage_bytes, b.src, static_cast<uint32_t>(nv * sizeof(RawVec<SRC>)), &bar);
  }
  __syncthreads();
  bool timed_out = false;
  if (!mbar_wait(&bar, 0, p.err, &timed_out)) return;
  // max|x|: from the codes while the source scale is finite and non-negative,
  // else over the decoded values as written (fmaxf, NaN left out)
  const bool src_ok = SRC == CFR_FMT_BF16 || (s_src >= 0.f && s_src <= 3.40282347e+38f);
  float amax;
  if (src_ok) {
    uint32_t m = 0u;
#pragma unroll 4
    for (int v = tid; v < nv; v += T) m = src_absmax_acc<SRC>(m, stage[v]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = src_absmax_combine<SRC>(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) redw[tid >> 5] = m;
    __syncthreads();
    m = redw[0];
#pragma unroll
    for (int w = 1; w < T / 32; ++w) m = src_absmax_combine<SRC>(m, redw[w]);
    amax = src_absmax_value<SRC>(m, s_src);
  } else {
    float a = 0.f;
    for (int v = tid; v < nv; v += T) {
      float x[kVec];
      decode_raw<SRC>(stage[v], s_src, x);
#pragma unroll
      for (int k = 0; k < kVec; ++k) a = fmaxf(a, fabsf(x[k]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((tid & 31) == 0) redf[tid >> 5] = a;
    __syncthreads();
    a = redf[0];
#pragma unroll
    for (int w = 1; w < T / 32; ++w) a = fmaxf(a, redf[w]);
    amax = a;
  }
  const float scale = __fdiv_rn(amax, qmax_of(DST));
  const bool fast = scale >= 1.17549435e-38f && scale <= 3.40282347e+38f;  // normal and finite
  if (tid == 0) *b.dst_scale = scale;
  // encode: vectors near a tie are marked in `redo` and encoded again after
  // the loop, which keeps the division out of the loop body
  uint32_t redo = 0u;
  if (fast) {
    const float r = __frcp_rn(scale);
    const float r_lo = __fmul_rn(r, 1.f - 0x1p-20f), r_hi = __fmul_rn(r, 1.f + 0x1p-20f);
#pragma unroll 4
    for (int i = 0; i < ITERS; ++i) {
      const int v = i * T + tid;
      if (v < nv) {
        float x[kVec];
        decode_raw<SRC>(stage[v], s_src, x);
        uint32_t tb[kVec];
        redo |= static_cast<uint32_t>(codes8_fast<DST>(x, r_lo, r_hi, tb)) << i;
        store_codes8<DST>(b.dst, v, tb);
      }
    }
  } else {
    for (int i = 0; i * T + tid < nv; ++i) redo |= 1u << i;
  }
  while (redo) {
    const int i = __ffs(redo) - 1;
    redo &= redo - 1;
    const int v = i * T + tid;
    float x[kVec];
    decode_raw<SRC>(stage[v], s_src, x);
    uint32_t tb[kVec];
    codes8_exact<DST>(x, scale, tb);
    store_codes8<DST>(b.dst, v, tb);
  }
  for (long long v = b.nvec_valid + tid; v < b.nvec; v += T) store_zero8(DST, b.dst, v * kVec);
}

template <int SRC, int DST>
cudaError_t launch_staged(const DemoteParams &p, unsigned blocks, cudaStream_t s) {
  auto kern = demote_staged_kernel<SRC, DST>;
  const cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBlockBytes);
  if (e != cudaSuccess) return e;
  kern<<<blocks, kSmemThreads, kSmemBlockBytes, s>>>(p);
  return cudaGetLastError();
}

// the staged kernel for (src, dst) when it serves the pair and the block fits;
// cudaErrorNotSupported otherwise
cudaError_t try_launch_staged(const DemoteParams &p, int src, int dst, unsigned blocks, cudaStream_t s) {
  const long long vecs = static_cast<long long>(p.P) * p.D / kVec;
  const long long bytes = static_cast<long long>(p.P) * row_bytes(src, p.D);
  if (vecs > kSmemMaxVecs || bytes > kSmemBlockBytes) return cudaErrorNotSupported;
#define CFR_STAGED(S, D) \
  if (src == S && dst == D) return launch_staged<S, D>(p, blocks, s);
  CFR_STAGED(CFR_FMT_BF16, CFR_FMT_I8) CFR_STAGED(CFR_FMT_BF16, CFR_FMT_I4) CFR_STAGED(CFR_FMT_BF16, CFR_FMT_FP8)
  CFR_STAGED(CFR_FMT_I8, CFR_FMT_I4) CFR_STAGED(CFR_FMT_I8, CFR_FMT_FP8) CFR_STAGED(CFR_FMT_FP8, CFR_FMT_I8)
#undef CFR_STAGED
  return cudaErrorNotSupported;
}

struct AppendParams {
  uint8_t *k_pool[kFmtCount];
  uint8_t *v_pool[kFmtCount];
  long long pool_pages[kFmtCount];
  const int32_t *page_table;
  const uint8_t *page_fmt;
  const int32_t *positions;
  const void *k_new, *v_new;
  uint32_t *err;
  int uniform_fmt, new_fmt, max_pages, Hkv, D, P;
};

// sequence b = blockIdx.x; threads cover Hkv x D elements of K and V
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
  const int b = blockIdx.x;
  const long long j = p.positions[b];
  if (j < 0) return;
  if (j >= static_cast<long long>(p.max_pages) * p.P) {
    if (threadIdx.x == 0) set_err(p.err, CFR_DEVERR_SEQ_LEN);
    return;
  }
  const long long cell = static_cast<long long>(b) * p.max_pages + j / p.P;
  const int fmt = p.page_fmt ? static_cast<int>(p.page_fmt[cell]) : p.uniform_fmt;
  if ((fmt != CFR_FMT_F32 && fmt != CFR_FMT_BF16) || !p.k_pool[fmt] || !p.v_pool[fmt]) {
    if (threadIdx.x == 0) set_err(p.err, CFR_DEVERR_PAGE_FMT);
    return;
  }
  const long long slot = p.page_table[cell];
  if (slot < 0 || slot >= p.pool_pages[fmt]) {
    if (threadIdx.x == 0) set_err(p.err, CFR_DEVERR_PAGE_ID);
    return;
  }
  const int rb = row_bytes(fmt, p.D);
  const int tin = static_cast<int>(j % p.P);
  const int n = p.Hkv * p.D;
  for (int i = threadIdx.x; i < 2 * n; i += blockDim.x) {
    const int kv = i >= n;
    const int e = kv ? i - n : i;
    const int g = e / p.D, c = e - g * p.D;
    const long long src_i = static_cast<long long>(b) * n + e;
    const void *srcv = kv ? p.v_new : p.k_new;
    const float x = p.new_fmt == CFR_FMT_F32
                        ? static_cast<const float *>(srcv)[src_i]
                        : __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t *>(srcv)[src_i]) << 16);
    uint8_t *row = (kv ? p.v_pool[fmt] : p.k_pool[fmt]) + ((slot * p.Hkv + g) * p.P + tin) * rb;
    if (fmt == CFR_FMT_F32)
      reinterpret_cast<float *>(row)[c] = x;
    else
      reinterpret_cast<uint16_t *>(row)[c] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
  }
}

bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// pool geometry shared by demotion and append
cfr_status check_geometry(const cfr_kv_pool *kv) {
  if (!kv) return CFR_ERR_INVALID_ARG;
  if (kv->num_kv_heads <= 0 || kv->head_dim <= 0 || kv->page_tokens <= 0) return CFR_ERR_INVALID_ARG;
  if (kv->head_dim != 64 && kv->head_dim != 128) return CFR_ERR_UNSUPPORTED;
  if (kv->page_tokens < 8) return CFR_ERR_UNSUPPORTED;
  return CFR_OK;
}

bool pool_bytes_fit(long long pages, const cfr_kv_pool *kv, int fmt) {
  if (pages < 0) return false;
  const long long per = static_cast<long long>(kv->num_kv_heads) * kv->page_tokens *
                        row_bytes(fmt, kv->head_dim);
  return pages == 0 || per <= LLONG_MAX / pages;
}

}  // namespace
}  // namespace cfr

using namespace cfr;

extern "C" {

cfr_status cfr_demote_pages(const cfr_kv_pool *kv, int32_t src_fmt, int32_t dst_fmt,
                            void *dst_k_pool, void *dst_v_pool, float *dst_scales,
                            int64_t dst_pool_pages, const int32_t *src_slots,
                            const int32_t *dst_slots, const int32_t *valid_tokens,
                            int32_t num_pages, uint32_t *err_word, void *stream) {
  cfr_status st = check_geometry(kv);
  if (st != CFR_OK) return st;
  if (src_fmt < 0 || src_fmt >= kFmtCount || dst_fmt < 0 || dst_fmt >= kFmtCount ||
      src_fmt == dst_fmt)
    return CFR_ERR_INVALID_ARG;
  if (num_pages < 0) return CFR_ERR_INVALID_ARG;
  if (!kv->k_pool[src_fmt] || !kv->v_pool[src_fmt] || !dst_k_pool || !dst_v_pool)
    return CFR_ERR_INVALID_ARG;
  if (!aligned_to(kv->k_pool[src_fmt], 16) || !aligned_to(kv->v_pool[src_fmt], 16) ||
      !aligned_to(dst_k_pool, 16) || !aligned_to(dst_v_pool, 16))
    return CFR_ERR_INVALID_ARG;
  if (is_quantised(src_fmt) && (!kv->scales[src_fmt] || !aligned_to(kv->scales[src_fmt], 8)))
    return CFR_ERR_INVALID_ARG;
  if (is_quantised(dst_fmt) && (!dst_scales || !aligned_to(dst_scales, 8))) return CFR_ERR_INVALID_ARG;
  if (!pool_bytes_fit(kv->pool_pages[src_fmt], kv, src_fmt) || !pool_bytes_fit(dst_pool_pages, kv, dst_fmt))
    return CFR_ERR_OVERFLOW;
  if (static_cast<long long>(num_pages) * kv->num_kv_heads * 2 > INT_MAX) return CFR_ERR_OVERFLOW;
  if (num_pages == 0) return CFR_OK;
  if (!src_slots || !dst_slots) return CFR_ERR_INVALID_ARG;
  DemoteParams p;
  p.src_k = static_cast<const uint8_t *>(kv->k_pool[src_fmt]);
  p.src_v = static_cast<const uint8_t *>(kv->v_pool[src_fmt]);
  p.src_scales = kv->scales[src_fmt];
  p.src_pages = kv->pool_pages[src_fmt];
  p.dst_k = static_cast<uint8_t *>(dst_k_pool);
  p.dst_v = static_cast<uint8_t *>(dst_v_pool);
  p.dst_scales = dst_scales;
  p.dst_pages = dst_pool_pages;
  p.src_slots = src_slots;
  p.dst_slots = dst_slots;
  p.valid_tokens = valid_tokens;
  p.err = err_word;
  p.src_fmt = src_fmt;
  p.dst_fmt = dst_fmt;
  p.Hkv = kv->num_kv_heads;
  p.D = kv->head_dim;
  p.P = kv->page_tokens;
  const unsigned blocks = static_cast<unsigned>(num_pages) * kv->num_kv_heads * 2u;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t staged = try_launch_staged(p, src_fmt, dst_fmt, blocks, s);
  if (staged != cudaErrorNotSupported) return staged == cudaSuccess ? CFR_OK : CFR_ERR_CUDA;
  switch (src_fmt) {
    case CFR_FMT_F32: demote_kernel<CFR_FMT_F32><<<blocks, kDemoteThreads, 0, s>>>(p); break;
    case CFR_FMT_BF16: demote_kernel<CFR_FMT_BF16><<<blocks, kDemoteThreads, 0, s>>>(p); break;
    case CFR_FMT_I8: demote_kernel<CFR_FMT_I8><<<blocks, kDemoteThreads, 0, s>>>(p); break;
    case CFR_FMT_I4: demote_kernel<CFR_FMT_I4><<<blocks, kDemoteThreads, 0, s>>>(p); break;
    default: demote_kernel<CFR_FMT_FP8><<<blocks, kDemoteThreads, 0, s>>>(p); break;
  }
  return cudaGetLastError() == cudaSuccess ? CFR_OK : CFR_ERR_CUDA;
}

cfr_status cfr_append_kv(const cfr_kv_pool *kv, const int32_t *page_table, int32_t max_pages,
                         const uint8_t *page_fmt, int32_t uniform_fmt, const int32_t *positions,
                         int32_t batch, const void *k_new, const void *v_new, int32_t new_fmt,
                         uint32_t *err_word, void *stream) {
  cfr_status st = check_geometry(kv);
  if (st != CFR_OK) return st;
  if (!page_table || !positions || !k_new || !v_new) return CFR_ERR_INVALID_ARG;
  if (batch <= 0 || max_pages <= 0) return CFR_ERR_INVALID_ARG;
  if (new_fmt != CFR_FMT_F32 && new_fmt != CFR_FMT_BF16) return CFR_ERR_INVALID_ARG;
  if (!page_fmt && uniform_fmt != CFR_FMT_F32 && uniform_fmt != CFR_FMT_BF16) return CFR_ERR_INVALID_ARG;
  if (static_cast<long long>(max_pages) * kv->page_tokens > INT_MAX ||
      static_cast<long long>(batch) * max_pages > INT_MAX)
    return CFR_ERR_OVERFLOW;
  AppendParams p;
  bool any = false;
  for (int f = 0; f < kFmtCount; ++f) {
    const bool hot = f == CFR_FMT_F32 || f == CFR_FMT_BF16;
    p.k_pool[f] = hot ? static_cast<uint8_t *>(const_cast<void *>(kv->k_pool[f])) : nullptr;
    p.v_pool[f] = hot ? static_cast<uint8_t *>(const_cast<void *>(kv->v_pool[f])) : nullptr;
    p.pool_pages[f] = p.k_pool[f] ? kv->pool_pages[f] : 0;
    if (!p.k_pool[f] != !p.v_pool[f]) return CFR_ERR_INVALID_ARG;
    if (p.k_pool[f]) {
      if (!aligned_to(p.k_pool[f], 16) || !aligned_to(p.v_pool[f], 16)) return CFR_ERR_INVALID_ARG;
      if (!pool_bytes_fit(kv->pool_pages[f], kv, f)) return CFR_ERR_OVERFLOW;
      any = true;
    }
  }
  if (!any) return CFR_ERR_INVALID_ARG;
  p.page_table = page_table;
  p.page_fmt = page_fmt;
  p.positions = positions;
  p.k_new = k_new;
  p.v_new = v_new;
  p.err = err_word;
  p.uniform_fmt = uniform_fmt;
  p.new_fmt = new_fmt;
  p.max_pages = max_pages;
  p.Hkv = kv->num_kv_heads;
  p.D = kv->head_dim;
  p.P = kv->page_tokens;
  append_kernel<<<batch, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? CFR_OK : CFR_ERR_CUDA;
}

}  // extern "C"
