// cfr_common.cuh -- device helpers shared by the decode-attention kernels (sm_100a).
//
// mbarrier-based producer/consumer hand-off with bounded waits, the 1-D bulk
// copy engine (TMA, no multicast), error-word reporting and small numeric
// helpers.  Every spin on an mbarrier gives up after a clock-cycle limit (about
// two seconds), sets CFR_DEVERR_TIMEOUT in the error word and lets the kernel
// return.
#pragma once

#include <cstdint>
#include <utility>

#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "cfr_paged.h"

namespace cfr {

constexpr int kFmtCount = CFR_FMT_COUNT;
constexpr int kMaxQHeads = 256;
constexpr int kMaxGroup = 16;              // query rows of one work-item group
// groups: a kv head with more than kMaxGroup query rows is split into several
// groups of at most kMaxGroup rows (each reads the kv head's pages itself)
constexpr int kMaxGroups = kMaxQHeads + kMaxQHeads / kMaxGroup;
// bytes of one query operand image of the tensor-core decode (16-column
// variants): bf16 hi/lo rows, fp16 hi/lo rows, int8 digit rows
constexpr int kQImgBytes = 16 * 256 * 2 + 16 * 128;

// Parameters of one decode call, shared by both decode kernels.
struct DecodeParams {
  const void *q;
  const uint8_t *k_pool[kFmtCount];
  const uint8_t *v_pool[kFmtCount];
  const float *scales[kFmtCount];
  long long pool_pages[kFmtCount];
  const int32_t *page_table;
  const uint8_t *page_fmt;
  const int32_t *seq_lens;
  const float *slopes;
  float *part_acc;      // [S][Hq][D]
  float *part_m;        // [S][Hq], base-2 maxima
  float *part_l;        // [S][Hq]
  const int32_t *splits;     // [S][3]: b, page begin, page end
  const int32_t *num_splits; // [0] = S
  int max_splits;            // capacity of this call's split arrays (part_*, splits)
  uint32_t *item_ctr;   // [0] work items claimed past the first per CTA, [1] CTAs finished; or null
  uint8_t *qimg;        // [B * ngroups][kQImgBytes]: query operand image of each (sequence, group)
  float *qscale;        // [B * ngroups][4]: its int8 digit scales
  uint32_t *err;
  int q_fmt, uniform_fmt;
  int batch, max_pages, Hq, Hkv, D, P;
  // the split table's unit: splits are ranges [pb, pe) of split_unit tokens (P,
  // or 128 when P is a larger multiple of 128); max_units = max_pages * P / split_unit
  int split_unit, max_units;
  int pitch;            // shared-memory row pitch (bytes) of the CUDA-core kernel's stages
  int stages;
  float sigma_log2e;    // softmax scale times log2(e)
  int gmax;             // largest group size
  int sink, window;     // window > 0: only tokens j < sink or j >= n - window take part
  int nq;               // query tokens per sequence (the last nq positions, causal)
  int hq_real;          // query heads; the Hq = nq * hq_real query rows are qi * hq_real + h
  int ngroups;          // row groups (Hkv, or more when a kv head has over kMaxGroup rows)
  int gsub;             // groups per kv head when every kv head has the same number (else 1)
  int16_t grp_off[kMaxGroups + 1];  // rows of group g: grp_heads[grp_off[g] .. grp_off[g+1])
  int16_t grp_kv[kMaxGroups];       // the kv head whose pages group g reads
  int16_t grp_heads[kMaxQHeads];
};

__host__ __device__ inline int row_bytes(int fmt, int d) {
  return fmt == CFR_FMT_F32 ? 4 * d : fmt == CFR_FMT_BF16 ? 2 * d : fmt == CFR_FMT_I4 ? d / 2 : d;
}

// formats whose values are codes times a per-(page, kv head) scale
__host__ __device__ inline bool is_quantised(int fmt) {
  return fmt == CFR_FMT_I8 || fmt == CFR_FMT_I4 || fmt == CFR_FMT_FP8;
}

__device__ __forceinline__ void set_err(uint32_t *err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier --------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile(
      "{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Spin limit of every wait, in SM clock cycles: 4e9 cycles is about 2 s at the
// B200's top SM clock (more at lower clocks).  The cycle counter is read only
// every 64 polls, so the limit check costs nothing on the fast path.
constexpr long long kWaitLimitCycles = 4000000000LL;

// Waits for the phase of `parity` to complete.  Returns false (and flags the
// error word) when the wait exceeded `limit` cycles (kWaitLimitCycles unless a
// caller asks for less); `*timed_out` then stays set so that callers stop
// waiting on anything else.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *err,
                                          bool *timed_out,
                                          long long limit = kWaitLimitCycles) {
  if (*timed_out) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t spins = 1;; ++spins) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spins & 63u) == 0 && clock64() - t0 > limit) {
      set_err(err, CFR_DEVERR_TIMEOUT);
      *timed_out = true;
      return false;
    }
  }
}

// ---- 1-D bulk copy global -> shared (TMA engine, no multicast) ---------------

// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---- programmatic dependent launch -------------------------------------------

// Lets the next kernel of the stream start its prologue now (it still waits for
// this grid's results before reading them).
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Waits until the previous kernel of the stream has completed and its writes are
// visible (returns at once when there is no such dependency).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launches `kernel` so that it may overlap the tail of the previous kernel in the
// stream (programmatic stream serialization); the kernel calls griddep_wait()
// before touching that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_after_previous(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---- numerics ----------------------------------------------------------------

// 2^x with the hardware approximation (PTX ex2.approx.ftz.f32); 2^-inf = 0.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float i8_at(uint32_t w, int k) {
  return static_cast<float>(static_cast<int8_t>((w >> (8 * k)) & 0xFF));
}

// 4-bit two's complement nibble k (0..7) of w: element 2i is the low nibble of byte i
__device__ __forceinline__ float i4_at(uint32_t w, int k) {
  int v = static_cast<int>((w >> (4 * k)) & 0xF);
  return static_cast<float>(v >= 8 ? v - 16 : v);
}

// bytes 2i and 2i+1 of w (E4M3 codes) as an fp16 pair, element 2i in the low
// half (every E4M3 value, NaN included, is exact in fp16)
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t w, int i) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
      static_cast<__nv_fp8x2_storage_t>((w >> (16 * i)) & 0xFFFFu), __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// E4M3 code k (0..3) of w as fp32
__device__ __forceinline__ float e4m3_at(uint32_t w, int k) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>((w >> (8 * k)) & 0xFFu),
                                               __NV_E4M3);
  return __half2float(__half(h));
}

constexpr float kLog2e = 1.4426950408889634f;

// Sets bits [lo, hi) of a 128-bit row mask held in four registers (every index
// is a compile-time constant, so the mask never leaves registers).
__device__ __forceinline__ void mask_set_range(uint32_t (&m)[4], int lo, int hi) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int a = max(lo, 32 * w), b = min(hi, 32 * w + 32);
    if (a < b) {
      const uint32_t n = static_cast<uint32_t>(b - a);
      const uint32_t bits = n >= 32u ? 0xFFFFFFFFu : ((1u << n) - 1u);
      m[w] |= bits << (a - 32 * w);
    }
  }
}

// Bit r (0..127) of a 128-bit row mask held in registers.
__device__ __forceinline__ bool mask_bit(const uint32_t (&m)[4], int r) {
  const uint32_t w = r < 32 ? m[0] : r < 64 ? m[1] : r < 96 ? m[2] : m[3];
  return (w >> (r & 31)) & 1u;
}

// ALiBi slope index and causal offset of query row vh (= qi * hq_real + h): the
// row is query qi of the last nq positions and sees tokens j <= n - 1 - offset.
__device__ __forceinline__ int row_head(const DecodeParams &p, int vh) { return vh % p.hq_real; }
__device__ __forceinline__ int row_offset(const DecodeParams &p, int vh) {
  return p.nq - 1 - vh / p.hq_real;
}

// Token j of a sequence of n tokens takes part in the softmax: every token, or
// with a window only the first `sink` tokens (attention sinks) and the last
// `window` tokens (the recent window).
__device__ __forceinline__ bool in_token_set(const DecodeParams &p, int n, int j) {
  return p.window <= 0 || j < p.sink || j >= n - p.window;
}

// Clears the rows of a tile (tokens t0 .. t0 + rows - 1) that fall between the
// sink tokens and the recent window.
__device__ __forceinline__ void mask_clear_gap(uint32_t (&m)[4], const DecodeParams &p, int n,
                                               int t0, int rows) {
  if (p.window <= 0) return;
  const int lo = max(p.sink - t0, 0), hi = min(n - p.window - t0, rows);
  if (lo >= hi) return;
  uint32_t gap[4] = {0u, 0u, 0u, 0u};
  mask_set_range(gap, lo, hi);
#pragma unroll
  for (int w = 0; w < 4; ++w) m[w] &= ~gap[w];
}

// Page ids and formats of a run of pages of one sequence, staged in shared
// memory by a producer warp so that resolving a tile reads no global memory.
template <int N>
struct PageCacheT {
  static constexpr int kEntries = N;
  int32_t id[N];
  uint8_t fmt[N];
  int seq, base, count;
};
constexpr int kPageCache = 128;
using PageCache = PageCacheT<kPageCache>;

// Called by all 32 lanes of one warp: makes pages [pg, pg_last] of sequence b
// available in the cache (pg_last - pg < N, pg_last < pg_end), refilling it from
// pg with one coalesced read of the page table (up to pg_end) when they are not
// all cached.
template <int N>
__device__ __forceinline__ void page_cache_ensure(PageCacheT<N> &pc, const DecodeParams &p, int b,
                                                  int pg, int pg_last, int pg_end, int lane) {
  __syncwarp();
  if (b == pc.seq && pg >= pc.base && pg_last < pc.base + pc.count) return;
  const int n = min(N, pg_end - pg);
  const long long row = static_cast<long long>(b) * p.max_pages + pg;
  for (int i = lane; i < n; i += 32) {
    pc.id[i] = p.page_table[row + i];
    pc.fmt[i] = p.page_fmt ? p.page_fmt[row + i] : static_cast<uint8_t>(p.uniform_fmt);
  }
  __syncwarp();
  if (lane == 0) {
    pc.seq = b;
    pc.base = pg;
    pc.count = n;
  }
  __syncwarp();
}

template <int N>
__device__ __forceinline__ void page_cache_reset(PageCacheT<N> &pc, int lane) {
  if (lane == 0) {
    pc.seq = -1;
    pc.base = 0;
    pc.count = 0;
  }
  __syncwarp();
}

// Number of splits of the schedule in the workspace, capped at the capacity of
// this call's split arrays.  The schedule launch of the same call never writes
// more; a larger (or negative) count can only come from a decode-only call on a
// workspace scheduled with other arguments, and sets CFR_DEVERR_SCHEDULE (when
// `report`) instead of letting the partial writes run past their arrays.
__device__ __forceinline__ int schedule_split_count(const DecodeParams &p, bool report) {
  const int s = p.num_splits[0];
  if (s >= 0 && s <= p.max_splits) return s;
  if (report) set_err(p.err, CFR_DEVERR_SCHEDULE);
  return s < 0 ? 0 : p.max_splits;
}

// Split `slot` of the schedule: sequence b and its page range [pb, pe).  An
// entry that is not a page range of this call's batch (again only possible on a
// workspace scheduled with other arguments) becomes an empty range of sequence 0
// and sets CFR_DEVERR_SCHEDULE, so no page-table row or sequence length outside
// the call's arrays is read.
struct SplitRange {
  int b, pb, pe;
};
__device__ __forceinline__ SplitRange split_at(const DecodeParams &p, int slot) {
  SplitRange r{p.splits[3 * slot], p.splits[3 * slot + 1], p.splits[3 * slot + 2]};
  if (r.b < 0 || r.b >= p.batch || r.pb < 0 || r.pe < r.pb || r.pe > p.max_units) {
    set_err(p.err, CFR_DEVERR_SCHEDULE);
    r.b = 0;
    r.pb = 0;
    r.pe = 0;
  }
  return r;
}

// Work item -> (split slot, row group).  Items are numbered split-fastest, so
// the CTAs that start together read different page slots of the pool rather
// than the kv heads of one slot (those sit a fixed sub-page stride apart).  When
// every kv head's rows form gsub > 1 groups (MQA, wide GQA), the gsub groups of
// one kv head and split are numbered next to each other, so the CTAs that take
// them read the same pages at about the same time and all but the first find
// them in L2.
__device__ __forceinline__ void item_coords(long long item, int nsplit, int gsub, int &slot, int &g) {
  if (gsub > 1) {
    const long long per = static_cast<long long>(nsplit) * gsub;  // items of one kv head
    const long long r = item % per;
    slot = static_cast<int>(r / gsub);
    g = static_cast<int>(item / per) * gsub + static_cast<int>(r % gsub);
  } else {
    slot = static_cast<int>(item % nsplit);
    g = static_cast<int>(item / nsplit);
  }
}

}  // namespace cfr
