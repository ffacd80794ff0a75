// cfr_decode_tc.cu -- paged decode attention on the 5th-generation tensor cores
// (tcgen05, accumulators in TMEM) for bf16, FP8 (E4M3), int8 and int4 K/V pages,
// head_dim 128.
//
// For a kv head serving G query rows (its query heads, times the queries per
// sequence in multi-query decode), one 128-token tile is two small dense
// contractions:
//   S^T[128 tok x N] = K_tile[128 x 128] . Q^T           (M = tokens, K = head_dim)
//   O^T[128 dim x N] = V_tile^T[128 x 128] . P^T          (M = head_dim, K = tokens)
// N = 16 (G <= 8) or 32 (G <= 16) columns: N/2 "hi" and N/2 "lo" columns, so that q
// (fp32 or bf16) and the probabilities p enter the 16-bit MMA as hi + lo pairs
// (about 16 significant bits for bf16, 22 for fp16), accumulated in fp32.
// bf16 pages run bf16 MMAs; FP8 pages are expanded to fp16 codes in shared
// memory (every E4M3 value is exact in fp16) and run fp16 MMAs.  int8 / int4
// pages take one of two routes:
//  - IMMA variants (at most 4 query rows per kv head): int8 MMAs (kind::i8,
//    int32 accumulators) on the codes themselves.  int8 tiles are loaded by TMA
//    straight into the operand layout; int4 codes are widened to one byte per
//    code (16 * code, exact).  The query enters as 4 signed digit columns per
//    head, q * 127 / max|q| = d0 + d1/128 + d2/128^2 + d3/128^3, and the
//    probabilities as 4 unsigned digit columns, p * 255 = e0 + e1/256 + e2/256^2
//    + e3/256^3; every int32 column sum stays below 2^23, so the fp32
//    recombination of the digit products loses only the usual fp32 rounding.
//  - otherwise the codes are expanded to fp16 in shared memory (exact) and run
//    fp16 MMAs like FP8 pages.
// Per-page K scales multiply the scores and V scales the tile's P.V result, in
// fp32 (ARGUS page, "Transient FP16 Reconstruction ... in GPU SRAM": pages are
// expanded on chip only).
//
// Warp roles (384 threads, one CTA per SM, persistent over work items =
// (split of a sequence, kv head)):
//   warps 0, 3  TMA producers, taking alternate tiles: resolve pages, bf16
//               tiles by 2-D tensor-map boxes straight into the 128-byte-swizzled
//               operand layout, int tiles by 1-D bulk copies of the raw rows.
//               Resolving and issuing a tile of many small pages is a serial
//               chain of dependent steps inside one warp, so two warps run two
//               such chains at once.
//   warp 1      TMEM allocation; lane 0 issues the QK products.
//   warp 2      lane 0 issues the P.V products (a thread of its own, so the two
//               kinds of MMA never wait for each other's issue).
//   warps 4-7   softmax / fold: thread t owns TMEM lane t = token t of S and
//               dim t of O.  Per tile: scores (scale, ALiBi from the integer
//               distance), tile max across the 128 tokens, p = 2^(s - m),
//               running normaliser, hi/lo split of p into the MMA's B operand,
//               and the exact fold acc = acc*2^(m_old-m_new) + O_tile of the
//               previous tile (CFR-Atlas page, "exact folded online-softmax
//               attention pass").
//   warps 8-11  staging: FP8/int8/int4 rows -> fp16 operand rows (int4 rows ->
//               int8 rows in IMMA variants); zeroes V rows of 16-bit tiles for
//               tokens that are not part of the input so stale or NaN bytes
//               never meet a zero probability inside the MMA (8-bit codes are
//               always finite, and meet an exact zero digit).
// Every mbarrier wait is bounded; on a timeout the error word is set, every
// role leaves its loop, the MMA pipe is drained and TMEM is freed.
//
// Three compile-time variants: plain decode; multi-query rows (per-row causal
// limits in the tiles that reach the query positions, and the row's ALiBi
// constant added to its maximum at the partial write); sink + recent-window
// subsets (gap rows cleared from the producer's row mask).  The roles share
// the SM's instruction cache, so code that is not on the current variant's
// path is kept out of it and loops off the critical path stay rolled.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstring>

#include "cfr_sched.cuh"
#include "cfr_tmap.cuh"

namespace cfr {

constexpr int TC_T = 128;            // tokens per tile
constexpr int TC_D = 128;            // head_dim of the operand layout (64 is read as its first half)
constexpr int TC_THREADS = 384;
// warp roles, one warpgroup each for the register split (setmaxnreg):
// warpgroup 0 = producers and MMA issuers, 1 = softmax, 2 = staging
constexpr int TC_PRODUCERS = 2;      // producer warps 0 and TC_PROD2_WARP, alternate tiles
constexpr int TC_PROD2_WARP = 3;
constexpr int TC_QK_WARP = 1;
constexpr int TC_PV_WARP = 2;
constexpr int TC_SOFTMAX_T0 = 128;   // first thread of the softmax warpgroup (warps 4-7)
constexpr int TC_STAGING_T0 = 256;   // first thread of the staging warpgroup (warps 8-11)
// registers per thread of each warpgroup after the split; the launch gives
// 384 x 168 = 64,512 and the split takes 128 x (104 + 224 + 152) = 61,440
constexpr int TC_REGS_IO = 104, TC_REGS_SOFTMAX = 224, TC_REGS_STAGING = 152;
constexpr int TC_REGS_STAGING_IMMA = 136;
// registers per thread at launch: the register file (65,536) over the block's
// threads, rounded down to the allocation unit of 8 (what __launch_bounds__ with
// one block per SM gives ptxas); the launch checks the kernel really has it
constexpr int TC_REGS_LAUNCH = 65536 / TC_THREADS / 8 * 8;
static_assert(128 * (TC_REGS_IO + TC_REGS_SOFTMAX + TC_REGS_STAGING) <= TC_REGS_LAUNCH * TC_THREADS,
              "the split must fit the registers the block was launched with");

// move this warpgroup's register count to N: setmaxnreg.dec below the launch
// count, .inc above it (a decrease must not name a larger count)
template <int N>
__device__ __forceinline__ void tc_setmaxnreg() {
  static_assert(N % 8 == 0 && N >= 24 && N <= 256, "setmaxnreg count");
  if constexpr (N < TC_REGS_LAUNCH)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
  else if constexpr (N > TC_REGS_LAUNCH)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
// work items reach the CTA's warps through a ring of this many slots; every
// slot is read by producer warp 3, the two MMA issuers and one thread of each of
// the softmax and staging warpgroups
constexpr int TC_ITEM_RING = 4;
constexpr int TC_ITEM_READERS = 5;
constexpr int TC_HALF = TC_T * 128;  // bytes of one 64-column half of a K or V tile
constexpr int TC_OP_BYTES = 4 * TC_HALF;  // K (2 halves) + V (2 halves) = 64 KiB
constexpr int TC_RAW_K = TC_T * TC_D;  // raw code offset of V inside a stage's V region (K at 0)

constexpr int KIND_BF16 = 0, KIND_I8 = 1, KIND_I4 = 2, KIND_FP8 = 3;
// compile-time variants: plain decode, multi-query rows, sink + window subset
constexpr int TC_FEAT_PLAIN = 0, TC_FEAT_MULTI = 1, TC_FEAT_SUBSET = 2;
// OR'ed into the feature: quantised pages shorter than a tile in a uniform-format
// cache (a tile holds several pages, each with its own scales); its own
// instantiations, so that the variants for larger pages carry none of it
constexpr int TC_FEAT_SMALL_PAGES = 4;
// OR'ed into the feature of int8-MMA variants: a uniform int8 cache, whose tiles
// (int8 codes only: 16 KiB of K and 16 KiB of V) fit six 32 KiB stages
constexpr int TC_FEAT_COMPACT_I8 = 8;
__host__ __device__ constexpr int tc_feat(int feat) { return feat & 3; }

// one work item as producer warp 0 publishes it (see tc_publish_item)
struct TcItem {
  int item;        // -1: past the CTA's last item, or a wait gave up
  int slot, g, b;  // split slot, kv head, sequence
  int tb, pg_end;  // the split's first token; the end of its logical pages
  int n, t_end;    // sequence length; the split's tokens are [tb, t_end)
};

template <int NP>
struct TcMetaT {
  uint32_t valid[4];
  int rows, t0, kind, direct;
  // quantised tiles: the K scale of each page piece (one piece when pages hold
  // 128 tokens or more; up to NP = 16 pieces of a uniform-format cache with
  // smaller pages in the 16-column variants), vs, the largest V scale, which the
  // fold applies to the tile's product, and vsp, each piece's V scale over vs,
  // which its rows' probabilities carry
  float vs;
  float ksp[NP], vsp[NP];
};

struct TcMaps {
  CUtensorMap k;   // bf16 pool
  CUtensorMap v;
  CUtensorMap k8;  // int8 pool (tiles loaded straight into the 8-bit operand layout)
  CUtensorMap v8;
};

template <int NCOL, bool INTP>
struct TcCfg {
  // quantised codes are copied into the stage's own V region and expanded in
  // place, so the variant with quantised pools keeps the same three stages of
  // 64 KiB; with head_dim 64 the 16-column variants cut the same bytes into six
  // stages of 32 KiB (K half, V half), twice the tiles in flight
  static constexpr int STAGES = 3;
  static constexpr int MAX_STAGES = NCOL == 16 ? 6 : 3;
  static constexpr int Q_BYTES = NCOL * 256;       // [NCOL rows][128 cols] 16-bit, 2 halves
  // [NCOL rows][128 cols] int8 query digits (int8 MMAs, 16 columns only)
  static constexpr int Q8_BYTES = (INTP && NCOL == 16) ? NCOL * 128 : 0;
  // one query operand buffer: bf16 hi/lo rows, then (quantised pools) fp16 hi/lo
  // rows and int8 digit rows
  static constexpr int QSTRIDE = INTP ? 2 * Q_BYTES + Q8_BYTES : Q_BYTES;
  static constexpr int P_BYTES = NCOL * TC_T * 2;  // [128 tokens][NCOL] 16-bit
  static constexpr int O_BUFS = 3;                 // O accumulators in flight (fold lags two tiles)
  static constexpr int TMEM_COLS = NCOL == 16 ? 128 : 256;  // S x2 + O x3 columns, power of two
  // page-table entries each producer keeps on chip; with 32 columns the q and P
  // buffers leave room for two caches of 48 beside the three stages (with
  // 16-token pages, one refill then serves 6 tiles)
  static constexpr int PAGE_CACHE = NCOL == 16 ? 128 : 48;
  // the 16-column variants keep each item's ALiBi slopes in shared memory (the
  // 32-column ones, which fill shared memory, read them at the item's start)
  static constexpr int RING_SLOPES = NCOL == 16 ? NCOL / 2 : 1;
  using PageCache = PageCacheT<PAGE_CACHE>;
};

template <int NCOL, bool INTP>
struct TcSmem {
  uint64_t op_full[TcCfg<NCOL, INTP>::MAX_STAGES], op_empty[TcCfg<NCOL, INTP>::MAX_STAGES],
      raw_full[TcCfg<NCOL, INTP>::MAX_STAGES];
  uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2];
  uint64_t o_full[TcCfg<NCOL, INTP>::O_BUFS], o_empty[TcCfg<NCOL, INTP>::O_BUFS];
  uint64_t q_full, drain;
  uint64_t item_full[TC_ITEM_RING], item_empty[TC_ITEM_RING];
  uint64_t qbuf_full[2], qbuf_empty[2];  // query operand buffers (16-column variants)
  TcItem ring[TC_ITEM_RING];  // work item k in slot k % TC_ITEM_RING
  // ALiBi slope * log2(e) of its query rows (16-column variants)
  float ring_slope[TC_ITEM_RING][TcCfg<NCOL, INTP>::RING_SLOPES];
  TcItem item_bc[2][2];       // [softmax, staging][k & 1]: the item in a warpgroup
  float slope_bc[2][TcCfg<NCOL, INTP>::RING_SLOPES];  // [k & 1]: its slopes, for the softmax
  // int8 digit scales of its query rows (16-column variants), and their copy for the softmax
  float ring_qs[TC_ITEM_RING][TcCfg<NCOL, INTP>::RING_SLOPES >= 4 ? 4 : 1];
  float qs_bc[2][TcCfg<NCOL, INTP>::RING_SLOPES >= 4 ? 4 : 1];
  uint32_t tmem_base;
  int flag_st[TcCfg<NCOL, INTP>::MAX_STAGES];
  // tile descriptions; the 32-column variants, which fill shared memory, take
  // quantised pages of 128 tokens or more only (one piece)
  TcMetaT<NCOL == 16 ? 16 : 1> meta[TcCfg<NCOL, INTP>::MAX_STAGES];
  alignas(16) float red_max[2][4][16];
  alignas(16) float red_l[4][16];
  typename TcCfg<NCOL, INTP>::PageCache pc[TC_PRODUCERS];
};

template <int NCOL, bool INTP>
struct TcLayout {
  static constexpr size_t head = (sizeof(TcSmem<NCOL, INTP>) + 1023) / 1024 * 1024;
  static constexpr size_t op = head;
  static constexpr size_t q = op + TcCfg<NCOL, INTP>::STAGES * static_cast<size_t>(TC_OP_BYTES);
  // query operand buffers: one (32 columns, written by the softmax warpgroup) or
  // two (16 columns, images copied by producer warp 0), QSTRIDE bytes apart
  static constexpr size_t q8 = q + 2 * static_cast<size_t>(TcCfg<NCOL, INTP>::Q_BYTES);
  static constexpr size_t pbuf = q + (NCOL == 16 ? 2 : 1) * static_cast<size_t>(TcCfg<NCOL, INTP>::QSTRIDE);
  static constexpr size_t total = pbuf + 2 * static_cast<size_t>(TcCfg<NCOL, INTP>::P_BYTES);
  static constexpr size_t launch_bytes = total + 1024;  // slack for 1024-byte alignment
};

// ---- tcgen05 / descriptor helpers -------------------------------------------

// instruction descriptor, kind::f16, fp32 accumulator, M = 128
__host__ __device__ constexpr uint32_t tc_idesc(int ab_bf16, int a_mn, int b_mn, int n) {
  return (1u << 4) | (static_cast<uint32_t>(ab_bf16) << 7) | (static_cast<uint32_t>(ab_bf16) << 10) |
         (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// instruction descriptor, kind::i8, s32 accumulator, M = 128: A signed 8-bit
// codes, B signed (query digits) or unsigned (probability digits) 8-bit
__host__ __device__ constexpr uint32_t tc_idesc_i8(int b_signed, int a_mn, int b_mn, int n) {
  return (2u << 4) | (1u << 7) | (static_cast<uint32_t>(b_signed) << 10) |
         (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// shared-memory matrix descriptor (sm_100: version 1); layout 2 = 128-byte swizzle, 0 = none
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                             uint32_t layout) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         (static_cast<uint64_t>(layout) << 61);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[N]);

template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15},"
      " [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, float (&v)[32]) {
  float a[16], b[16];
  tmem_ld<16>(taddr, a);
  tmem_ld<16>(taddr + 16, b);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v[i] = a[i];
    v[16 + i] = b[i];
  }
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// four int8 codes (one word) -> two half2 words holding the same integers
__device__ __forceinline__ void i8x4_to_h2x2(uint32_t w, uint32_t &a, uint32_t &b) {
  const uint32_t u = w ^ 0x80808080u;                         // code + 128, unsigned
  const __half2 bias = bits_h2(0x64806480u);                   // 1152 = 1024 + 128
  a = h2_bits(__hsub2(bits_h2(prmt(u, 0x64646464u, 0x4140u)), bias));  // 1024 + u0, 1024 + u1
  b = h2_bits(__hsub2(bits_h2(prmt(u, 0x64646464u, 0x4342u)), bias));
}

// one byte k (0..3) of a word of int4 codes (low nibble = even element) -> half2
__device__ __forceinline__ uint32_t i4x2_to_h2(uint32_t u_biased, int k) {
  const uint32_t t = prmt(u_biased, 0u, 0x4040u | static_cast<uint32_t>(k) | (static_cast<uint32_t>(k) << 8));
  const uint32_t m = (t & 0x00F0000Fu) | 0x64006400u;  // 1024 + lo nibble, 1024 + 16 * hi nibble
  const __half2 scale = __halves2half2(__float2half_rn(1.f), __float2half_rn(0.0625f));
  const __half2 off = __halves2half2(__float2half_rn(-1032.f), __float2half_rn(-72.f));
  return h2_bits(__hfma2(bits_h2(m), scale, off));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// ---- roles ------------------------------------------------------------------

template <int NCOL, bool INTP, int FEAT, bool IMMA>
struct TcCtx {
  const DecodeParams &p;
  const TcMaps &maps;
  TcSmem<NCOL, INTP> &S;
  uint8_t *op, *qop, *pop;
  long long nitems;
  int nsplit;
  // six stages of 32 KiB (K, V) instead of three of 64 KiB: head_dim 64 in a
  // 16-column variant other than int8-MMA (compact, set at run time), and the
  // int8-MMA variants of uniform int8 caches (always)
  bool compact;
  // stage geometry: nst() stages of sbytes() bytes; the V operand (and the raw
  // codes of quantised tiles) at voff() in a stage, the raw V codes rawv() bytes
  // after the raw K codes.  Compile-time constants where the choice is.
  static constexpr bool kMayCompact = NCOL == 16 && !IMMA;
  static constexpr bool kAlwaysCompact = IMMA && (FEAT & TC_FEAT_COMPACT_I8) != 0;
  __device__ __forceinline__ bool is_compact() const { return kAlwaysCompact || (kMayCompact && compact); }
  __device__ __forceinline__ int nst() const {
    return is_compact() ? 2 * TcCfg<NCOL, INTP>::STAGES : TcCfg<NCOL, INTP>::STAGES;
  }
  __device__ __forceinline__ int sbytes() const { return is_compact() ? TC_OP_BYTES / 2 : TC_OP_BYTES; }
  __device__ __forceinline__ int voff() const { return is_compact() ? TC_HALF : 2 * TC_HALF; }
  __device__ __forceinline__ int rawv() const { return is_compact() ? TC_RAW_K / 2 : TC_RAW_K; }
};

// query rows one tile holds: 4 in IMMA variants (their int8 digit columns are 4
// digits x 4 rows), else NCOL / 2 (hi + lo columns per row)
template <int NCOL, bool IMMA>
__host__ __device__ constexpr int tc_rows() {
  return IMMA ? 4 : NCOL / 2;
}

// an int32 value |x| < 2^22 as fp32, exactly, with two full-rate operations:
// 1.5 * 2^23 + x has x in its low mantissa bits
__device__ __forceinline__ float small_i2f(float bits) {
  return __int_as_float(__float_as_int(bits) + 0x4B400000) - 12582912.f;
}

// With IMMA, int8 and int4 tiles run kind::i8 MMAs on 8-bit operands: int8 codes
// as stored, int4 codes widened to bytes (times 16, so that the sign needs no
// extension), query and probability as base-128 / base-256 digit columns.
template <bool IMMA>
__device__ __forceinline__ bool tc_int_tile(int kind) {
  return IMMA && (kind == KIND_I8 || kind == KIND_I4);
}


// Maximum over the 32 lanes of each of NV values per lane (NV a power of two,
// NV <= 16), by a transposing reduction: each exchange step halves the values a
// lane keeps, so the warp spends NV-1 + log2(32/NV) shuffles instead of 5*NV.
// Returns the maximum of value `head` (written to *head); lanes whose low bits
// below the last halving offset are zero hold distinct heads.
template <int NV>
__device__ __forceinline__ float warp_multi_max(const float (&v)[NV], int lane, int *head) {
  float cur[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) cur[i] = v[i];
  int h = 0;
  int off = 16;
#pragma unroll
  for (int n = NV; n > 1; n >>= 1) {
    const int half = n >> 1;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? cur[i] : cur[half + i];
      const float keep = upper ? cur[half + i] : cur[i];
      cur[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
    }
    h = 2 * h + (upper ? 1 : 0);
    off >>= 1;
  }
  float r = cur[0];
#pragma unroll
  for (int o = off; o > 0; o >>= 1) r = fmaxf(r, __shfl_xor_sync(0xffffffffu, r, o));
  *head = h;
  return r;
}

// non-blocking probe of an mbarrier phase
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// ---- work items --------------------------------------------------------------
// An item is one split of one kv head.  Producer warp 0 takes the CTA's items in
// order and publishes item k in ring slot k % TC_ITEM_RING together with what
// every other role needs to know about it (split, sequence length, token range,
// the ALiBi slopes of its query rows), so that no other role reads global
// memory at an item boundary; a slot whose item is -1 ends every loop.  In the
// 16-column variants warp 0 also bulk-copies the query operand image of the
// item's (sequence, kv head) -- built once per decode by tc_qimage_kernel --
// into query buffer kq & 1 (kq counting the items with tiles), so that no role
// builds query operands inside the pipeline.  Two ways of choosing the items,
// by measurement:
//  - fixed: CTA x takes items x, x + grid, x + 2 grid, ...
//  - claimed (plain, multi-query and sink + window decode over bf16 pools, or
//    over int8 / int4 pools of one format in the IMMA variants): CTA x starts with item x and
//    claims every further item from a global counter when producer warp 0
//    reaches it, so SMs that the memory system serves faster take more items and
//    all CTAs finish together.  Over pools of mixed formats the items differ in
//    cost several-fold and the fixed share measured faster; the host then passes
//    no counter (item_ctr = null), which selects the fixed share.
template <bool INTP, int FEAT, bool IMMA>
__host__ __device__ constexpr bool tc_claimed_items() {
  return !INTP || IMMA;
}

// quantised pages shorter than a tile (several pages, each with its scales, in
// one tile): the small-page instantiations of the 16-column variants with
// quantised pools
template <int NCOL, bool INTP, int FEAT>
__host__ __device__ constexpr bool tc_pieces() {
  return NCOL == 16 && INTP && (FEAT & TC_FEAT_SMALL_PAGES) != 0;
}

// query operands as prebuilt images, double-buffered (16-column variants)
template <int NCOL>
__host__ __device__ constexpr bool tc_qimg() {
  return NCOL == 16;
}

// producer warp 0 (all lanes): takes item k, publishes it and (16-column
// variants) starts the copy of its query operand image into query buffer kq & 1,
// kq counting the items with tiles.  Returns the item (item = -1 past the last,
// or when a wait gave up).
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ __forceinline__ TcItem tc_publish_item(TcCtx<NCOL, INTP, FEAT, IMMA> &c, int k, int &kq,
                                                  bool *timed_out, int lane) {
  const DecodeParams &p = c.p;
  const int s = k & (TC_ITEM_RING - 1);
  TcItem d;
  d.item = -1;
  d.slot = d.g = d.b = d.tb = d.pg_end = d.n = d.t_end = 0;
  int ok = 1;
  if (lane == 0)
    ok = mbar_wait(&c.S.item_empty[s], static_cast<uint32_t>((k / TC_ITEM_RING) & 1) ^ 1u, p.err,
                   timed_out) ? 1 : 0;
  if (!__shfl_sync(0xffffffffu, ok, 0)) return d;
  long long it = 0;
  if (lane == 0)
    it = k == 0 ? static_cast<long long>(blockIdx.x)
         : (tc_claimed_items<INTP, FEAT, IMMA>() && p.item_ctr)
             ? static_cast<long long>(gridDim.x) + atomicAdd(p.item_ctr, 1u)
             : static_cast<long long>(blockIdx.x) + static_cast<long long>(k) * gridDim.x;
  it = __shfl_sync(0xffffffffu, it, 0);
  if (it < c.nitems) {
    d.item = static_cast<int>(it);
    item_coords(it, c.nsplit, p.gsub, d.slot, d.g);
    const SplitRange sr = split_at(p, d.slot);
    d.b = sr.b;
    // the split's range of schedule units, in tokens and in pages
    d.tb = sr.pb * p.split_unit;
    d.pg_end = p.split_unit == p.P ? sr.pe : (sr.pe * p.split_unit + p.P - 1) / p.P;
    d.n = p.seq_lens[d.b];
    d.t_end = min(d.n, sr.pe * p.split_unit);
    const int h0 = p.grp_off[d.g], cnt = p.grp_off[d.g + 1] - h0;
    if (tc_qimg<NCOL>() && lane < NCOL / 2)
      c.S.ring_slope[s][lane] =
          (p.slopes && lane < cnt) ? p.slopes[row_head(p, p.grp_heads[h0 + lane])] * kLog2e : 0.f;
    if (tc_qimg<NCOL>() && d.tb < d.t_end) {
      const int buf = kq & 1;
      const long long grp = static_cast<long long>(d.b) * p.ngroups + d.g;
      constexpr uint32_t bytes = static_cast<uint32_t>(TcCfg<NCOL, INTP>::QSTRIDE);
      int qok = 1;
      if (lane == 0) {
        qok = mbar_wait(&c.S.qbuf_empty[buf], static_cast<uint32_t>((kq >> 1) & 1) ^ 1u, p.err,
                        timed_out) ? 1 : 0;
        if (qok) {
          mbar_arrive_expect_tx(&c.S.qbuf_full[buf], bytes);
          bulk_g2s(c.qop + buf * TcCfg<NCOL, INTP>::QSTRIDE, p.qimg + grp * kQImgBytes, bytes,
                   &c.S.qbuf_full[buf]);
        }
      }
      if (lane < 4) c.S.ring_qs[s][lane & (TcCfg<NCOL, INTP>::RING_SLOPES >= 4 ? 3 : 0)] = p.qscale[grp * 4 + lane];
      if (!__shfl_sync(0xffffffffu, qok, 0)) d.item = -1;
      ++kq;
    }
  }
  if (lane == 0) c.S.ring[s] = d;
  __syncwarp();
  if (lane == 0) mbar_arrive(&c.S.item_full[s]);
  return d;
}

// item k read by one thread (an MMA issuer) or by every lane of a warp
// (producer warp 3: lane 0 waits, reads and frees the slot, the lanes get the
// fields by shuffles).  item = -1 past the last item or when the wait gave up.
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ __forceinline__ TcItem tc_read_item(TcCtx<NCOL, INTP, FEAT, IMMA> &c, int k, bool *timed_out,
                                               bool warp_wide) {
  const int s = k & (TC_ITEM_RING - 1);
  TcItem d;
  d.item = -1;
  d.slot = d.g = d.b = d.tb = d.pg_end = d.n = d.t_end = 0;
  if (!warp_wide || (threadIdx.x & 31) == 0) {
    if (mbar_wait(&c.S.item_full[s], static_cast<uint32_t>((k / TC_ITEM_RING) & 1), c.p.err,
                  timed_out)) {
      d = c.S.ring[s];
      mbar_arrive(&c.S.item_empty[s]);
    }
  }
  if (warp_wide) {
    d.item = __shfl_sync(0xffffffffu, d.item, 0);
    d.slot = __shfl_sync(0xffffffffu, d.slot, 0);
    d.g = __shfl_sync(0xffffffffu, d.g, 0);
    d.b = __shfl_sync(0xffffffffu, d.b, 0);
    d.tb = __shfl_sync(0xffffffffu, d.tb, 0);
    d.pg_end = __shfl_sync(0xffffffffu, d.pg_end, 0);
    d.n = __shfl_sync(0xffffffffu, d.n, 0);
    d.t_end = __shfl_sync(0xffffffffu, d.t_end, 0);
  }
  return d;
}

// item k read by a 128-thread warpgroup that synchronises on named barrier
// `bar` (2: softmax, 3: staging): thread t = 0 waits, copies the slot (and the
// ALiBi slopes) to the warpgroup's broadcast area and frees it; the barrier
// hands the copy to all 128 threads, so they leave their loop together even when
// the wait gave up (named barriers have no time limit).
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ __forceinline__ TcItem tc_read_item_wg(TcCtx<NCOL, INTP, FEAT, IMMA> &c, int k, int bar, int t,
                                                  bool *timed_out) {
  TcItem *bc = &c.S.item_bc[bar - 2][k & 1];
  if (t == 0) {
    const int s = k & (TC_ITEM_RING - 1);
    TcItem d;
    d.item = -1;
    d.slot = d.g = d.b = d.tb = d.pg_end = d.n = d.t_end = 0;
    if (mbar_wait(&c.S.item_full[s], static_cast<uint32_t>((k / TC_ITEM_RING) & 1), c.p.err,
                  timed_out)) {
      d = c.S.ring[s];
      if (tc_qimg<NCOL>() && bar == 2) {
#pragma unroll
        for (int h = 0; h < TcCfg<NCOL, INTP>::RING_SLOPES; ++h)
          c.S.slope_bc[k & 1][h] = c.S.ring_slope[s][h];
#pragma unroll
        for (int h = 0; h < (TcCfg<NCOL, INTP>::RING_SLOPES >= 4 ? 4 : 1); ++h)
          c.S.qs_bc[k & 1][h] = c.S.ring_qs[s][h];
      }
      mbar_arrive(&c.S.item_empty[s]);
    }
    *bc = d;
  }
  named_sync(bar, 128);
  return *const_cast<const TcItem *>(bc);
}

// Per-kernel constants of a producer warp: which formats have their pools (and
// scales) and the geometry of a tile's copy boxes.
struct TcProdGeom {
  uint32_t fmt_ok;  // bit f: format f can be read on this path
  int box_rows;     // rows of one copy box: min(P, 128); a power of two
  int box_shift;    // log2(box_rows)
};

// one tile of a producer warp.  Everything that does not need the stage --
// page resolution (lane f resolves page piece f, so a tile made of many small
// pages is resolved in parallel), the row mask (one ballot per 32 rows), scales,
// byte count -- is done first; then lane 0 waits for the stage, and the moment
// it is free lane 0 publishes the tile description and the expected byte count
// while every lane issues its own copies.  The tile starts at row tin0 of
// logical page pg0 (tin0 = 0 when pages are shorter than a tile).
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ __forceinline__ bool tc_produce_tile(TcCtx<NCOL, INTP, FEAT, IMMA> &c,
                                                const typename TcCfg<NCOL, INTP>::PageCache &pc,
                                                const TcProdGeom &geo, int b, int g, int n,
                                                int t0, int rows, int npiece, int pg0, int tin0,
                                                int stage, uint32_t phase, bool *timed_out,
                                                int lane) {
  const DecodeParams &p = c.p;
  const int box_rows = geo.box_rows;
  // ---- resolve piece `lane` ----
  bool pvalid = false;
  int fmt = -1;
  long long id = 0;
  if (lane < npiece) {
    fmt = pc.fmt[pg0 + lane - pc.base];
    id = pc.id[pg0 + lane - pc.base];
    long long lim = 0;
#pragma unroll
    for (int f = 0; f < kFmtCount; ++f)
      if (f == fmt) lim = p.pool_pages[f];
    if (fmt >= kFmtCount) {
      set_err(p.err, CFR_DEVERR_PAGE_FMT);
    } else if (((geo.fmt_ok >> fmt) & 1u) == 0u) {
      set_err(p.err, CFR_DEVERR_POOL);
    } else if (id < 0 || id >= lim) {
      set_err(p.err, CFR_DEVERR_PAGE_ID);
    } else {
      pvalid = true;
    }
  }
  const uint32_t vb = __ballot_sync(0xffffffffu, pvalid);
  // rows of valid pieces that hold tokens, 32 rows per ballot (every lane gets the mask)
  uint32_t valid[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int row = 32 * w + lane;
    valid[w] = __ballot_sync(0xffffffffu, row < rows && ((vb >> (row >> geo.box_shift)) & 1u));
  }
  if constexpr (tc_feat(FEAT) == TC_FEAT_SUBSET)
    mask_clear_gap(valid, p, n, t0, rows);  // tokens between the sinks and the recent window
  // the tile's kind is the format of its first valid piece: a cache whose page
  // formats differ has quantised pages of 128 tokens or more (one piece per
  // tile), and a uniform-format cache gives every piece the same format
  const int kind0 = !pvalid                ? KIND_BF16
                    : fmt == CFR_FMT_I8    ? KIND_I8
                    : fmt == CFR_FMT_I4    ? KIND_I4
                    : fmt == CFR_FMT_FP8   ? KIND_FP8
                                           : KIND_BF16;
  // (a tile with no valid piece in a uniform int8 cache keeps the int8 kind: its
  // stage has no room for a bf16 V, and its stale int8 codes meet zero
  // probabilities)
  const int kind = !vb && TcCtx<NCOL, INTP, FEAT, IMMA>::kAlwaysCompact
                       ? KIND_I8
                       : __shfl_sync(0xffffffffu, kind0, vb ? __ffs(vb) - 1 : 0);
  // a bf16 tile whose 128 rows all hold tokens goes straight to the MMA, and so
  // does every int8 tile of an IMMA variant (its codes are the operand; rows
  // that hold no token carry finite codes that meet a zero probability); every
  // other tile passes through the staging warps
  const bool direct = (kind == KIND_BF16 && (valid[0] & valid[1] & valid[2] & valid[3]) == 0xFFFFFFFFu) ||
                      (IMMA && kind == KIND_I8);
  // ---- the tile's byte count (lane 0) and, for quantised tiles, its pieces'
  // scales (lane f: piece f) and their largest V scale ----
  float ks = 1.f, vs = 1.f, vs_max = 1.f;
  constexpr bool pieces = tc_pieces<NCOL, INTP, FEAT>();
  if (!pieces) {
    // one piece per quantised tile (pages of 128 tokens or more): lane 0's scales
    if (lane == 0 && kind != KIND_BF16 && pvalid) {
      const float2 sc = *reinterpret_cast<const float2 *>(p.scales[fmt] + (id * p.Hkv + p.grp_kv[g]) * 2);
      ks = sc.x;
      vs = vs_max = sc.y;
    }
  } else if (kind != KIND_BF16) {  // the same in every lane
    if (pvalid) {
      const float2 sc = *reinterpret_cast<const float2 *>(p.scales[fmt] + (id * p.Hkv + p.grp_kv[g]) * 2);
      ks = sc.x;
      vs = sc.y;
    }
    vs_max = pvalid ? vs : 0.f;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) vs_max = fmaxf(vs_max, __shfl_xor_sync(0xffffffffu, vs_max, o));
    vs_max = __shfl_sync(0xffffffffu, vs_max, 0);
  }
  uint32_t bytes = 0;
  if (lane == 0) {
    if (kind == KIND_BF16) {
      // a K and a V box per 64 dims (2 with head_dim 64, 4 with 128) per valid piece
      bytes = static_cast<uint32_t>(__popc(vb)) * ((IMMA || p.D == TC_D) ? 4u : 2u) * box_rows * 128u;
    } else if (IMMA && kind == KIND_I8) {
      // a full box of K and of V per valid piece (one 128-row box with pages of
      // 128 tokens or more)
      bytes = static_cast<uint32_t>(__popc(vb)) * 2u * box_rows * 128u;
    } else if (p.P >= TC_T) {
      bytes = 2u * rows * static_cast<uint32_t>(row_bytes(fmt, p.D));  // the tile's rows of one page
    } else {
      // whole pieces of box_rows rows (a uniform format: every piece's row bytes)
      bytes = static_cast<uint32_t>(__popc(vb)) * 2u * box_rows * static_cast<uint32_t>(row_bytes(fmt, p.D));
    }
  }
  uint64_t *done = direct ? &c.S.op_full[stage] : &c.S.raw_full[stage];
  // ---- wait for the stage ----
  int ok = 1;
  if (lane == 0) ok = mbar_wait(&c.S.op_empty[stage], phase ^ 1u, p.err, timed_out) ? 1 : 0;
  if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
  if (lane == 0) {
    auto &m = c.S.meta[stage];
    for (int w = 0; w < 4; ++w) m.valid[w] = valid[w];
    m.rows = rows;
    m.t0 = t0;
    m.kind = kind;
    m.direct = direct ? 1 : 0;
    m.vs = vs_max;
  }
  if constexpr (pieces) {
    if (kind != KIND_BF16 && lane < 16) {
      c.S.meta[stage].ksp[lane] = ks;
      c.S.meta[stage].vsp[lane] = vs_max > 0.f ? vs / vs_max : 1.f;
    }
    __syncwarp();  // the whole description is written before lane 0 publishes it
  } else if (lane == 0) {
    c.S.meta[stage].ksp[0] = ks;
  }
  if (lane == 0) {
    if (direct) mbar_arrive(&c.S.raw_full[stage]);  // lets the staging warps skip this tile
    mbar_arrive_expect_tx(done, bytes);
  }
  __syncwarp();
  if (pvalid) {
    const int r = lane * box_rows;
    uint8_t *op = c.op + static_cast<size_t>(stage) * c.sbytes();
    if (kind == KIND_BF16) {
      const int y = static_cast<int>((id * p.Hkv + p.grp_kv[g]) * p.P + tin0);
      // head_dim 64 fills only the first half of K and of V: the QK products
      // stop at dim 64 and the P.V rows of dims 64..127 are never read
      tma_load_2d(op + 0 * TC_HALF + r * 128, &c.maps.k, 0, y, done);
      if (IMMA || p.D == TC_D) tma_load_2d(op + 1 * TC_HALF + r * 128, &c.maps.k, 64, y, done);
      tma_load_2d(op + c.voff() + r * 128, &c.maps.v, 0, y, done);
      if (IMMA || p.D == TC_D) tma_load_2d(op + 3 * TC_HALF + r * 128, &c.maps.v, 64, y, done);
    } else if (IMMA && kind == KIND_I8) {
      // K codes at 0, V codes at 2 * TC_HALF, 128-byte swizzled rows; piece
      // `lane` at row r (boxes of min(P, 128) rows)
      const int y = static_cast<int>((id * p.Hkv + p.grp_kv[g]) * p.P + tin0);
      tma_load_2d(op + r * 128, &c.maps.k8, 0, y, done);
      tma_load_2d(op + c.voff() + r * 128, &c.maps.v8, 0, y, done);
    } else if (IMMA && kind == KIND_I4) {
      // raw codes above the int8 operands the staging warps write (K at TC_HALF,
      // V at 3 * TC_HALF), piece `lane` at row r
      const int rb = row_bytes(fmt, TC_D);
      const long long off = ((id * p.Hkv + p.grp_kv[g]) * p.P + tin0) * rb;
      const int nrows = p.P >= TC_T ? rows : box_rows;
      bulk_g2s(op + TC_HALF + r * rb, p.k_pool[fmt] + off, nrows * rb, done);
      bulk_g2s(op + 3 * TC_HALF + r * rb, p.v_pool[fmt] + off, nrows * rb, done);
    } else if (INTP) {
      const int rb = row_bytes(fmt, p.D);
      const long long off = ((id * p.Hkv + p.grp_kv[g]) * p.P + tin0) * rb;
      // codes go to the stage's V region (K codes first, V codes rawv bytes in),
      // piece `lane` at row r; the staging warps expand them in place
      const int nrows = p.P >= TC_T ? rows : box_rows;
      uint8_t *raw = op + c.voff() + r * rb;
      bulk_g2s(raw, p.k_pool[fmt] + off, nrows * rb, done);
      bulk_g2s(raw + c.rawv(), p.v_pool[fmt] + off, nrows * rb, done);
    }
  }
  return true;
}

// Producer warp `pk` (0 or 1): walks every tile of the CTA's items in order and
// produces tiles pk, pk + 2, pk + 4, ...; warp 0 also claims the items.  Two producers never hold one stage at a
// time: tile i waits for the consumers of tile i - 3 (the same stage), and the
// warp's previous tile i - 2 waited for tile i - 5, so the stage's barrier can
// never be two phases behind when tile i starts waiting on it.
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ void tc_producer(TcCtx<NCOL, INTP, FEAT, IMMA> &c, bool *timed_out, int pk) {
  using Cfg = TcCfg<NCOL, INTP>;
  const DecodeParams &p = c.p;
  const int P = p.P;
  const int lane = threadIdx.x & 31;
  typename Cfg::PageCache &pc = c.S.pc[pk];
  TcProdGeom geo;
  geo.fmt_ok = 0u;
#pragma unroll
  for (int f = 0; f < kFmtCount; ++f)
    if (f != CFR_FMT_F32 && p.k_pool[f] && (!is_quantised(f) || p.scales[f])) geo.fmt_ok |= 1u << f;
  // the path takes P a power of two dividing 128, or a multiple of 128
  geo.box_rows = P < TC_T ? P : TC_T;
  geo.box_shift = 31 - __clz(geo.box_rows);
  const int pages_per_tile = P < TC_T ? TC_T / P : 0;
  int stage = 0;
  uint32_t phase = 0;
  if (lane == 0 && p.k_pool[CFR_FMT_BF16]) {
    prefetch_map(&c.maps.k);
    prefetch_map(&c.maps.v);
  }
  if (IMMA && lane == 0 && p.k_pool[CFR_FMT_I8]) {
    prefetch_map(&c.maps.k8);
    prefetch_map(&c.maps.v8);
  }
  page_cache_reset(pc, lane);
  long long tile = 0;
  int kq = 0;  // items with tiles so far (query-row buffers)
  for (int k = 0;; ++k) {
    const TcItem it = pk == 0 ? tc_publish_item(c, k, kq, timed_out, lane)
                              : tc_read_item(c, k, timed_out, true);
    if (it.item < 0) break;
    const int b = it.b, g = it.g, pe = it.pg_end, n = it.n, tok_end = it.t_end;
    // the first tile's page and row in it (a split starts on a page boundary, or
    // on a 128-token boundary inside pages that are multiples of 128 tokens)
    int pg0 = it.tb / P, tin0 = it.tb - pg0 * P;
    for (int t0 = it.tb; t0 < tok_end; t0 += TC_T, ++tile) {
      if ((tile & (TC_PRODUCERS - 1)) == pk) {
        const int rows = min(TC_T, tok_end - t0);
        const int npiece = (rows + geo.box_rows - 1) >> geo.box_shift;  // <= 16
        page_cache_ensure(pc, p, b, pg0, pages_per_tile ? pg0 + npiece - 1 : pg0, pe, lane);
        if (!tc_produce_tile(c, pc, geo, b, g, n, t0, rows, npiece, pg0, tin0, stage, phase,
                             timed_out, lane))
          return;
      }
      if (pages_per_tile) {
        pg0 += pages_per_tile;
      } else if ((tin0 += TC_T) == P) {
        tin0 = 0;
        ++pg0;
      }
      if (++stage == c.nst()) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
}

// Staging of row r of a quantised tile for the fp16 MMAs: the int8 / int4 /
// E4M3 codes of K and V, copied raw into the stage's V region at voff (K codes
// first, V codes rawv bytes in), become fp16 operand rows (K halves at 0, V
// halves at voff), 128-byte swizzled.  HD = head_dim: 128 fills both 64-dim halves,
// 64 the first (the QK products stop at dim 64; the P.V rows of dims 64..127 are
// never read).  A thread loads its whole row before converting it, starting at
// a row-dependent 16-byte chunk (no bank conflicts), and the V rows, which are
// expanded over the codes, are all loaded (named barrier 3) before any is
// written.  Rows that hold no token become zeros.
template <int HD>
__device__ __forceinline__ void tc_expand_codes(uint8_t *op, int voff, int rawv, int r, bool valid,
                                                int kind) {
  constexpr int NCH = HD / 16;   // 16-byte chunks of an int8 / E4M3 code row
  constexpr int NCH4 = HD / 32;  // 16-byte chunks of an int4 code row
  const uint8_t *raw = op + voff;
  const bool i4 = kind == KIND_I4;
  const int rb = i4 ? HD / 2 : HD;  // row bytes of the codes
  // K then V through one copy of the code (the kernel's roles share the SM's
  // instruction cache; unrolling this loop costs more than it saves)
#pragma unroll 1
  for (int kv = 0; kv < 2; ++kv) {
    uint8_t *dst = op + kv * voff;
    const uint8_t *src = raw + kv * rawv + r * rb;
    uint4 w[NCH];
    if (valid) {
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const int ci = i4 ? ((j + (r >> 1)) & (NCH4 - 1)) : ((j + r) & (NCH - 1));
        if (!i4 || j < NCH4) w[j] = *reinterpret_cast<const uint4 *>(src + 16 * ci);
      }
    }
    if (kv == 1) named_sync(3, 128);  // every V row has been read
    if (!valid) {
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        *reinterpret_cast<uint4 *>(dst + sw128(r, ch)) = make_uint4(0, 0, 0, 0);
        if (HD == TC_D) *reinterpret_cast<uint4 *>(dst + TC_HALF + sw128(r, ch)) = make_uint4(0, 0, 0, 0);
      }
      continue;
    }
    if (kind == KIND_I8) {
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const int ci = (j + r) & (NCH - 1);  // codes 16ci .. 16ci+15
        uint32_t o[8];
        i8x4_to_h2x2(w[j].x, o[0], o[1]);
        i8x4_to_h2x2(w[j].y, o[2], o[3]);
        i8x4_to_h2x2(w[j].z, o[4], o[5]);
        i8x4_to_h2x2(w[j].w, o[6], o[7]);
        // output chunks 2ci, 2ci+1 (8 fp16 each) in half ci/4
        uint8_t *hb = dst + (ci >> 2) * TC_HALF;
        const int oc = (2 * ci) & 7;
        *reinterpret_cast<uint4 *>(hb + sw128(r, oc)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4 *>(hb + sw128(r, oc + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
    } else if (kind == KIND_FP8) {
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const int ci = (j + r) & (NCH - 1);  // E4M3 codes 16ci .. 16ci+15
        const uint32_t wv[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
        uint32_t o[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          o[2 * q] = e4m3x2_to_h2(wv[q], 0);
          o[2 * q + 1] = e4m3x2_to_h2(wv[q], 1);
        }
        uint8_t *hb = dst + (ci >> 2) * TC_HALF;
        const int oc = (2 * ci) & 7;
        *reinterpret_cast<uint4 *>(hb + sw128(r, oc)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4 *>(hb + sw128(r, oc + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < NCH4; ++j) {
        const int ci = (j + (r >> 1)) & (NCH4 - 1);  // codes 32ci .. 32ci+31
        const uint32_t wv[4] = {w[j].x ^ 0x88888888u, w[j].y ^ 0x88888888u, w[j].z ^ 0x88888888u,
                                w[j].w ^ 0x88888888u};
        uint32_t o[16];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int k = 0; k < 4; ++k) o[4 * q + k] = i4x2_to_h2(wv[q], k);
        // output chunks 4ci .. 4ci+3 in half ci/2
        uint8_t *hb = dst + (ci >> 1) * TC_HALF;
        const int oc = (4 * ci) & 7;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4 *>(hb + sw128(r, oc + q)) =
              make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      }
    }
  }
}

// staging warpgroup: thread r (0..127) owns row r of every tile that is not direct
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ void tc_staging(TcCtx<NCOL, INTP, FEAT, IMMA> &c, bool *timed_out) {
  using Cfg = TcCfg<NCOL, INTP>;
  const DecodeParams &p = c.p;
  const int r = threadIdx.x - TC_STAGING_T0;
  const int P = p.P;
  int stage = 0;
  uint32_t phase = 0;
  for (int k = 0;; ++k) {
    const TcItem it = tc_read_item_wg(c, k, 3, r, timed_out);
    if (it.item < 0) break;
    const int tok_end = it.t_end;
    for (int t0 = it.tb; t0 < tok_end; t0 += TC_T) {
      // elected bounded wait; the outcome slot is per stage, so a slow reader can
      // never see the next use of the slot (that needs every thread's barrier)
      if (r == 0) c.S.flag_st[stage] = mbar_wait(&c.S.raw_full[stage], phase, p.err, timed_out) ? 1 : 0;
      named_sync(3, 128);
      if (c.S.flag_st[stage] == 0) {
        *timed_out = true;
        return;
      }
      (void)mbar_try_wait(&c.S.raw_full[stage], phase);
      const auto &m = c.S.meta[stage];
      if (!m.direct) {
        const bool valid = (m.valid[r >> 5] >> (r & 31)) & 1u;
        uint8_t *op = c.op + static_cast<size_t>(stage) * c.sbytes();
        if (m.kind == KIND_BF16) {
          if (!valid) {
            // V rows that hold no token become zeros (their probability is 0)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              *reinterpret_cast<uint4 *>(op + c.voff() + sw128(r, ch)) = make_uint4(0, 0, 0, 0);
              if ((IMMA || p.D == TC_D) && !c.is_compact())
                *reinterpret_cast<uint4 *>(op + 3 * TC_HALF + sw128(r, ch)) = make_uint4(0, 0, 0, 0);
            }
          }
        } else if (IMMA && m.kind == KIND_I4) {
          // int4 codes (raw rows of 64 bytes at TC_HALF for K, 3 * TC_HALF for V)
          // -> one byte per code, 16 * code, in the 128-byte-swizzled int8 operand
          // rows at 0 (K) and 2 * TC_HALF (V).  Raw and widened rows do not
          // overlap; rows past the tile's tokens hold finite codes that meet a
          // zero probability.
#pragma unroll 1
          for (int kv = 0; kv < 2; ++kv) {
            const uint8_t *src = op + (2 * kv + 1) * TC_HALF + r * (TC_D / 2);
            uint8_t *dst = op + kv * 2 * TC_HALF;
            uint4 w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              w[j] = *reinterpret_cast<const uint4 *>(src + 16 * ((j + (r >> 1)) & 3));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int ci = (j + (r >> 1)) & 3;  // codes 32ci .. 32ci+31: output chunks 2ci, 2ci+1
              const uint32_t wv[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
              uint32_t o[8];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint32_t lo = (wv[q] << 4) & 0xF0F0F0F0u;  // 16 * even elements
                const uint32_t hi = wv[q] & 0xF0F0F0F0u;         // 16 * odd elements
                o[2 * q] = prmt(lo, hi, 0x5140u);
                o[2 * q + 1] = prmt(lo, hi, 0x7362u);
              }
              *reinterpret_cast<uint4 *>(dst + sw128(r, 2 * ci)) = make_uint4(o[0], o[1], o[2], o[3]);
              *reinterpret_cast<uint4 *>(dst + sw128(r, 2 * ci + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
            }
          }
        } else if (INTP) {
          if (IMMA || p.D == TC_D)  // int8-MMA variants only run head_dim 128
            tc_expand_codes<TC_D>(op, c.voff(), c.rawv(), r, valid, m.kind);
          else
            tc_expand_codes<TC_D / 2>(op, c.voff(), c.rawv(), r, valid, m.kind);
        }
        fence_async_smem();
        named_sync(3, 128);
        if (r == 0) mbar_arrive(&c.S.op_full[stage]);
      }
      // the stage (and its description) may be refilled only once this
      // warpgroup is done with it, as well as the P.V product
      if (r == 0) mbar_arrive(&c.S.op_empty[stage]);
      if (++stage == c.nst()) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
}

// QK issuer (warp 1, one thread): for every tile in order, once its operands
// are staged and an S buffer is free, S^T = K . [q_hi | q_lo]^T into TMEM.
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ void tc_qk_issuer(TcCtx<NCOL, INTP, FEAT, IMMA> &c, bool *timed_out) {
  using Cfg = TcCfg<NCOL, INTP>;
  const DecodeParams &p = c.p;
  const int P = p.P;
  const uint32_t tmem = c.S.tmem_base;
  const uint32_t op0 = smem_u32(c.op), q0 = smem_u32(c.qop);
  int stage = 0;
  uint32_t phase = 0;
  long long tc = 0;
  int q_items = 0;  // items with tiles so far: one query operand (phase or buffer) each
  for (int item_k = 0; !*timed_out; ++item_k) {
    const TcItem it = tc_read_item(c, item_k, timed_out, false);
    if (it.item < 0) break;
    const int tok_end = it.t_end;
    if (it.tb >= tok_end) continue;
    // the item's query operand: buffer q_items & 1 filled by producer warp 0
    // (16 columns), or the one buffer the softmax warpgroup wrote (32 columns)
    const int qb = tc_qimg<NCOL>() ? (q_items & 1) : 0;
    if (tc_qimg<NCOL>()) {
      if (!mbar_wait(&c.S.qbuf_full[qb], static_cast<uint32_t>((q_items >> 1) & 1), p.err, timed_out))
        break;
    } else if (!mbar_wait(&c.S.q_full, static_cast<uint32_t>(q_items & 1), p.err, timed_out)) {
      break;
    }
    ++q_items;
    const uint32_t qop = q0 + static_cast<uint32_t>(qb * Cfg::QSTRIDE);
    for (int t0 = it.tb; t0 < tok_end; t0 += TC_T) {
      if (!mbar_wait(&c.S.op_full[stage], phase, p.err, timed_out)) break;
      if (!mbar_wait(&c.S.s_empty[tc & 1], static_cast<uint32_t>((tc >> 1) & 1) ^ 1u, p.err,
                     timed_out))
        break;
      tc_fence_after();
      const int kind = c.S.meta[stage].kind;
      const uint32_t kbase = op0 + stage * c.sbytes();
      const uint32_t d = tmem + static_cast<uint32_t>(tc & 1) * NCOL;
      if (tc_int_tile<IMMA>(kind)) {
        // int8 codes [128 tok][128 dims] x query digits [NCOL][128 dims], K = 32 per MMA
        const uint32_t idesc = tc_idesc_i8(1, 0, 0, NCOL);
        const uint32_t q8 = qop + 2 * static_cast<uint32_t>(Cfg::Q_BYTES);
#pragma unroll
        for (int k = 0; k < TC_D / 32; ++k) {
          const uint64_t a = tc_sdesc(kbase + k * 32, 16, 1024, 2);
          const uint64_t bd = tc_sdesc(q8 + k * 32, 16, 1024, 2);
          tc_mma_i8(d, a, bd, idesc, k > 0 ? 1u : 0u);
        }
      } else {
        const uint32_t idesc = tc_idesc(kind == KIND_BF16 ? 1 : 0, 0, 0, NCOL);
        const uint32_t qbase = qop + (kind == KIND_BF16 ? 0u : static_cast<uint32_t>(Cfg::Q_BYTES));
        // 8 K-steps of 16 dims, or 4 for head_dim 64 (the first half)
#pragma unroll
        for (int k = 0; k < TC_D / 16; ++k) {
          if (!IMMA && k >= 4 && p.D != TC_D) break;  // (int8-MMA variants: head_dim 128)
          const uint64_t a = tc_sdesc(kbase + (k >> 2) * TC_HALF + (k & 3) * 32, 16, 1024, 2);
          const uint64_t bd = tc_sdesc(qbase + (k >> 2) * (NCOL * 128) + (k & 3) * 32, 16, 1024, 2);
          tc_mma(d, a, bd, idesc, k > 0 ? 1u : 0u);
        }
      }
      tc_commit(&c.S.s_full[tc & 1]);
      ++tc;
      if (++stage == c.nst()) {
        stage = 0;
        phase ^= 1u;
      }
    }
    // the buffer can be refilled once the item's products have read it
    if (tc_qimg<NCOL>()) tc_commit(&c.S.qbuf_empty[qb]);
  }
  // drain: every MMA this thread issued has completed before TMEM is released
  tc_commit(&c.S.drain);
}

// P.V issuer (warp 2, one thread): for every tile in order, once its
// probabilities are written and an O buffer is free, O^T = V^T . [p_hi | p_lo]^T
// into TMEM; the commit then frees the stage, the P buffer and signals the fold.
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ void tc_pv_issuer(TcCtx<NCOL, INTP, FEAT, IMMA> &c, bool *timed_out) {
  using Cfg = TcCfg<NCOL, INTP>;
  const DecodeParams &p = c.p;
  const int P = p.P;
  const uint32_t tmem = c.S.tmem_base;
  const uint32_t op0 = smem_u32(c.op), p0 = smem_u32(c.pop);
  int stage = 0;
  long long tc = 0;
  for (int k = 0; !*timed_out; ++k) {
    const TcItem it = tc_read_item(c, k, timed_out, false);
    if (it.item < 0) break;
    const int tok_end = it.t_end;
    for (int t0 = it.tb; t0 < tok_end; t0 += TC_T) {
      const int ob = static_cast<int>(tc % Cfg::O_BUFS);
      if (!mbar_wait(&c.S.p_full[tc & 1], static_cast<uint32_t>((tc >> 1) & 1), p.err, timed_out))
        break;
      if (!mbar_wait(&c.S.o_empty[ob], static_cast<uint32_t>((tc / Cfg::O_BUFS) & 1) ^ 1u, p.err,
                     timed_out))
        break;
      tc_fence_after();
      // the tile description stays valid until this P.V has freed the stage
      const int kind = c.S.meta[stage].kind;
      // with the 32 KiB stages of head_dim 64 the MMA's rows of dims 64..127
      // read the next 16 KiB of shared memory (another stage, or the query
      // buffers): their products are never read
      const uint32_t vbase = op0 + stage * c.sbytes() + c.voff();
      const uint32_t pbase = p0 + static_cast<uint32_t>(tc & 1) * Cfg::P_BYTES;
      const uint32_t d = tmem + 2 * NCOL + static_cast<uint32_t>(ob) * NCOL;
      if (tc_int_tile<IMMA>(kind)) {
        // V^T: int8 codes [128 tok][128 dims] read dim-major; P^T: unsigned digits
        // [128 tok][16 columns]; K = 32 tokens per MMA
        const uint32_t idesc = tc_idesc_i8(0, 1, 1, NCOL);
#pragma unroll
        for (int k = 0; k < TC_T / 32; ++k) {
          const uint64_t a = tc_sdesc(vbase + k * 4096, TC_HALF, 1024, 2);
          const uint64_t bd = tc_sdesc(pbase + k * 512, 128, 2048, 0);
          tc_mma_i8(d, a, bd, idesc, k > 0 ? 1u : 0u);
        }
      } else {
        const uint32_t idesc = tc_idesc(kind == KIND_BF16 ? 1 : 0, 1, 1, NCOL);
#pragma unroll
        for (int k = 0; k < TC_T / 16; ++k) {
          const uint64_t a = tc_sdesc(vbase + k * 2048, TC_HALF, 1024, 2);
          const uint64_t bd = tc_sdesc(pbase + k * 256, 128, 2048, 0);
          tc_mma(d, a, bd, idesc, k > 0 ? 1u : 0u);
        }
      }
      tc_commit(&c.S.o_full[ob]);
      tc_commit(&c.S.p_empty[tc & 1]);
      tc_commit(&c.S.op_empty[stage]);
      ++tc;
      if (++stage == c.nst()) stage = 0;
    }
  }
  tc_commit(&c.S.drain);
}

// folds the P.V product of tile i into the running accumulators (dim t of each
// head); `oint`: the product is in int32 digit columns (an int tile of an IMMA
// variant), column 4 * l + h holding digit l of head h
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ __forceinline__ void tc_fold(TcCtx<NCOL, INTP, FEAT, IMMA> &c, long long i, uint32_t tmem, int lane,
                                        int cnt, float (&acc)[tc_rows<NCOL, IMMA>()],
                                        const float (&alpha_prev)[tc_rows<NCOL, IMMA>()],
                                        float vscale_prev, bool oint, bool *timed_out) {
  const int ob = static_cast<int>(i % TcCfg<NCOL, INTP>::O_BUFS);
  (void)mbar_wait(&c.S.o_full[ob], static_cast<uint32_t>((i / TcCfg<NCOL, INTP>::O_BUFS) & 1),
                  c.p.err, timed_out);
  tc_fence_after();
  float o[NCOL];
  tmem_ld<NCOL>(tmem + 2 * NCOL + static_cast<uint32_t>(ob) * NCOL, o);
  tc_wait_ld();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&c.S.o_empty[ob]);
  if (IMMA && oint) {
    // sum_l digit_l 256^-l in fp32 (every int32 product sum is below 2^22, exact)
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      if (h < cnt) {
        float t = fmaf(small_i2f(o[12 + h]), 1.f / 256.f, small_i2f(o[8 + h]));
        t = fmaf(t, 1.f / 256.f, small_i2f(o[4 + h]));
        t = fmaf(t, 1.f / 256.f, small_i2f(o[h]));
        acc[h] = fmaf(acc[h], alpha_prev[h], t * vscale_prev);
      }
    }
    return;
  }
#pragma unroll
  for (int h = 0; h < tc_rows<NCOL, IMMA>(); ++h)
    if (h < cnt) acc[h] = fmaf(acc[h], alpha_prev[h], (o[h] + o[NCOL / 2 + h]) * vscale_prev);
}

// element `dim` of query row vh of sequence b, as fp32 (head_dim 128: the int8
// digit operands of the int8-MMA variants)
__device__ __forceinline__ float q_elem(const DecodeParams &p, int b, int vh, int dim) {
  const long long i = (static_cast<long long>(b) * p.Hq + vh) * TC_D + dim;
  return p.q_fmt == CFR_FMT_F32
             ? static_cast<const float *>(p.q)[i]
             : __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t *>(p.q)[i]) << 16);
}

// Builds the query operand of (sequence b, kv head g) at dst, in the shared-memory
// layout the QK products read (dst is shared memory, or a global image that is
// later copied byte for byte to a 1024-byte-aligned shared buffer):
//  - dst: bf16 operand, NCOL rows x 128 dims (2 halves of 64), 128-byte swizzled:
//    rows [0, NCOL/2) the hi parts of the group's query rows, rows [NCOL/2, NCOL)
//    the lo parts (q - bf16(q));
//  - dst + Q_BYTES (quantised pools): the same with fp16 hi/lo;
//  - dst + 2 Q_BYTES (IMMA): int8 digit operand, row 4 * l + h = digit l of head
//    h (h < 4) of q_h * 127 / max|q_h| = d0 + d1 / 128 + d2 / 128^2 + d3 / 128^3,
//    d0 in [-127, 127], d1..d3 in [-64, 64]; qsc[h] receives max|q_h| / 127.
// The 128 threads of a warpgroup or block (index tsm) share the work; the IMMA
// part synchronises them once (sync()) through red[4][4] floats.
template <int HD, int NCOL, bool INTP, bool IMMA, class Sync>
__device__ __forceinline__ void tc_build_q_d(const DecodeParams &p, int b, int g, int tsm, int lane,
                                           uint8_t *dst, float (*red)[4], Sync sync,
                                           float (&qsc)[4]) {
  using Cfg = TcCfg<NCOL, INTP>;
  const int h0 = p.grp_off[g], cnt = p.grp_off[g + 1] - h0;
  for (int idx = tsm; idx < NCOL * 16; idx += 128) {
    const int n = idx >> 4, ch = idx & 15;  // row n, 8-element chunk ch of 16
    constexpr int GM = NCOL / 2;            // rows [0, GM): hi parts, [GM, NCOL): lo parts
    const bool lo_part = n >= GM;
    const int head = lo_part ? n - GM : n;
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = 0.f;
    if (head < cnt && 8 * ch < HD) {  // dims past head_dim 64 stay 0
      const long long qi = (static_cast<long long>(b) * p.Hq + p.grp_heads[h0 + head]) * HD + 8 * ch;
      if (p.q_fmt == CFR_FMT_F32) {
        const float4 a = *reinterpret_cast<const float4 *>(static_cast<const float *>(p.q) + qi);
        const float4 bb = *reinterpret_cast<const float4 *>(static_cast<const float *>(p.q) + qi + 4);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = bb.x; x[5] = bb.y; x[6] = bb.z; x[7] = bb.w;
      } else {
        const uint4 w = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.q) + qi);
        const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x[2 * k] = bf16_lo(a[k]);
          x[2 * k + 1] = bf16_hi(a[k]);
        }
      }
    }
    uint32_t wb[4], wh[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float bl[2], fl[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float v = x[2 * k + e];
        const float bh = __bfloat162float(__float2bfloat16_rn(v));
        const float fh = __half2float(__float2half_rn(v));
        bl[e] = lo_part ? v - bh : bh;
        fl[e] = lo_part ? v - fh : fh;
      }
      wb[k] = pack_bf16(bl[0], bl[1]);
      wh[k] = pack_f16(fl[0], fl[1]);
    }
    const int off = (ch >> 3) * (NCOL * 128) + sw128(n, ch & 7);
    *reinterpret_cast<uint4 *>(dst + off) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
    if (INTP) *reinterpret_cast<uint4 *>(dst + Cfg::Q_BYTES + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
  }
  if constexpr (IMMA) {
    static_assert(NCOL == 16, "int8 digit operand: 4 digits x 4 heads");
    // max|q_h| over the 128 dims: thread tsm holds dim tsm of every head
    float mx[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      float v = 0.f;
      if (h < cnt) v = fabsf(q_elem(p, b, p.grp_heads[h0 + h], tsm));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      mx[h] = v;
    }
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < 4; ++h) red[tsm >> 5][h] = mx[h];
    }
    sync();
#pragma unroll
    for (int h = 0; h < 4; ++h)
      qsc[h] = fmaxf(fmaxf(red[0][h], red[1][h]), fmaxf(red[2][h], red[3][h])) * (1.f / 127.f);
    // row n = 4 * l + h, 16-dim chunk ch of it
    const int n = tsm >> 3, ch = tsm & 7, l = n >> 2, h = n & 3;
    float sc = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k == h) sc = qsc[k];
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (h < cnt && sc > 0.f) {
      const float inv = 1.f / sc;
      const int head = p.grp_heads[h0 + h];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float r = q_elem(p, b, head, 16 * ch + e) * inv;
        float d = rintf(r);
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          if (k < l) {
            r = (r - d) * 128.f;
            d = rintf(r);
          }
        }
        w[e >> 2] |= (static_cast<uint32_t>(static_cast<int>(d)) & 0xFFu) << (8 * (e & 3));
      }
    }
    *reinterpret_cast<uint4 *>(dst + 2 * Cfg::Q_BYTES + sw128(n, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// head_dim 128 or 64 (the operand's second half left at 0), with the row
// stride as a compile-time constant
template <int NCOL, bool INTP, bool IMMA, class Sync>
__device__ __forceinline__ void tc_build_q(const DecodeParams &p, int b, int g, int tsm, int lane,
                                           uint8_t *dst, float (*red)[4], Sync sync,
                                           float (&qsc)[4]) {
  if (IMMA || p.D == TC_D)  // int8-MMA variants only run head_dim 128
    tc_build_q_d<TC_D, NCOL, INTP, IMMA>(p, b, g, tsm, lane, dst, red, sync, qsc);
  else if constexpr (!IMMA)
    tc_build_q_d<TC_D / 2, NCOL, INTP, IMMA>(p, b, g, tsm, lane, dst, red, sync, qsc);
}

// 32-column variants: the softmax warpgroup writes the query operand of item
// `it` into the one query buffer, then each warp arrives on q_full.
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ __forceinline__ void tc_write_q(TcCtx<NCOL, INTP, FEAT, IMMA> &c, const TcItem &it, int tsm,
                                           int lane) {
  float unused[4];  // (int8 digit operands exist only in 16-column variants)
  tc_build_q<NCOL, INTP, false>(c.p, it.b, it.g, tsm, lane, c.qop,
                                reinterpret_cast<float (*)[4]>(c.S.red_l), [] {}, unused);
  fence_async_smem();
  __syncwarp();
  if (lane == 0) mbar_arrive(&c.S.q_full);
}

// The query operand image of every (sequence, kv head), one 128-thread block
// each, for the 16-column variants: built once per decode call, copied into
// shared memory for every work item of the group.  Sequences outside
// [1, max_pages * page_tokens] are skipped (the decode skips them too).
template <int NCOL, bool INTP, bool IMMA>
__global__ void __launch_bounds__(128) tc_qimage_kernel(const __grid_constant__ DecodeParams p,
                                                        const __grid_constant__ SchedArgs sched,
                                                        int with_schedule) {
  __shared__ float red[4][4];
  if (with_schedule && blockIdx.x == 0) {
    // block 0 computes the split schedule (one launch for both)
    schedule_block(sched);
    return;
  }
  const long long grp = static_cast<long long>(blockIdx.x) - with_schedule;
  const int b = static_cast<int>(grp / p.ngroups), g = static_cast<int>(grp % p.ngroups);
  const int n = p.seq_lens[b];
  if (n < p.nq || n > p.max_pages * p.P) return;
  float qsc[4] = {0.f, 0.f, 0.f, 0.f};
  tc_build_q<NCOL, INTP, IMMA>(p, b, g, threadIdx.x, threadIdx.x & 31, p.qimg + grp * kQImgBytes, red,
                               [] { __syncthreads(); }, qsc);
  if (threadIdx.x < 4) p.qscale[grp * 4 + threadIdx.x] = qsc[threadIdx.x];
}

// softmax / fold warpgroup.  Every thread waits on the mbarriers itself; a
// thread whose wait gives up keeps the same control flow (later waits return at
// once), so the one named barrier per tile is always reached by all 128 threads.
template <int NCOL, bool INTP, int FEAT, bool IMMA>
__device__ void tc_softmax(TcCtx<NCOL, INTP, FEAT, IMMA> &c, bool *timed_out) {
  using Cfg = TcCfg<NCOL, INTP>;
  constexpr int GM = NCOL / 2;  // offset of the lo columns of the 16-bit operands
  constexpr int GH = tc_rows<NCOL, IMMA>();  // query rows a tile holds
  const DecodeParams &p = c.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int t = 32 * quarter + lane;  // TMEM lane: token t of S, dim t of O
  const int tsm = threadIdx.x - TC_SOFTMAX_T0;  // 0..127 within the warpgroup
  const uint32_t tmem = c.S.tmem_base + (static_cast<uint32_t>(32 * quarter) << 16);
  const int P = p.P;
  const int pshift = 31 - __clz(P < TC_T ? P : TC_T);  // log2 of a page piece's rows
  int stage = 0;
  uint32_t phase = 0;
  long long tc = 0;
  bool q_ready = false;
  // 32-column variants write the query operand themselves: the next item's is
  // written at the last tile of the current one, right after its last QK product
  // has been read; nxt_read says whether that read has happened
  int k = 0;
  TcItem nxt;
  nxt.item = -1;
  bool nxt_read = false;

  for (TcItem it = tc_read_item_wg(c, 0, 2, tsm, timed_out); it.item >= 0; ++k) {
    const int slot = it.slot, g = it.g, n = it.n, tok_end = it.t_end;
    const int h0 = p.grp_off[g], cnt = p.grp_off[g + 1] - h0;
    if constexpr (!tc_qimg<NCOL>())
      if (!q_ready && it.tb < tok_end) tc_write_q(c, it, tsm, lane);
    q_ready = false;
    nxt_read = false;
    float qs[4] = {0.f, 0.f, 0.f, 0.f};  // this item's int8 digit scales (max|q_h| / 127)
    if constexpr (IMMA) {
#pragma unroll
      for (int h = 0; h < 4; ++h) qs[h] = c.S.qs_bc[k & 1][h];
    }

    // folds lag two tiles behind the scores: tiles prev2 (older) and prev1 wait,
    // each with its rescale factors and V scale
    float slope2[GH], m_run[GH], l_part[GH], acc[GH], alpha1[GH], alpha2[GH];
    // causal offsets of the query rows, 4 bits each (at most 16 rows of offset <= 15)
    uint32_t qoff[2] = {0u, 0u};
#pragma unroll
    for (int h = 0; h < GH; ++h) {
      // 0 past the group's rows and without ALiBi
      if constexpr (tc_qimg<NCOL>())
        slope2[h] = c.S.slope_bc[k & 1][h];
      else
        slope2[h] = (p.slopes && h < cnt) ? p.slopes[row_head(p, p.grp_heads[h0 + h])] * kLog2e : 0.f;
      if constexpr (tc_feat(FEAT) == TC_FEAT_MULTI)
        if (h < cnt) qoff[h >> 3] |= static_cast<uint32_t>(row_offset(p, p.grp_heads[h0 + h])) << (4 * (h & 7));
      m_run[h] = -INFINITY;
      l_part[h] = 0.f;
      acc[h] = 0.f;
      alpha1[h] = 1.f;
      alpha2[h] = 1.f;
    }
    float vs1 = 1.f, vs2 = 1.f;
    bool oi1 = false, oi2 = false;  // the pending P.V products are int32 digit columns
    long long prev1 = -1, prev2 = -1;

    for (int t0 = it.tb; t0 < tok_end; t0 += TC_T) {
      // ---- scores of tile tc ----
      (void)mbar_wait(&c.S.s_full[tc & 1], static_cast<uint32_t>((tc >> 1) & 1), p.err, timed_out);
      tc_fence_after();
      float sv[NCOL];
      tmem_ld<NCOL>(tmem + static_cast<uint32_t>(tc & 1) * NCOL, sv);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.S.s_empty[tc & 1]);
      // acquire the tile description published through the stage's op_full phase
      // (that phase cannot move on before this tile's P.V has run)
      (void)mbar_try_wait(&c.S.op_full[stage], phase);
      const auto &m = c.S.meta[stage];
      const bool valid = (m.valid[t >> 5] >> (t & 31)) & 1u;
      const int kind = m.kind;
      const bool itile = tc_int_tile<IMMA>(kind);
      // int4 codes enter the int8 MMAs times 16; probability digits are of p * 255
      const float i4f = itile && kind == KIND_I4 ? 1.f / 16.f : 1.f;
      // quantised tiles: token t's page piece gives its K scale and its V scale
      // relative to the tile's (1 with one piece per tile: pages of 128 tokens
      // or more)
      float scale = p.sigma_log2e, vratio = 1.f;
      if (kind != KIND_BF16) {
        constexpr bool pieces = tc_pieces<NCOL, INTP, FEAT>();
        const int piece = pieces ? t >> pshift : 0;
        scale = m.ksp[piece] * p.sigma_log2e * i4f;
        if (pieces) vratio = m.vsp[piece];
      }
      const float vsc = kind == KIND_BF16 ? 1.f
                        : itile           ? m.vs * i4f * (1.f / 255.f)
                                          : m.vs * (1.f / 32768.f);
      // ALiBi from the last position; a query row at offset o before it differs by the
      // row constant slope * o, added back to its maximum at the partial write
      const int j = m.t0 + t;
      const float dist = static_cast<float>(n - 1 - j);
      float s[GH];
      if (IMMA && itile) {
        // column 4 * l + h: digit l of head h; sum_l S_l 128^-l, exact terms below 2^22
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          s[h] = -INFINITY;
          if (h < 4 && valid && h < cnt) {
            float u = fmaf(small_i2f(sv[12 + h]), 1.f / 128.f, small_i2f(sv[8 + h]));
            u = fmaf(u, 1.f / 128.f, small_i2f(sv[4 + h]));
            u = fmaf(u, 1.f / 128.f, small_i2f(sv[h]));
            s[h] = fmaf(u, scale * qs[h], -slope2[h] * dist);
          }
        }
      } else {
#pragma unroll
        for (int h = 0; h < GH; ++h)
          s[h] = (valid && h < cnt) ? fmaf(sv[h] + sv[GM + h], scale, -slope2[h] * dist) : -INFINITY;
      }
      if (tc_feat(FEAT) == TC_FEAT_MULTI && m.t0 + TC_T - 1 > n - p.nq) {
        // the tile reaches the query positions: row h sees tokens j <= n - 1 - offset_h
#pragma unroll
        for (int h = 0; h < GH; ++h)
          if (j > n - 1 - static_cast<int>((qoff[h >> 3] >> (4 * (h & 7))) & 15u)) s[h] = -INFINITY;
      }
      {
        int hm;
        const float mx = warp_multi_max<GH>(s, lane, &hm);
        // lanes whose bits below the last halving offset are zero hold head hm's max
        if ((lane & ((32 / GH) - 1)) == 0) c.S.red_max[tc & 1][quarter][hm] = mx;
      }
      // the P buffer of this tile must be free (P.V of tile tc-2 done)
      (void)mbar_wait(&c.S.p_empty[tc & 1], static_cast<uint32_t>((tc >> 1) & 1) ^ 1u, p.err, timed_out);
      named_sync(2, 128);
      float pr[GH], alpha[GH], mt[GH];
#pragma unroll
      for (int h4 = 0; h4 < GH; h4 += 4) {
        float4 a[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) a[q] = *reinterpret_cast<const float4 *>(&c.S.red_max[tc & 1][q][h4]);
        mt[h4 + 0] = fmaxf(fmaxf(a[0].x, a[1].x), fmaxf(a[2].x, a[3].x));
        mt[h4 + 1] = fmaxf(fmaxf(a[0].y, a[1].y), fmaxf(a[2].y, a[3].y));
        mt[h4 + 2] = fmaxf(fmaxf(a[0].z, a[1].z), fmaxf(a[2].z, a[3].z));
        mt[h4 + 3] = fmaxf(fmaxf(a[0].w, a[1].w), fmaxf(a[2].w, a[3].w));
      }
#pragma unroll
      for (int h = 0; h < GH; ++h) {
        const float m_new = fmaxf(m_run[h], mt[h]);
        if (m_new == -INFINITY) {
          alpha[h] = 1.f;
          pr[h] = 0.f;
        } else {
          alpha[h] = exp2_approx(m_run[h] - m_new);
          pr[h] = exp2_approx(s[h] - m_new);
        }
        l_part[h] = fmaf(l_part[h], alpha[h], pr[h]);
        m_run[h] = m_new;
      }
      if (IMMA && itile) {
        // P^T row t: 16 unsigned digit columns, column 4 * l + h = digit l of
        // p_h * 255 = e0 + e1 / 256 + e2 / 256^2 + e3 / 256^3: the bytes, most
        // significant first, of X_h = round(p_h * 255 * 2^24) (< 2^32 for p <= 1)
        uint32_t x[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) x[h] = __float2uint_rn(pr[h] * vratio * 4278190080.f);
        // transpose the 4 x 4 bytes: word l = byte 3 - l of x[0..3]
        const uint32_t lo01 = prmt(x[0], x[1], 0x5140u), hi01 = prmt(x[0], x[1], 0x7362u);
        const uint32_t lo23 = prmt(x[2], x[3], 0x5140u), hi23 = prmt(x[2], x[3], 0x7362u);
        *reinterpret_cast<uint4 *>(c.pop + (tc & 1) * Cfg::P_BYTES + t * 16) =
            make_uint4(prmt(hi01, hi23, 0x7632u), prmt(hi01, hi23, 0x5410u), prmt(lo01, lo23, 0x7632u),
                       prmt(lo01, lo23, 0x5410u));
      } else {
        // P^T row t: columns [hi(0..GM) | lo(0..GM)]
        float colv[NCOL];
#pragma unroll
        for (int k = 0; k < NCOL; ++k) colv[k] = 0.f;
        // fp16 probabilities of quantised tiles are scaled up by 2^15 (and by the
        // row's V-scale ratio) to use the fp16 range
        const float pre = kind == KIND_BF16 ? 1.f : 32768.f * vratio;
#pragma unroll
        for (int h = 0; h < GH; ++h) {
          const float x = pr[h] * pre;  // 0 for the padding heads h >= cnt
          const float xh = kind == KIND_BF16 ? __bfloat162float(__float2bfloat16_rn(x))
                                             : __half2float(__float2half_rn(x));
          colv[h] = xh;
          colv[GM + h] = x - xh;
        }
        uint8_t *pb_ = c.pop + (tc & 1) * Cfg::P_BYTES;
#pragma unroll
        for (int grp = 0; grp < NCOL / 8; ++grp) {
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            w[k] = kind == KIND_BF16 ? pack_bf16(colv[8 * grp + 2 * k], colv[8 * grp + 2 * k + 1])
                                     : pack_f16(colv[8 * grp + 2 * k], colv[8 * grp + 2 * k + 1]);
          *reinterpret_cast<uint4 *>(pb_ + grp * 2048 + t * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.S.p_full[tc & 1]);

      if (!tc_qimg<NCOL>() && t0 + TC_T >= tok_end) {
        // the next item's query operand can be written as soon as this item's
        // last QK product has been read
        nxt = tc_read_item_wg(c, k + 1, 2, tsm, timed_out);
        nxt_read = true;
        if (nxt.item >= 0 && nxt.tb < nxt.t_end) {
          tc_write_q(c, nxt, tsm, lane);
          q_ready = true;
        }
      }
      // fold the tile two behind (its P.V has long been issued)
      if (prev2 >= 0) tc_fold(c, prev2, tmem, lane, cnt, acc, alpha2, vs2, oi2, timed_out);
      prev2 = prev1;
      vs2 = vs1;
      oi2 = oi1;
#pragma unroll
      for (int h = 0; h < GH; ++h) {
        alpha2[h] = alpha1[h];
        alpha1[h] = alpha[h];
      }
      prev1 = tc;
      vs1 = vsc;
      oi1 = itile;
      ++tc;
      if (++stage == c.nst()) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (prev2 >= 0) tc_fold(c, prev2, tmem, lane, cnt, acc, alpha2, vs2, oi2, timed_out);
    if (prev1 >= 0) tc_fold(c, prev1, tmem, lane, cnt, acc, alpha1, vs1, oi1, timed_out);

    // split partial: acc (dim t), m, and l summed over the 128 token slots
#pragma unroll
    for (int h = 0; h < GH; ++h) {
      if (h < cnt) {
        const int head = p.grp_heads[h0 + h];
        if (IMMA || p.D == TC_D)  // (head_dim 64: dims 64..127 of O hold nothing)
          p.part_acc[(static_cast<long long>(slot) * p.Hq + head) * TC_D + t] = acc[h];
        else if (t < TC_D / 2)
          p.part_acc[(static_cast<long long>(slot) * p.Hq + head) * (TC_D / 2) + t] = acc[h];
        float l = l_part[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) c.S.red_l[quarter][h] = l;
      }
    }
    named_sync(2, 128);
    if (tsm < cnt) {
      const long long cidx = static_cast<long long>(slot) * p.Hq + p.grp_heads[h0 + tsm];
      float mrun = -INFINITY;
#pragma unroll
      for (int h = 0; h < GH; ++h)
        if (h == tsm) mrun = m_run[h];
      if constexpr (tc_feat(FEAT) == TC_FEAT_MULTI) {
        const int vh = p.grp_heads[h0 + tsm];
        float sl = 0.f;
#pragma unroll
        for (int h = 0; h < GH; ++h)
          if (h == tsm) sl = slope2[h];
        if (mrun != -INFINITY) mrun = fmaf(sl, static_cast<float>(row_offset(p, vh)), mrun);
      }
      p.part_m[cidx] = mrun;
      p.part_l[cidx] = (c.S.red_l[0][tsm] + c.S.red_l[1][tsm]) + (c.S.red_l[2][tsm] + c.S.red_l[3][tsm]);
    }
    named_sync(2, 128);
    it = nxt_read ? nxt : tc_read_item_wg(c, k + 1, 2, tsm, timed_out);
  }
}

template <int NCOL, bool INTP, int FEAT, bool IMMA>
__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_decode_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ TcMaps maps) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t a0 = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + ((1024u - (a0 & 1023u)) & 1023u);
  using L = TcLayout<NCOL, INTP>;
  TcSmem<NCOL, INTP> &S = *reinterpret_cast<TcSmem<NCOL, INTP> *>(smem);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < TcCfg<NCOL, INTP>::MAX_STAGES; ++s) {
      mbar_init(&S.op_full[s], 1);
      mbar_init(&S.op_empty[s], 2);  // P.V commit + staging warpgroup
      mbar_init(&S.raw_full[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_empty[i], 4);
      mbar_init(&S.p_full[i], 4);
      mbar_init(&S.p_empty[i], 1);
    }
    for (int i = 0; i < TcCfg<NCOL, INTP>::O_BUFS; ++i) {
      mbar_init(&S.o_full[i], 1);
      mbar_init(&S.o_empty[i], 4);
    }
    for (int i = 0; i < TC_ITEM_RING; ++i) {
      mbar_init(&S.item_full[i], 1);
      mbar_init(&S.item_empty[i], TC_ITEM_READERS);
    }
    mbar_init(&S.q_full, 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.qbuf_full[i], 1);
      mbar_init(&S.qbuf_empty[i], 1);  // the QK issuer's commit after the item's last product
    }
    mbar_init(&S.drain, 2);  // one commit from each MMA issuer
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&S.tmem_base)),
                 "r"(TcCfg<NCOL, INTP>::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // the split schedule comes from the previous kernel (returns at once
                   // when the launch did not overlap it)

  const int nsplit = schedule_split_count(p, threadIdx.x == 0 && blockIdx.x == 0);
  TcCtx<NCOL, INTP, FEAT, IMMA> c{p,
                                  maps,
                                  S,
                                  smem + L::op,
                                  smem + L::q,
                                  smem + L::pbuf,
                                  static_cast<long long>(nsplit) * p.ngroups,
                                  nsplit,
                                  NCOL == 16 && !IMMA && p.D == TC_D / 2};
  bool timed_out = false;
  if (warp < 4) {
    tc_setmaxnreg<TC_REGS_IO>();
    if (warp == 0 || warp == TC_PROD2_WARP) {
      tc_producer<NCOL, INTP, FEAT, IMMA>(c, &timed_out, warp == 0 ? 0 : 1);
    } else if (warp == TC_QK_WARP) {
      if ((threadIdx.x & 31) == 0) tc_qk_issuer<NCOL, INTP, FEAT, IMMA>(c, &timed_out);
    } else {
      if ((threadIdx.x & 31) == 0) tc_pv_issuer<NCOL, INTP, FEAT, IMMA>(c, &timed_out);
    }
  } else if (warp < 8) {
    tc_setmaxnreg<TC_REGS_SOFTMAX>();
    tc_softmax<NCOL, INTP, FEAT, IMMA>(c, &timed_out);
  } else {
    // the int8-MMA variants' staging (int4 widening only) runs in fewer registers,
    // which measured faster there
    tc_setmaxnreg<IMMA ? TC_REGS_STAGING_IMMA : TC_REGS_STAGING>();
    tc_staging<NCOL, INTP, FEAT, IMMA>(c, &timed_out);
  }
  tc_fence_before();
  __syncthreads();
  if (tc_claimed_items<INTP, FEAT, IMMA>() && threadIdx.x == 0 && p.item_ctr) {
    // every CTA has stopped claiming once all have counted themselves finished;
    // the last one leaves both counters at 0 for the next launch
    __threadfence();
    if (atomicAdd(&p.item_ctr[1], 1u) == gridDim.x - 1) {
      atomicExch(&p.item_ctr[0], 0u);
      atomicExch(&p.item_ctr[1], 0u);
    }
  }
  if (warp == 1) {
    if ((threadIdx.x & 31) == 0) {
      bool t2 = false;
      (void)mbar_wait(&S.drain, 0, p.err, &t2);  // every MMA of both issuers has completed
    }
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(S.tmem_base),
                 "r"(TcCfg<NCOL, INTP>::TMEM_COLS)
                 : "memory");
  }
}

// quantised pools present: tiles pass through the raw staging buffers
static bool tc_int_pools(const DecodeParams &p, bool page_fmt_given) {
  if (page_fmt_given) return p.k_pool[CFR_FMT_I8] || p.k_pool[CFR_FMT_I4] || p.k_pool[CFR_FMT_FP8];
  return is_quantised(p.uniform_fmt);
}

bool tc_supported(const DecodeParams &p, bool page_fmt_given) {
  if ((p.D != TC_D && p.D != TC_D / 2) || p.gmax > 16) return false;
  if ((reinterpret_cast<uintptr_t>(p.q) & 15) != 0) return false;
  if (page_fmt_given) {
    if (p.k_pool[CFR_FMT_F32]) return false;
    if (!p.k_pool[CFR_FMT_BF16] && !p.k_pool[CFR_FMT_I8] && !p.k_pool[CFR_FMT_I4] &&
        !p.k_pool[CFR_FMT_FP8])
      return false;
  } else if (p.uniform_fmt == CFR_FMT_F32) {
    return false;
  }
  const bool ints = tc_int_pools(p, page_fmt_given);
  const bool p_ok = (p.P <= TC_T && TC_T % p.P == 0) || p.P % TC_T == 0;
  // quantised pages shorter than a tile only in a uniform-format cache (a tile
  // then holds pieces of one format, each with its own scales) and with at most
  // 8 rows per group (the 16-column variants keep the pieces' scales)
  if (!p_ok || (ints && p.P % TC_T != 0 && (page_fmt_given || p.gmax > 8))) return false;
  const long long rows = p.pool_pages[CFR_FMT_BF16] * p.Hkv * static_cast<long long>(p.P);
  if (rows > 0x7fffffffLL) return false;
  // int8 pools are read through a tensor map when their tiles run int8 MMAs
  const long long rows8 = p.pool_pages[CFR_FMT_I8] * p.Hkv * static_cast<long long>(p.P);
  if (p.k_pool[CFR_FMT_I8] && p.gmax <= 4 && rows8 > 0x7fffffffLL) return false;
  return true;
}

void launch_schedule(const int32_t *seq_lens, int batch, int P, int max_pages, int target,
                     int sink, int window, int nq, int unit, int32_t *split_off, int32_t *splits,
                     int max_splits, int32_t *num_splits, uint32_t *item_ctr, uint32_t *err,
                     cudaStream_t stream);

// `sched`, when set, is this call's split schedule, which runs before the decode:
// in one extra block of the query-image kernel where the variant has one, else
// as the schedule kernel
template <int NCOL, bool INTP, int FEAT, bool IMMA>
static cudaError_t tc_launch_t(const DecodeParams &p, int grid, cudaStream_t stream,
                               const SchedArgs *sched) {
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (p.k_pool[CFR_FMT_BF16] && p.pool_pages[CFR_FMT_BF16] > 0) {
    const long long rows = p.pool_pages[CFR_FMT_BF16] * p.Hkv * static_cast<long long>(p.P);
    const int box_rows = p.P < TC_T ? p.P : TC_T;
    if (!encode_pool_map(&maps.k, p.k_pool[CFR_FMT_BF16], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows,
                         p.D, box_rows) ||
        !encode_pool_map(&maps.v, p.v_pool[CFR_FMT_BF16], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows,
                         p.D, box_rows))
      return cudaErrorInvalidValue;
  }
  if (IMMA && p.k_pool[CFR_FMT_I8] && p.pool_pages[CFR_FMT_I8] > 0) {
    // one box per page piece: 128 rows, or a whole page when pages are shorter
    const long long rows = p.pool_pages[CFR_FMT_I8] * p.Hkv * static_cast<long long>(p.P);
    const int box_rows = p.P < TC_T ? p.P : TC_T;
    if (!encode_pool_map(&maps.k8, p.k_pool[CFR_FMT_I8], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows,
                         TC_D, box_rows) ||
        !encode_pool_map(&maps.v8, p.v_pool[CFR_FMT_I8], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows,
                         TC_D, box_rows))
      return cudaErrorInvalidValue;
  }
  constexpr size_t smem = TcLayout<NCOL, INTP>::launch_bytes;
  static_assert(smem <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(tc_decode_kernel<NCOL, INTP, FEAT, IMMA>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // the warpgroups' register split assumes the launch count it was written for
  static const int launch_regs = [] {
    cudaFuncAttributes fa;
    return cudaFuncGetAttributes(&fa, tc_decode_kernel<NCOL, INTP, FEAT, IMMA>) == cudaSuccess
               ? fa.numRegs
               : -1;
  }();
  if (launch_regs != TC_REGS_LAUNCH) return cudaErrorInvalidConfiguration;
  if constexpr (tc_qimg<NCOL>()) {
    // the query operand image of every (sequence, row group), after the schedule
    // in block 0 when this call schedules
    const long long groups = static_cast<long long>(p.batch) * p.ngroups;
    const SchedArgs sa = sched ? *sched : SchedArgs{};
    const int extra = sched ? 1 : 0;
    tc_qimage_kernel<NCOL, INTP, IMMA>
        <<<dim3(static_cast<unsigned>(groups + extra)), dim3(128), 0, stream>>>(p, sa, extra);
  } else if (sched) {
    launch_schedule(sched->seq_lens, sched->batch, sched->P, sched->max_pages, sched->target,
                    sched->sink, sched->window, sched->nq, sched->unit, sched->split_off, sched->splits,
                    sched->max_splits, sched->num_splits, sched->item_ctr, sched->err, stream);
  }
  // a plain launch: overlapping this kernel's start with the previous kernel
  // (programmatic dependent launch) measured slower for this kernel
  tc_decode_kernel<NCOL, INTP, FEAT, IMMA><<<dim3(grid), dim3(TC_THREADS), smem, stream>>>(p, maps);
  e = cudaSuccess;
  return e != cudaSuccess ? e : cudaGetLastError();
}

// int8 or int4 pools whose tiles can run the int8 MMAs: up to 4 query rows per
// kv head (4 digit columns each fill the 16-column operand)
static bool tc_imma(const DecodeParams &p, bool page_fmt_given) {
  // (quantised pages under 128 tokens: uniform-format caches only)
  if (p.gmax > 4 || p.D != TC_D || (p.P % TC_T != 0 && page_fmt_given)) return false;
  if (page_fmt_given) return p.k_pool[CFR_FMT_I8] || p.k_pool[CFR_FMT_I4];
  return p.uniform_fmt == CFR_FMT_I8 || p.uniform_fmt == CFR_FMT_I4;
}

template <int FEAT>
static cudaError_t tc_launch_f(const DecodeParams &p, int grid, cudaStream_t stream,
                               const SchedArgs *sched) {
  const bool ints = tc_int_pools(p, p.page_fmt != nullptr);
  // quantised pages under 128 tokens (uniform format, at most 8 rows per group)
  const bool small = ints && p.P < TC_T;
  if (ints && tc_imma(p, p.page_fmt != nullptr)) {
    constexpr int S = TC_FEAT_SMALL_PAGES, C = TC_FEAT_COMPACT_I8;
    if (!p.page_fmt && p.uniform_fmt == CFR_FMT_I8)  // int8 tiles only: six 32 KiB stages
      return small ? tc_launch_t<16, true, FEAT | S | C, true>(p, grid, stream, sched)
                   : tc_launch_t<16, true, FEAT | C, true>(p, grid, stream, sched);
    return small ? tc_launch_t<16, true, FEAT | S, true>(p, grid, stream, sched)
                 : tc_launch_t<16, true, FEAT, true>(p, grid, stream, sched);
  }
  if (small) return tc_launch_t<16, true, FEAT | TC_FEAT_SMALL_PAGES, false>(p, grid, stream, sched);
  if (p.gmax <= 8)
    return ints ? tc_launch_t<16, true, FEAT, false>(p, grid, stream, sched)
                : tc_launch_t<16, false, FEAT, false>(p, grid, stream, sched);
  return ints ? tc_launch_t<32, true, FEAT, false>(p, grid, stream, sched)
              : tc_launch_t<32, false, FEAT, false>(p, grid, stream, sched);
}

cudaError_t launch_decode_tc(const DecodeParams &p, int grid, cudaStream_t stream,
                             const SchedArgs *sched) {
  // plain decode runs neither the per-row causal masks nor the subset masks
  if (p.nq > 1) return tc_launch_f<TC_FEAT_MULTI>(p, grid, stream, sched);
  if (p.window > 0) return tc_launch_f<TC_FEAT_SUBSET>(p, grid, stream, sched);
  return tc_launch_f<TC_FEAT_PLAIN>(p, grid, stream, sched);
}

}  // namespace cfr
