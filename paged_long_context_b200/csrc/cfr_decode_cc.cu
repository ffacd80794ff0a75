// cfr_decode_cc.cu -- split-KV paged decode attention on the CUDA cores.
//
// Persistent kernel, one CTA per SM.  Work item = (split of one sequence, kv
// head): a contiguous range of pages of sequence b and the G query heads that
// share kv head g (GQA: one K/V read serves the whole group; CFR-Atlas page,
// "MHA/MQA/GQA head mapping").
//
// Warp roles (W = 16 consumer warps, or 8 when GT x D > 512 leaves too few
// registers for 16):
//  - warp W is the producer: lane i resolves page piece i of a tile (the
//    tile's rows of one page) through the page table, checks slot, format and
//    pool, and copies its K and V rows into a shared-memory ring with one 1-D
//    bulk copy each (TMA engine, completion on an mbarrier), packed at the
//    piece's own row size.  Pages that do not resolve are skipped and reported
//    in the error word, never dereferenced.
//  - warps 0..W-1 consume tiles.  Per tile: (1) scores s = sigma*(q.k)*scale_k +
//    ALiBi, in base 2, eight lanes per token row; (2) per head, the tile max,
//    the rescale factor 2^(m_old - m_new), p = 2^(s - m_new) and the running
//    normaliser -- the exact fold of online softmax (CFR-Atlas page, "exact
//    folded online-softmax attention pass"; ARGUS page, "page-by-page online
//    softmax"); (3) acc = acc*alpha + sum_t p_t*scale_v*v_t, one warp per 64 / W
//    tokens, lanes across head_dim.  Quantised rows are expanded to fp32 in
//    registers only (ARGUS page, "Transient FP16 Reconstruction ... in GPU
//    SRAM"); scales multiply the dot product and p, never the stored codes.
//  - At the end of an item the W warps' accumulators are summed in a fixed
//    order and (m, l, acc) is written as the split's partial for the merge.
//
// Tokens past the sequence length, tokens outside a sink + recent-window subset
// and rows of skipped pages get p = 0 and are never read, so stale or NaN
// shared-memory bytes cannot reach an FMA.
#include "cfr_common.cuh"

namespace cfr {

constexpr int CC_T = 64;       // tokens per tile
// consumer warps W: 16 while the accumulators (GT x D / 32 floats per lane)
// leave room for them in the register file, else 8; one producer warp more
__host__ __device__ constexpr int cc_warps(int D, int GT) { return GT * D <= 512 ? 16 : 8; }
template <int W>
__host__ __device__ constexpr int cc_threads() { return (W + 1) * 32; }
constexpr int CC_MAXF = 16;    // fragments (page pieces) per tile; page_tokens >= 8 gives <= 9

// A page piece of a tile (the producer's view): tile rows [r0, r0 + rows of
// the piece) of one page, whose K rows sit packed at their own row size rb
// from byte `off` of the stage's K region (V rows likewise in the V region).
struct CcFrag {
  int fmt;
  int ok;
  float ks, vs;
  int off, rb, r0;
};

// Tile row r of a stage: its K row at byte `off` of the stage's K region (its
// V row at the same offset of the V region), format and readability, scales.
struct __align__(16) CcRow {
  int off;
  int fmt_ok;  // format | 256 when the row's page resolved (else the row is not read)
  float ks, vs;
};

struct CcStageMeta {
  CcRow row[CC_T];
  int rows;
  int t0;
};

template <int W>
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(W * 32) : "memory");
}

// N consecutive elements starting at element e0 of a stored row, widened to fp32
// (codes for quantised formats; the scale is applied by the caller).
template <int N>
__device__ __forceinline__ void load_elems(int fmt, const uint8_t *row, int e0, float (&x)[N]) {
  if (fmt == CFR_FMT_F32) {
    const float4 *p = reinterpret_cast<const float4 *>(row + 4 * e0);
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const float4 v = p[i];
      x[4 * i] = v.x;
      x[4 * i + 1] = v.y;
      x[4 * i + 2] = v.z;
      x[4 * i + 3] = v.w;
    }
    if constexpr (N % 4 == 2) {
      const float2 v = *reinterpret_cast<const float2 *>(row + 4 * e0 + 4 * (N - 2));
      x[N - 2] = v.x;
      x[N - 1] = v.y;
    }
  } else if (fmt == CFR_FMT_BF16) {
    const uint8_t *p = row + 2 * e0;
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N / 8; ++i) {
        const uint4 w = reinterpret_cast<const uint4 *>(p)[i];
        const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x[8 * i + 2 * k] = bf16_lo(a[k]);
          x[8 * i + 2 * k + 1] = bf16_hi(a[k]);
        }
      }
    } else if constexpr (N == 4) {
      const uint2 w = *reinterpret_cast<const uint2 *>(p);
      x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
      x[0] = bf16_lo(w); x[1] = bf16_hi(w);
    }
  } else if (fmt == CFR_FMT_I8) {
    const uint8_t *p = row + e0;
    if constexpr (N % 16 == 0) {
#pragma unroll
      for (int i = 0; i < N / 16; ++i) {
        const uint4 w = reinterpret_cast<const uint4 *>(p)[i];
        const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 16; ++k) x[16 * i + k] = i8_at(a[k / 4], k % 4);
      }
    } else if constexpr (N == 8) {
      const uint2 w = *reinterpret_cast<const uint2 *>(p);
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = i8_at(k < 4 ? w.x : w.y, k % 4);
    } else if constexpr (N == 4) {
      const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = i8_at(w, k);
    } else {
      const uint32_t w = *reinterpret_cast<const uint16_t *>(p);
      x[0] = i8_at(w, 0); x[1] = i8_at(w, 1);
    }
  } else if (fmt == CFR_FMT_FP8) {
    const uint8_t *p = row + e0;
    if constexpr (N % 16 == 0) {
#pragma unroll
      for (int i = 0; i < N / 16; ++i) {
        const uint4 w = reinterpret_cast<const uint4 *>(p)[i];
        const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 16; ++k) x[16 * i + k] = e4m3_at(a[k / 4], k % 4);
      }
    } else if constexpr (N == 8) {
      const uint2 w = *reinterpret_cast<const uint2 *>(p);
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = e4m3_at(k < 4 ? w.x : w.y, k % 4);
    } else if constexpr (N == 4) {
      const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = e4m3_at(w, k);
    } else {
      const uint32_t w = *reinterpret_cast<const uint16_t *>(p);
      x[0] = e4m3_at(w, 0); x[1] = e4m3_at(w, 1);
    }
  } else {  // CFR_FMT_I4
    const uint8_t *p = row + e0 / 2;
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N / 8; ++i) {
        const uint32_t w = reinterpret_cast<const uint32_t *>(p)[i];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[8 * i + k] = i4_at(w, k);
      }
    } else if constexpr (N == 4) {
      const uint32_t w = *reinterpret_cast<const uint16_t *>(p);
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = i4_at(w, k);
    } else {
      const uint32_t w = *p;
      x[0] = i4_at(w, 0); x[1] = i4_at(w, 1);
    }
  }
}

struct CcLayout {
  uint64_t *full, *empty;
  CcStageMeta *meta;
  float *q_s;      // [GT][D]
  float *sc;       // [2][GT][T]
  float *alpha;    // [2][GT]
  float *slope2;   // [GT] slope * log2(e)
  int *qoff;       // [GT] causal offset of each query row
  float *red;      // [W][4][D]
  int *flag;       // [1] wait outcome broadcast
  uint8_t *ring;   // [stages][2][T][pitch]
};

template <int D, int GT>
__host__ __device__ inline size_t cc_fixed_bytes(int stages) {
  constexpr int W = cc_warps(D, GT);
  size_t o = 0;
  o += 2 * stages * sizeof(uint64_t);
  o = (o + 15) & ~size_t(15);
  o += stages * sizeof(CcStageMeta);
  o = (o + 15) & ~size_t(15);
  o += GT * D * 4 + 2 * GT * CC_T * 4 + 2 * GT * 4 + GT * 4 + GT * 4 + W * 4 * D * 4 + 16;
  o = (o + 127) & ~size_t(127);
  return o;
}

template <int D, int GT>
__device__ inline CcLayout cc_layout(uint8_t *smem, int stages, int pitch) {
  constexpr int W = cc_warps(D, GT);
  CcLayout L;
  size_t o = 0;
  L.full = reinterpret_cast<uint64_t *>(smem);
  L.empty = L.full + stages;
  o += 2 * stages * sizeof(uint64_t);
  o = (o + 15) & ~size_t(15);
  L.meta = reinterpret_cast<CcStageMeta *>(smem + o);
  o += stages * sizeof(CcStageMeta);
  o = (o + 15) & ~size_t(15);
  L.q_s = reinterpret_cast<float *>(smem + o);
  o += GT * D * 4;
  L.sc = reinterpret_cast<float *>(smem + o);
  o += 2 * GT * CC_T * 4;
  L.alpha = reinterpret_cast<float *>(smem + o);
  o += 2 * GT * 4;
  L.slope2 = reinterpret_cast<float *>(smem + o);
  o += GT * 4;
  L.qoff = reinterpret_cast<int *>(smem + o);
  o += GT * 4;
  L.red = reinterpret_cast<float *>(smem + o);
  o += W * 4 * D * 4;
  L.flag = reinterpret_cast<int *>(smem + o);
  o += 16;
  o = (o + 127) & ~size_t(127);
  L.ring = smem + o;
  (void)pitch;
  return L;
}

// Producer (warp 8): every tile of every item of this CTA.  Lane i resolves
// piece i of the tile, so a tile's page-table reads are one round trip.
template <int D>
__device__ void cc_producer(const DecodeParams &p, const CcLayout &L, long long nitems,
                            bool *timed_out) {
  const int lane = threadIdx.x & 31;
  int stage = 0;
  uint32_t phase = 0;
  const int P = p.P;
  for (long long item = blockIdx.x; item < nitems; item += gridDim.x) {
    int slot, g;
    item_coords(item, static_cast<int>(nitems / p.ngroups), p.gsub, slot, g);
    const SplitRange sr = split_at(p, slot);
    const int b = sr.b, pb = sr.pb, pe = sr.pe;
    const int n = p.seq_lens[b];
    const int tok_end = min(n, pe * p.split_unit);
    for (int t0 = pb * p.split_unit; t0 < tok_end; t0 += CC_T) {
      const int rows = min(CC_T, tok_end - t0);
      // piece `lane`: tile rows [r0, r1) of page pg
      const int pg = t0 / P + lane;
      const int r0 = max(t0, pg * P) - t0;
      const int r1 = min(t0 + rows, (pg + 1) * P) - t0;
      const bool have = lane < CC_MAXF && r0 < r1;
      CcFrag f;
      f.fmt = -1;
      f.ok = 0;
      f.ks = f.vs = 1.f;
      f.rb = 0;
      f.r0 = r0;
      long long id = -1;
      if (have) {
        const long long cell = static_cast<long long>(b) * p.max_pages + pg;
        f.fmt = p.page_fmt ? static_cast<int>(p.page_fmt[cell]) : p.uniform_fmt;
        id = p.page_table[cell];
        if (f.fmt < 0 || f.fmt >= kFmtCount) {
          set_err(p.err, CFR_DEVERR_PAGE_FMT);
        } else if (!p.k_pool[f.fmt] || !p.v_pool[f.fmt] || (is_quantised(f.fmt) && !p.scales[f.fmt])) {
          set_err(p.err, CFR_DEVERR_POOL);
        } else if (id < 0 || id >= p.pool_pages[f.fmt]) {
          set_err(p.err, CFR_DEVERR_PAGE_ID);
        } else {
          f.ok = 1;
          f.rb = row_bytes(f.fmt, D);
          if (is_quantised(f.fmt)) {
            const float2 s = *reinterpret_cast<const float2 *>(p.scales[f.fmt] + (id * p.Hkv + p.grp_kv[g]) * 2);
            f.ks = s.x;
            f.vs = s.y;
          }
        }
      }
      // packed byte offsets of the pieces in the K (and V) region: an
      // exclusive prefix sum over the lanes (every row size is a multiple of 16)
      const uint32_t pbytes = f.ok ? static_cast<uint32_t>((r1 - r0) * f.rb) : 0u;
      uint32_t incl = pbytes;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      f.off = static_cast<int>(incl - pbytes);
      const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
      // the stage must be free before its description and bytes are replaced
      const bool waited = mbar_wait(&L.empty[stage], phase ^ 1u, p.err, timed_out);
      if (!__all_sync(0xffffffffu, waited)) return;
      CcStageMeta &m = L.meta[stage];
      uint8_t *kst = L.ring + static_cast<size_t>(stage) * 2 * CC_T * p.pitch;
      uint8_t *vst = kst + CC_T * p.pitch;
      if (have) {
        CcRow rw;
        rw.fmt_ok = f.ok ? (f.fmt | 256) : 0;
        rw.ks = f.ks;
        rw.vs = f.vs;
        for (int r = r0; r < r1; ++r) {
          rw.off = f.off + (r - r0) * f.rb;
          m.row[r] = rw;
        }
      }
      if (lane == 0) {
        m.rows = rows;
        m.t0 = t0;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&L.full[stage], 2u * total);
      __syncwarp();
      if (f.ok) {
        const long long off = ((id * p.Hkv + p.grp_kv[g]) * P + (t0 + r0 - pg * P)) * f.rb;
        bulk_g2s(kst + f.off, p.k_pool[f.fmt] + off, pbytes, &L.full[stage]);
        bulk_g2s(vst + f.off, p.v_pool[f.fmt] + off, pbytes, &L.full[stage]);
      }
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
}

template <int D, int GT>
__device__ void cc_consumer(const DecodeParams &p, const CcLayout &L, long long nitems,
                            bool *timed_out) {
  constexpr int W = cc_warps(D, GT);      // consumer warps
  constexpr int HK = (16 + W - 1) / W;    // query rows per warp in the fold
  constexpr int EPT = D / 8;    // elements per thread in the score step (8 lanes per row)
  constexpr int DPL = D / 32;   // dims per lane in the P.V step
  constexpr int HC = GT < 4 ? GT : 4;  // heads per reduction round
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int stage = 0;
  uint32_t phase = 0;
  int tile_ctr = 0;

  for (long long item = blockIdx.x; item < nitems; item += gridDim.x) {
    int slot, g;
    item_coords(item, static_cast<int>(nitems / p.ngroups), p.gsub, slot, g);
    const SplitRange sr = split_at(p, slot);
    const int b = sr.b, pb = sr.pb, pe = sr.pe;
    const int n = p.seq_lens[b];
    const int tok_end = min(n, pe * p.split_unit);
    const int h0 = p.grp_off[g], cnt = p.grp_off[g + 1] - h0;

    // the group's queries (fp32) and ALiBi slopes
    for (int i = tid; i < GT * D; i += W * 32) {
      const int hh = i / D, e = i - hh * D;
      float v = 0.f;
      if (hh < cnt) {
        const long long qi = (static_cast<long long>(b) * p.Hq + p.grp_heads[h0 + hh]) * D + e;
        v = p.q_fmt == CFR_FMT_F32 ? static_cast<const float *>(p.q)[qi]
                                   : __uint_as_float(static_cast<uint32_t>(
                                         static_cast<const uint16_t *>(p.q)[qi]) << 16);
      }
      L.q_s[i] = v;
    }
    if (tid < GT) {
      L.slope2[tid] =
          (p.slopes && tid < cnt) ? p.slopes[row_head(p, p.grp_heads[h0 + tid])] * kLog2e : 0.f;
      L.qoff[tid] = tid < cnt ? row_offset(p, p.grp_heads[h0 + tid]) : 0;
    }
    consumers_sync<W>();
    // this lane's query elements of the score step (8 lanes per token row,
    // EPT dims each), in registers while they fit beside the accumulators
    constexpr bool kQRegs = GT * EPT * (D / 64) <= 32;
    float qr[kQRegs ? GT : 1][kQRegs ? EPT : 1];
    if constexpr (kQRegs) {
#pragma unroll
      for (int h = 0; h < GT; ++h)
#pragma unroll
        for (int i = 0; i < EPT; ++i) qr[h][i] = L.q_s[h * D + (lane & 7) * EPT + i];
    }

    float acc[GT][DPL];
#pragma unroll
    for (int h = 0; h < GT; ++h)
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[h][i] = 0.f;
    float m_run[HK], l_run[HK];
#pragma unroll
    for (int k = 0; k < HK; ++k) {
      m_run[k] = -INFINITY;
      l_run[k] = 0.f;
    }

    for (int t0 = pb * p.split_unit; t0 < tok_end; t0 += CC_T) {
      // one thread waits (bounded); the outcome is broadcast so all warps agree
      if (tid == 0) *L.flag = mbar_wait(&L.full[stage], phase, p.err, timed_out) ? 1 : 0;
      consumers_sync<W>();
      if (*L.flag == 0) {
        *timed_out = true;
        return;
      }
      (void)mbar_try_wait(&L.full[stage], phase);  // acquire the copied bytes in every thread
      const CcStageMeta &m = L.meta[stage];
      const uint8_t *kst = L.ring + static_cast<size_t>(stage) * 2 * CC_T * p.pitch;
      const uint8_t *vst = kst + CC_T * p.pitch;
      float *sc = L.sc + (tile_ctr & 1) * GT * CC_T;
      float *al = L.alpha + (tile_ctr & 1) * GT;
      const int rows = m.rows;

      // (1) scores, base 2
#pragma unroll
      for (int pass = 0; pass < CC_T / (4 * W); ++pass) {
        const int r = pass * 4 * W + warp * 4 + (lane >> 3), j8 = lane & 7;
        float dot[GT];
#pragma unroll
        for (int h = 0; h < GT; ++h) dot[h] = 0.f;
        bool valid = false;
        float ks = 1.f;
        if (r < rows) {
          const CcRow rw = m.row[r];
          if ((rw.fmt_ok & 256) && in_token_set(p, n, m.t0 + r)) {
            valid = true;
            ks = rw.ks;
            float x[EPT];
            load_elems<EPT>(rw.fmt_ok & 255, kst + rw.off, j8 * EPT, x);
#pragma unroll
            for (int h = 0; h < GT; ++h) {
              if constexpr (kQRegs) {
#pragma unroll
                for (int i = 0; i < EPT; ++i) dot[h] = fmaf(qr[h][i], x[i], dot[h]);
              } else {
                const float4 *qq = reinterpret_cast<const float4 *>(L.q_s + h * D + j8 * EPT);
#pragma unroll
                for (int i = 0; i < EPT / 4; ++i) {
                  const float4 q4 = qq[i];
                  dot[h] = fmaf(q4.x, x[4 * i], dot[h]);
                  dot[h] = fmaf(q4.y, x[4 * i + 1], dot[h]);
                  dot[h] = fmaf(q4.z, x[4 * i + 2], dot[h]);
                  dot[h] = fmaf(q4.w, x[4 * i + 3], dot[h]);
                }
              }
            }
          }
        }
#pragma unroll
        for (int h = 0; h < GT; ++h) {
          dot[h] += __shfl_xor_sync(0xffffffffu, dot[h], 1);
          dot[h] += __shfl_xor_sync(0xffffffffu, dot[h], 2);
          dot[h] += __shfl_xor_sync(0xffffffffu, dot[h], 4);
        }
        if (r < CC_T) {
#pragma unroll
          for (int h = 0; h < GT; ++h)
            if ((h & 7) == j8) {
              // query row h sits at position n - 1 - qoff[h] and sees tokens up to it
              const int dist = n - 1 - L.qoff[h] - (m.t0 + r);
              sc[h * CC_T + r] = (valid && dist >= 0) ? fmaf(dot[h] * ks, p.sigma_log2e,
                                                             -L.slope2[h] * static_cast<float>(dist))
                                                      : -INFINITY;
            }
        }
      }
      consumers_sync<W>();

      // (2) fold: tile max, rescale factor, probabilities, running normaliser
#pragma unroll
      for (int k = 0; k < HK; ++k) {
        const int hh = warp + W * k;
        if (hh < GT) {
          const float v0 = sc[hh * CC_T + lane], v1 = sc[hh * CC_T + lane + 32];
          float mt = fmaxf(v0, v1);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
          const float m_new = fmaxf(m_run[k], mt);
          float alpha = 1.f, p0 = 0.f, p1 = 0.f;
          if (m_new != -INFINITY) {
            alpha = exp2_approx(m_run[k] - m_new);
            p0 = exp2_approx(v0 - m_new);
            p1 = exp2_approx(v1 - m_new);
          }
          sc[hh * CC_T + lane] = p0;
          sc[hh * CC_T + lane + 32] = p1;
          float ls = p0 + p1;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
          l_run[k] = fmaf(l_run[k], alpha, ls);
          m_run[k] = m_new;
          if (lane == 0) al[hh] = alpha;
        }
      }
      consumers_sync<W>();

      // (3) acc = acc*alpha + sum_t p_t * scale_v * v_t over this warp's 8 tokens
#pragma unroll
      for (int h = 0; h < GT; ++h) {
        const float a = al[h];
        if (a != 1.f) {
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc[h][i] *= a;
        }
      }
#pragma unroll 2
      for (int rr = 0; rr < CC_T / W; ++rr) {
        const int r = warp * (CC_T / W) + rr;
        if (r >= rows) break;
        const CcRow rw = m.row[r];
        if (!(rw.fmt_ok & 256) || !in_token_set(p, n, m.t0 + r)) continue;
        float v[DPL];
        load_elems<DPL>(rw.fmt_ok & 255, vst + rw.off, lane * DPL, v);
#pragma unroll
        for (int h = 0; h < GT; ++h) {
          const float pw = sc[h * CC_T + r] * rw.vs;
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc[h][i] = fmaf(pw, v[i], acc[h][i]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&L.empty[stage]);
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1u;
      }
      ++tile_ctr;
    }

    // split partial: (m, l) from the fold warps, acc summed over the 8 warps
    float *pa = p.part_acc + static_cast<long long>(slot) * p.Hq * D;
#pragma unroll
    for (int c0 = 0; c0 < GT; c0 += HC) {
      consumers_sync<W>();
#pragma unroll
      for (int hh = 0; hh < HC; ++hh)
#pragma unroll
        for (int i = 0; i < DPL; ++i) L.red[(warp * HC + hh) * D + lane * DPL + i] = acc[c0 + hh][i];
      consumers_sync<W>();
      for (int e = tid; e < HC * D; e += W * 32) {
        const int hh = e / D, i = e - hh * D;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) s += L.red[(w * HC + hh) * D + i];
        if (c0 + hh < cnt) pa[static_cast<long long>(p.grp_heads[h0 + c0 + hh]) * D + i] = s;
      }
    }
#pragma unroll
    for (int k = 0; k < HK; ++k) {
      const int hh = warp + W * k;
      if (hh < GT && hh < cnt && lane == 0) {
        const long long c = static_cast<long long>(slot) * p.Hq + p.grp_heads[h0 + hh];
        p.part_m[c] = m_run[k];
        p.part_l[c] = l_run[k];
      }
    }
    consumers_sync<W>();
  }
}

template <int D, int GT>
__global__ void __launch_bounds__(cc_threads<cc_warps(D, GT)>(), 1)
    cc_decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int W = cc_warps(D, GT);
  extern __shared__ __align__(128) uint8_t smem[];
  const CcLayout L = cc_layout<D, GT>(smem, p.stages, p.pitch);
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&L.full[s], 1);
      mbar_init(&L.empty[s], W);
    }
    fence_mbar_init();
  }
  griddep_launch_dependents();
  __syncthreads();
  griddep_wait();  // the split schedule comes from the previous kernel
  const long long nitems =
      static_cast<long long>(schedule_split_count(p, threadIdx.x == 0 && blockIdx.x == 0)) * p.ngroups;
  bool timed_out = false;
  if (threadIdx.x >= W * 32) {
    cc_producer<D>(p, L, nitems, &timed_out);
  } else {
    cc_consumer<D, GT>(p, L, nitems, &timed_out);
  }
}

template <int D, int GT>
static cudaError_t cc_launch_t(const DecodeParams &p, int grid, cudaStream_t stream) {
  const size_t smem = cc_fixed_bytes<D, GT>(p.stages) +
                      static_cast<size_t>(p.stages) * 2 * CC_T * p.pitch;
  cudaError_t e = cudaFuncSetAttribute(cc_decode_kernel<D, GT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = launch_after_previous(cc_decode_kernel<D, GT>, dim3(grid), dim3(cc_threads<cc_warps(D, GT)>()), smem,
                            stream, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Number of ring stages that fit next to the fixed shared-memory part.
int cc_stages(int D, int gt, int pitch, size_t smem_limit) {
  size_t fixed = 0;
  const size_t stage = static_cast<size_t>(2) * CC_T * pitch;
  for (int s = 8; s >= 2; --s) {
#define CFR_FIX(DD, GG) \
  if (D == DD && gt == GG) fixed = cc_fixed_bytes<DD, GG>(s);
    CFR_FIX(64, 1) CFR_FIX(64, 2) CFR_FIX(64, 4) CFR_FIX(64, 8) CFR_FIX(64, 16)
    CFR_FIX(128, 1) CFR_FIX(128, 2) CFR_FIX(128, 4) CFR_FIX(128, 8) CFR_FIX(128, 16)
#undef CFR_FIX
    if (fixed + s * stage <= smem_limit) return s;
  }
  return 0;
}

int cc_group_tile(int gmax) {
  return gmax <= 1 ? 1 : gmax <= 2 ? 2 : gmax <= 4 ? 4 : gmax <= 8 ? 8 : 16;
}

cudaError_t launch_decode_cc(const DecodeParams &p, int grid, cudaStream_t stream) {
  const int gt = cc_group_tile(p.gmax);
#define CFR_CASE(DD, GG) \
  if (p.D == DD && gt == GG) return cc_launch_t<DD, GG>(p, grid, stream);
  CFR_CASE(64, 1) CFR_CASE(64, 2) CFR_CASE(64, 4) CFR_CASE(64, 8) CFR_CASE(64, 16)
  CFR_CASE(128, 1) CFR_CASE(128, 2) CFR_CASE(128, 4) CFR_CASE(128, 8) CFR_CASE(128, 16)
#undef CFR_CASE
  return cudaErrorInvalidValue;
}

}  // namespace cfr
