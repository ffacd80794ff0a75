// cfr_decode_f32.cu -- split-KV paged decode attention for fp32 K/V pages (CUDA cores).
//
// The fp32 cache has 0.5 flop per byte at one query head per kv head, far
// below any ALU limit, so the kernel is built to move bytes: every K/V tile is
// fetched by the TMA engine as 128-byte-wide boxes of the pool (2-D tensor
// map, 128-byte swizzle) into a three-stage shared-memory ring, and each
// element then costs about one FMA plus a quarter of a 16-byte shared load.
// fp32 products are kept in fp32 (tensor cores would round K to tf32).
//
// Work item = (split of one sequence, kv head) with its G <= 2 query heads;
// one persistent CTA per SM walks its items.
//  - warp 8 lane 0 (producer): resolves each page of the tile through the page
//    table (slot, format, pool checks; bad pages are skipped and reported),
//    issues the TMA boxes, records which rows hold valid tokens.
//  - warps 0-7 (consumers), per tile of T = 8192/d tokens:
//      scores  thread = (row, 128-byte column block): eight swizzled 16-byte
//              loads, dot with its 32 query values kept in registers, one or
//              two shuffles across the blocks of the row; base-2 logits with
//              ALiBi added from the integer distance n-1-j.
//      fold    one warp per head: tile max, rescale 2^(m_old-m_new), p = 2^(s-m),
//              running normaliser -- the exact online-softmax fold of the
//              CFR-Atlas page ("exact folded online-softmax attention pass").
//      P.V     thread = (4-dim chunk, group of 8 tokens): acc = acc*alpha + sum p*v.
//  - item end: accumulators of the token groups are summed in a fixed order
//    and (m, l, acc) is written as the split partial.
#include "cfr_tmap.cuh"

namespace cfr {

constexpr int F_WARPS = 8;
constexpr int F_THREADS = (F_WARPS + 1) * 32;
constexpr int F_STAGES = 3;

template <int D>
struct F32Cfg {
  static constexpr int T = 8192 / D;                   // tokens per tile
  static constexpr int NB = D / 32;                    // 128-byte column blocks per row
  static constexpr int BLOCK_BYTES = T * 128;          // one column block of one tile
  static constexpr int TILE_BYTES = NB * BLOCK_BYTES;  // K (or V) tile: 32 KiB
  static constexpr int NCH = D / 4;                    // 16-byte chunks per row
  static constexpr int TG = F_WARPS * 32 / NCH;        // token groups of the P.V step
  static constexpr int TPG = T / TG;                   // tokens per group (8)
  static_assert(TPG == 8, "eight tokens per group");
};

struct F32Meta {
  uint32_t valid[4];  // bit r: row r holds a token of a resolved page
  int rows;
  int t0;
};

struct F32Maps {
  CUtensorMap k;
  CUtensorMap v;
};

__device__ __forceinline__ void f_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(F_WARPS * 32) : "memory");
}

template <int D, int GT>
struct F32Smem {
  uint64_t full[F_STAGES], empty[F_STAGES];
  F32Meta meta[F_STAGES];
  alignas(16) float sc[2][GT][F32Cfg<D>::T];
  alignas(16) float alpha[2][GT];
  alignas(16) float red[F_WARPS][GT][D];
  int flag;
  PageCache pc;
};

template <int D, int GT>
__host__ __device__ constexpr size_t f32_ring_offset() {
  return (sizeof(F32Smem<D, GT>) + 1023) / 1024 * 1024;
}

// shared memory asked for at launch: the struct, the ring, and 1 KiB of slack so
// the ring can start on a 1024-byte boundary (the 128-byte swizzle atom)
template <int D, int GT>
__host__ __device__ constexpr size_t f32_smem_bytes() {
  return f32_ring_offset<D, GT>() + static_cast<size_t>(F_STAGES) * 2 * F32Cfg<D>::TILE_BYTES + 1024;
}

// one tile of the producer warp: lane f resolves page
// piece f of the tile and issues its boxes; lane 0 publishes which rows are valid
// and the expected byte count.  Pages are resolved before the wait for the
// stage, so that only the publication and the copies follow it.
template <int D>
__device__ __forceinline__ bool f32_produce_tile(const DecodeParams &p, const F32Maps &maps,
                                                 uint64_t *full, uint64_t *empty, F32Meta *meta,
                                                 uint8_t *ring, const PageCache &pc, int g, int n,
                                                 int t0, int tok_end, int box_rows, int stage,
                                                 uint32_t phase, bool *timed_out, int lane) {
  using C = F32Cfg<D>;
  const int P = p.P;
  const int rows = min(C::T, tok_end - t0);
  const int npiece = (rows + box_rows - 1) / box_rows;  // <= 16
  bool pvalid = false;
  long long id = 0;
  const int r = lane * box_rows;
  if (lane < npiece) {
    const int pg = (t0 + r) / P;
    const int fmt = pc.fmt[pg - pc.base];
    id = pc.id[pg - pc.base];
    if (fmt != CFR_FMT_F32) {
      set_err(p.err, fmt >= 0 && fmt < kFmtCount ? CFR_DEVERR_POOL : CFR_DEVERR_PAGE_FMT);
    } else if (id < 0 || id >= p.pool_pages[CFR_FMT_F32]) {
      set_err(p.err, CFR_DEVERR_PAGE_ID);
    } else {
      pvalid = true;
    }
  }
  const uint32_t vb = __ballot_sync(0xffffffffu, pvalid);
  uint32_t valid[4] = {0u, 0u, 0u, 0u};
  if (lane == 0) {
    for (int f = 0; f < npiece; ++f)
      if ((vb >> f) & 1u) mask_set_range(valid, f * box_rows, min(rows, (f + 1) * box_rows));
    mask_clear_gap(valid, p, n, t0, rows);  // tokens between the sinks and the recent window
  }
  // the stage is needed only from here on
  int ok = 1;
  if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1u, p.err, timed_out) ? 1 : 0;
  if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
  if (lane == 0) {
    F32Meta &m = meta[stage];
    for (int w = 0; w < 4; ++w) m.valid[w] = valid[w];
    m.rows = rows;
    m.t0 = t0;
    mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(__popc(vb)) * 2u * C::NB * box_rows * 128u);
  }
  if (pvalid) {
    uint8_t *kst = ring + static_cast<size_t>(stage) * 2 * C::TILE_BYTES;
    uint8_t *vst = kst + C::TILE_BYTES;
    const int tin = (t0 + r) % P;
    const int y = static_cast<int>((id * p.Hkv + p.grp_kv[g]) * P + tin);
#pragma unroll
    for (int blk = 0; blk < C::NB; ++blk) {
      tma_load_2d(kst + blk * C::BLOCK_BYTES + r * 128, &maps.k, 32 * blk, y, &full[stage]);
      tma_load_2d(vst + blk * C::BLOCK_BYTES + r * 128, &maps.v, 32 * blk, y, &full[stage]);
    }
  }
  return true;
}

// Producer warp: all 32 lanes keep the page-table cache filled and issue the
// boxes of each tile together.
template <int D>
__device__ void f32_producer(const DecodeParams &p, const F32Maps &maps, uint64_t *full,
                             uint64_t *empty, F32Meta *meta, uint8_t *ring, PageCache &pc,
                             long long nitems, bool *timed_out) {
  using C = F32Cfg<D>;
  const int P = p.P;
  const int lane = threadIdx.x & 31;
  const int box_rows = P < C::T ? P : C::T;
  int stage = 0;
  uint32_t phase = 0;
  if (lane == 0) {
    prefetch_map(&maps.k);
    prefetch_map(&maps.v);
  }
  page_cache_reset(pc, lane);
  for (long long item = blockIdx.x; item < nitems; item += gridDim.x) {
    int slot, g;
    item_coords(item, static_cast<int>(nitems / p.ngroups), p.gsub, slot, g);
    const SplitRange sr = split_at(p, slot);
    const int b = sr.b, pb = sr.pb, pe = sr.pe;
    const int n = p.seq_lens[b];
    const int U = p.split_unit;
    const int tok_end = min(n, pe * U);
    const int pg_end = U == P ? pe : (pe * U + P - 1) / P;  // pages the split reaches into
    for (int t0 = pb * U; t0 < tok_end; t0 += C::T) {
      page_cache_ensure(pc, p, b, t0 / P, (min(t0 + C::T, tok_end) - 1) / P, pg_end, lane);
      if (!f32_produce_tile<D>(p, maps, full, empty, meta, ring, pc, g, n, t0, tok_end, box_rows,
                               stage, phase, timed_out, lane))
        return;
      if (++stage == F_STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
}

template <int D, int GT>
__device__ void f32_consumer(const DecodeParams &p, F32Smem<D, GT> &S, uint8_t *ring,
                             long long nitems, bool *timed_out) {
  using C = F32Cfg<D>;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // score step: row and 128-byte block of this thread (8 consecutive lanes share a block)
  const int q_row = (D == 64) ? warp * 16 + (lane & 7) + 8 * (lane >> 4) : warp * 8 + (lane & 7);
  const int q_blk = (D == 64) ? (lane >> 3) & 1 : (lane >> 3);
  // P.V step: 16-byte chunk and token group of this thread
  const int v_chk = (D == 64) ? (lane & 15) : lane;
  const int v_grp = (D == 64) ? warp * 2 + (lane >> 4) : warp;
  const int P = p.P;
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

    float q[GT][32];
    float slope2[GT];
    int qoff[GT];  // causal offset of each query row (0 with one query per sequence)
#pragma unroll
    for (int h = 0; h < GT; ++h) {
      slope2[h] = 0.f;
      qoff[h] = 0;
      if (h < cnt) {
        const int head = p.grp_heads[h0 + h];
        const long long base = (static_cast<long long>(b) * p.Hq + head) * D + 32 * q_blk;
        if (p.q_fmt == CFR_FMT_F32) {
          const float4 *qp = reinterpret_cast<const float4 *>(static_cast<const float *>(p.q) + base);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 v = qp[i];
            q[h][4 * i] = v.x; q[h][4 * i + 1] = v.y; q[h][4 * i + 2] = v.z; q[h][4 * i + 3] = v.w;
          }
        } else {
          const uint4 *qp = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.q) + base);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 w = qp[i];
            const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              q[h][8 * i + 2 * k] = bf16_lo(a[k]);
              q[h][8 * i + 2 * k + 1] = bf16_hi(a[k]);
            }
          }
        }
        if (p.slopes) slope2[h] = p.slopes[row_head(p, head)] * kLog2e;
        qoff[h] = row_offset(p, head);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) q[h][i] = 0.f;
      }
    }

    float acc[GT][4];
#pragma unroll
    for (int h = 0; h < GT; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[h][i] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;  // of head `warp` (warps < GT)

    for (int t0 = pb * p.split_unit; t0 < tok_end; t0 += C::T) {
      if (tid == 0) S.flag = mbar_wait(&S.full[stage], phase, p.err, timed_out) ? 1 : 0;
      f_sync();
      if (S.flag == 0) {
        *timed_out = true;
        return;
      }
      (void)mbar_try_wait(&S.full[stage], phase);
      const F32Meta &m = S.meta[stage];
      const uint8_t *kst = ring + static_cast<size_t>(stage) * 2 * C::TILE_BYTES;
      const uint8_t *vst = kst + C::TILE_BYTES;
      float(*sc)[C::T] = S.sc[tile_ctr & 1];
      float *al = S.alpha[tile_ctr & 1];

      // scores
      {
        const uint8_t *row = kst + q_blk * C::BLOCK_BYTES;
        float dot[GT];
#pragma unroll
        for (int h = 0; h < GT; ++h) dot[h] = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 x = *reinterpret_cast<const float4 *>(row + sw128(q_row, c));
#pragma unroll
          for (int h = 0; h < GT; ++h) {
            dot[h] = fmaf(q[h][4 * c], x.x, dot[h]);
            dot[h] = fmaf(q[h][4 * c + 1], x.y, dot[h]);
            dot[h] = fmaf(q[h][4 * c + 2], x.z, dot[h]);
            dot[h] = fmaf(q[h][4 * c + 3], x.w, dot[h]);
          }
        }
#pragma unroll
        for (int h = 0; h < GT; ++h) {
          dot[h] += __shfl_xor_sync(0xffffffffu, dot[h], 8);
          if (D == 128) dot[h] += __shfl_xor_sync(0xffffffffu, dot[h], 16);
        }
        if (q_blk == 0) {
          const bool valid = (m.valid[q_row >> 5] >> (q_row & 31)) & 1u;
          const int j = m.t0 + q_row;
#pragma unroll
          for (int h = 0; h < GT; ++h) {
            // query row h sits at position n - 1 - qoff[h] and sees tokens up to it
            const int dist = n - 1 - qoff[h] - j;
            sc[h][q_row] = (valid && dist >= 0)
                               ? fmaf(dot[h], p.sigma_log2e, -slope2[h] * static_cast<float>(dist))
                               : -INFINITY;
          }
        }
      }
      f_sync();

      // fold: warp h owns head h
      if (warp < GT) {
        constexpr int PER = C::T / 32;
        float v[PER];
        float mt = -INFINITY;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
          v[k] = sc[warp][lane + 32 * k];
          mt = fmaxf(mt, v[k]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
        const float m_new = fmaxf(m_run, mt);
        float alpha = 1.f, ls = 0.f;
        if (m_new != -INFINITY) {
          alpha = exp2_approx(m_run - m_new);
#pragma unroll
          for (int k = 0; k < PER; ++k) {
            v[k] = exp2_approx(v[k] - m_new);
            ls += v[k];
          }
        } else {
#pragma unroll
          for (int k = 0; k < PER; ++k) v[k] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < PER; ++k) sc[warp][lane + 32 * k] = v[k];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
        l_run = fmaf(l_run, alpha, ls);
        m_run = m_new;
        if (lane == 0) al[warp] = alpha;
      }
      f_sync();

      // P.V over this thread's 8 tokens and 4 dims
#pragma unroll
      for (int h = 0; h < GT; ++h) {
        const float a = al[h];
        if (a != 1.f) {
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[h][i] *= a;
        }
      }
      {
        const int tb = v_grp * 8;
        const uint32_t vbits = (m.valid[tb >> 5] >> (tb & 31)) & 0xFFu;
        float pw[GT][8];
#pragma unroll
        for (int h = 0; h < GT; ++h) {
          const float4 a = *reinterpret_cast<const float4 *>(&sc[h][tb]);
          const float4 c = *reinterpret_cast<const float4 *>(&sc[h][tb + 4]);
          pw[h][0] = a.x; pw[h][1] = a.y; pw[h][2] = a.z; pw[h][3] = a.w;
          pw[h][4] = c.x; pw[h][5] = c.y; pw[h][6] = c.z; pw[h][7] = c.w;
        }
        const uint8_t *vb = vst + (v_chk >> 3) * C::BLOCK_BYTES;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (!((vbits >> k) & 1u)) continue;
          const float4 x = *reinterpret_cast<const float4 *>(vb + sw128(tb + k, v_chk & 7));
#pragma unroll
          for (int h = 0; h < GT; ++h) {
            acc[h][0] = fmaf(pw[h][k], x.x, acc[h][0]);
            acc[h][1] = fmaf(pw[h][k], x.y, acc[h][1]);
            acc[h][2] = fmaf(pw[h][k], x.z, acc[h][2]);
            acc[h][3] = fmaf(pw[h][k], x.w, acc[h][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[stage]);
      if (++stage == F_STAGES) {
        stage = 0;
        phase ^= 1u;
      }
      ++tile_ctr;
    }

    // split partial: sum the token groups in a fixed order
    if (D == 64) {
#pragma unroll
      for (int h = 0; h < GT; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][i] += __shfl_xor_sync(0xffffffffu, acc[h][i], 16);
    }
    f_sync();
    if (D == 128 || lane < 16) {
#pragma unroll
      for (int h = 0; h < GT; ++h)
        *reinterpret_cast<float4 *>(&S.red[warp][h][4 * v_chk]) =
            make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
    }
    f_sync();
    for (int e = tid; e < GT * D; e += F_WARPS * 32) {
      const int h = e / D, i = e - h * D;
      if (h < cnt) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < F_WARPS; ++w) s += S.red[w][h][i];
        p.part_acc[(static_cast<long long>(slot) * p.Hq + p.grp_heads[h0 + h]) * D + i] = s;
      }
    }
    if (warp < GT && warp < cnt && lane == 0) {
      const long long c = static_cast<long long>(slot) * p.Hq + p.grp_heads[h0 + warp];
      p.part_m[c] = m_run;
      p.part_l[c] = l_run;
    }
    f_sync();
  }
}

template <int D, int GT>
__global__ void __launch_bounds__(F_THREADS, 1)
    f32_decode_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ F32Maps maps) {
  extern __shared__ __align__(1024) uint8_t smem[];
  F32Smem<D, GT> &S = *reinterpret_cast<F32Smem<D, GT> *>(smem);
  const uint32_t raw = smem_u32(smem + f32_ring_offset<D, GT>());
  uint8_t *ring = smem + f32_ring_offset<D, GT>() + ((1024u - (raw & 1023u)) & 1023u);
  if (threadIdx.x == 0) {
    for (int s = 0; s < F_STAGES; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], F_WARPS);
    }
    fence_mbar_init();
  }
  griddep_launch_dependents();
  __syncthreads();
  griddep_wait();  // the split schedule comes from the previous kernel
  const long long nitems =
      static_cast<long long>(schedule_split_count(p, threadIdx.x == 0 && blockIdx.x == 0)) * p.ngroups;
  bool timed_out = false;
  if (threadIdx.x >= F_WARPS * 32) {
    f32_producer<D>(p, maps, S.full, S.empty, S.meta, ring, S.pc, nitems, &timed_out);
  } else {
    f32_consumer<D, GT>(p, S, ring, nitems, &timed_out);
  }
}

bool f32_supported(const DecodeParams &p, bool page_fmt_given) {
  if (p.D != 64 && p.D != 128) return false;
  if (p.gmax > 2) return false;
  if (!p.k_pool[CFR_FMT_F32]) return false;
  if (page_fmt_given) {
    for (int f = 0; f < kFmtCount; ++f)
      if (f != CFR_FMT_F32 && p.k_pool[f]) return false;
  } else if (p.uniform_fmt != CFR_FMT_F32) {
    return false;
  }
  const int T = 8192 / p.D;
  if (!((p.P < T && T % p.P == 0) || p.P % T == 0)) return false;
  const long long rows = p.pool_pages[CFR_FMT_F32] * p.Hkv * static_cast<long long>(p.P);
  if (rows <= 0 || rows > 0x7fffffffLL) return false;
  if ((reinterpret_cast<uintptr_t>(p.q) & 15) != 0) return false;
  return true;
}

template <int D, int GT>
static cudaError_t f32_launch_t(const DecodeParams &p, int grid, cudaStream_t stream) {
  F32Maps maps;
  const long long rows = p.pool_pages[CFR_FMT_F32] * p.Hkv * static_cast<long long>(p.P);
  const int box_rows = p.P < F32Cfg<D>::T ? p.P : F32Cfg<D>::T;
  if (!encode_pool_map(&maps.k, p.k_pool[CFR_FMT_F32], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, rows, D,
                       box_rows) ||
      !encode_pool_map(&maps.v, p.v_pool[CFR_FMT_F32], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, rows, D,
                       box_rows))
    return cudaErrorInvalidValue;
  constexpr size_t smem = f32_smem_bytes<D, GT>();
  cudaError_t e = cudaFuncSetAttribute(f32_decode_kernel<D, GT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = launch_after_previous(f32_decode_kernel<D, GT>, dim3(grid), dim3(F_THREADS), smem, stream, p,
                            maps);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_decode_f32(const DecodeParams &p, int grid, cudaStream_t stream) {
  if (p.D == 64) return p.gmax <= 1 ? f32_launch_t<64, 1>(p, grid, stream) : f32_launch_t<64, 2>(p, grid, stream);
  return p.gmax <= 1 ? f32_launch_t<128, 1>(p, grid, stream) : f32_launch_t<128, 2>(p, grid, stream);
}

}  // namespace cfr
