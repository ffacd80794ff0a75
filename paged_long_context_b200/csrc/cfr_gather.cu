// cfr_gather.cu -- raw page gather: the page-table resolution of the decode
// kernels, copying stored row bytes out in token order (diagnostic).
//
// Token j of sequence b is row t = j mod P of logical page p = j / P, which
// lives in slot page_table[b][p] of the pool of format page_fmt[b][p]; the row
// of kv head g starts at byte ((slot * Hkv + g) * P + t) * row_bytes(fmt)
// (pages keyed by layer/head with a token range, stored row-major
// [token][head_dim]: CFR-Atlas page, "KvRegenerator").  Rows of pages that do
// not resolve are skipped and reported in the error word.
#include "cfr_common.cuh"

namespace cfr {

__global__ void gather_kernel(DecodeParams p, int b, int g, int n_tokens, uint8_t *k_out,
                              uint8_t *v_out, long long pitch) {
  const int chunks = p.D * 4 / 16;  // 16-byte pieces of the widest row
  const long long total = static_cast<long long>(n_tokens) * chunks;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(i / chunks), c = static_cast<int>(i % chunks);
    const int pg = j / p.P, t = j % p.P;
    const long long cell = static_cast<long long>(b) * p.max_pages + pg;
    const int fmt = p.page_fmt ? static_cast<int>(p.page_fmt[cell]) : p.uniform_fmt;
    if (fmt < 0 || fmt >= kFmtCount) {
      if (c == 0) set_err(p.err, CFR_DEVERR_PAGE_FMT);
      continue;
    }
    const long long slot = p.page_table[cell];
    if (!p.k_pool[fmt] || !p.v_pool[fmt]) {
      if (c == 0) set_err(p.err, CFR_DEVERR_POOL);
      continue;
    }
    if (slot < 0 || slot >= p.pool_pages[fmt]) {
      if (c == 0) set_err(p.err, CFR_DEVERR_PAGE_ID);
      continue;
    }
    const int rb = row_bytes(fmt, p.D);
    if (c * 16 >= rb) continue;
    const long long off = ((slot * p.Hkv + g) * p.P + t) * rb + c * 16;
    const uint4 kv = *reinterpret_cast<const uint4 *>(p.k_pool[fmt] + off);
    const uint4 vv = *reinterpret_cast<const uint4 *>(p.v_pool[fmt] + off);
    *reinterpret_cast<uint4 *>(k_out + j * pitch + c * 16) = kv;
    *reinterpret_cast<uint4 *>(v_out + j * pitch + c * 16) = vv;
  }
}

void launch_gather(const DecodeParams &p, int b, int g, int n_tokens, void *k_out, void *v_out,
                   long long pitch, cudaStream_t stream) {
  const long long total = static_cast<long long>(n_tokens) * (p.D * 4 / 16);
  long long blocks = (total + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) return;
  gather_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      p, b, g, n_tokens, static_cast<uint8_t *>(k_out), static_cast<uint8_t *>(v_out), pitch);
}

}  // namespace cfr
