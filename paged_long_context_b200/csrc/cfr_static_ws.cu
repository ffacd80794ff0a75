// cfr_static_ws.cu -- cfr_paged_decode for callers that cannot allocate device memory.
//
// Some callers only ever hand a kernel its inputs and outputs: plugin and
// operator interfaces that expose no workspace, code that runs where the
// framework owns every device allocation, or code that must not call
// cudaMalloc at the call site.  cfr_paged_decode needs caller-owned scratch
// (the split schedule and the per-split partials); this variant takes that
// scratch from a fixed array compiled into the library instead.
//
// The array is a file-scope __device__ object of CFR_STATIC_WORKSPACE_BYTES:
// every GPU that loads the library holds it until the process exits.  Host code
// cannot use the array's name as a device address, so the first call on each
// device looks the address up with cudaGetSymbolAddress (with that device
// current) and caches it; later calls on that device reuse the cached pointer.
// That first call should therefore happen before any stream capture.
//
// Every call shares the one array.  Nothing in it needs to start at zero: each
// call's schedule launch rewrites everything the later launches read.  Calls
// whose GPU work overlaps (on different streams) race on the array and must be
// serialised by the caller.
#include <mutex>

#include "cfr_common.cuh"

namespace {

constexpr int kMaxStaticDevices = 64;

static __device__ __align__(256) unsigned char g_static_workspace[CFR_STATIC_WORKSPACE_BYTES];

std::mutex g_static_mutex;
void *g_static_ptr[kMaxStaticDevices] = {nullptr};

// Device address of g_static_workspace on the current device (looked up once per device).
cfr_status static_workspace(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxStaticDevices)
    return CFR_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return CFR_ERR_CUDA;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return CFR_OK;
}

}  // namespace

extern "C" cfr_status cfr_paged_decode_static_workspace(
    const void *q, int32_t q_fmt, const cfr_kv_pool *kv, const int32_t *page_table,
    int32_t max_pages, const int32_t *seq_lens, int32_t batch, const uint8_t *page_fmt,
    int32_t uniform_fmt, int32_t num_q_heads, const int32_t *head_map, const float *alibi_slopes,
    float softmax_scale, float *out, float *lse, uint32_t *err_word, void *stream) {
  // Reject a problem whose scratch exceeds the array before touching the device.
  const size_t need = cfr_paged_decode_workspace_size(batch, num_q_heads,
                                                      kv ? kv->num_kv_heads : 0,
                                                      kv ? kv->head_dim : 0, max_pages,
                                                      kv ? kv->page_tokens : 0);
  if (need > static_cast<size_t>(CFR_STATIC_WORKSPACE_BYTES)) return CFR_ERR_WORKSPACE;
  void *ws = nullptr;
  const cfr_status st = static_workspace(&ws);
  if (st != CFR_OK) return st;
  return cfr_paged_decode(q, q_fmt, kv, page_table, max_pages, seq_lens, batch, page_fmt,
                          uniform_fmt, num_q_heads, head_map, alibi_slopes, softmax_scale, out,
                          lse, ws, static_cast<size_t>(CFR_STATIC_WORKSPACE_BYTES), err_word,
                          stream);
}
