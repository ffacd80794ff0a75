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
// current) and caches it together with the id of the CUDA context it belongs
// to; later calls in the same context reuse the cached pointer.  A call in a
// new context on that device (after cudaDeviceReset, or a primary context torn
// down and created again) looks the address up again, since the old pointer
// belonged to the destroyed context.  The first call in a context should
// therefore happen before any stream capture.
//
// Every call shares the one array.  Nothing in it needs to start at zero: each
// call's schedule launch rewrites everything the later launches read.  Calls
// whose GPU work overlaps (on different streams) race on the array and must be
// serialised by the caller.
#include <cuda.h>

#include <mutex>

#include "cfr_common.cuh"

namespace {

constexpr int kMaxStaticDevices = 64;

static __device__ __align__(256) unsigned char g_static_workspace[CFR_STATIC_WORKSPACE_BYTES];

std::mutex g_static_mutex;
void *g_static_ptr[kMaxStaticDevices] = {nullptr};
unsigned long long g_static_ctx[kMaxStaticDevices] = {0};

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current CUDA context (driver entry points
// fetched at run time, so the library does not link libcuda); false when it
// cannot be read.
bool current_context_id(unsigned long long *id) {
  static std::once_flag once;
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_static_workspace on the current device, looked up once
// per device and context.
cfr_status static_workspace(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxStaticDevices)
    return CFR_ERR_CUDA;
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!have_ctx || !g_static_ptr[dev] || g_static_ctx[dev] != ctx) {
    // the lookup also makes the device's primary context current on this thread
    // when no context was current yet
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return CFR_ERR_CUDA;
    if (!current_context_id(&ctx)) return CFR_ERR_CUDA;
    g_static_ptr[dev] = p;
    g_static_ctx[dev] = ctx;
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
