// cfr_diag.cu -- diagnostic of the device-side failure handling.
//
// Every on-device wait of the decode kernels is a bounded mbarrier wait
// (mbar_wait in cfr_common.cuh): past its cycle limit it gives up, ORs
// CFR_DEVERR_TIMEOUT into the error word and lets the kernel return, so a
// stuck pipeline ends as a status the host reads instead of a hung GPU.  This
// file runs that same wait, with a short limit, on an mbarrier that one thread
// initialises and (optionally) arrives on, so that a test can make the wait run
// out on purpose.  No copy or tensor-core operation is in flight in this
// kernel, so giving up leaves nothing outstanding.
#include "cfr_common.cuh"

namespace cfr {
namespace {

// 1 thread: waits on phase 0 of an mbarrier of arrival count 1, after one
// arrival when `arrive` is set.  *result = 1 when the phase completed, 0 when
// the wait gave up.
__global__ void wait_probe_kernel(long long limit, int arrive, uint32_t *err, uint32_t *result) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (arrive) mbar_arrive(&bar);
  bool timed_out = false;
  const bool ok = mbar_wait(&bar, 0u, err, &timed_out, limit);
  if (result) *result = ok ? 1u : 0u;
}

}  // namespace
}  // namespace cfr

extern "C" cfr_status cfr_wait_probe(int64_t limit_cycles, int32_t arrive, uint32_t *err_word,
                                     uint32_t *result, void *stream) {
  if (limit_cycles < 1 || limit_cycles > cfr::kWaitLimitCycles) return CFR_ERR_INVALID_ARG;
  cfr::wait_probe_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<long long>(limit_cycles), arrive ? 1 : 0, err_word, result);
  return cudaGetLastError() == cudaSuccess ? CFR_OK : CFR_ERR_CUDA;
}
