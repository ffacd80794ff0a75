// cfr_decode_tc.cu -- tensor-core (tcgen05) paged decode attention.
#include "cfr_common.cuh"

namespace cfr {

bool tc_supported(const DecodeParams &p, bool page_fmt_given) {
  (void)p;
  (void)page_fmt_given;
  return false;
}

cudaError_t launch_decode_tc(const DecodeParams &p, int grid, cudaStream_t stream) {
  (void)p;
  (void)grid;
  (void)stream;
  return cudaErrorNotSupported;
}

}  // namespace cfr
