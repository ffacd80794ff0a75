// cfr_sched.cu -- the ragged-batch split scheduler kernel (one CTA); the
// schedule itself is schedule_block in cfr_sched.cuh.
#include "cfr_sched.cuh"

namespace cfr {

constexpr int kSchedThreads = 1024;

__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(const SchedArgs a) {
  griddep_launch_dependents();
  schedule_block(a);
}

void launch_schedule(const int32_t *seq_lens, int batch, int P, int max_pages, int target,
                     int sink, int window, int nq, int unit, int32_t *split_off, int32_t *splits,
                     int max_splits, int32_t *num_splits, uint32_t *item_ctr, uint32_t *err,
                     cudaStream_t stream) {
  const SchedArgs a{seq_lens, batch, P, max_pages, target, sink, window, nq, unit,
                    split_off, splits, max_splits, num_splits, item_ctr, err};
  schedule_kernel<<<1, kSchedThreads, 0, stream>>>(a);
}

}  // namespace cfr
