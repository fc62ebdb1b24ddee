// Tensor-core refinement (placeholder until the tcgen05 kernel lands).
#include "tc.h"

namespace muse {

bool tc_supported(int, int, int) { return false; }

cudaError_t run_refine_tc(const MuseTables &, int, int, int, int, SortedSide, const int32_t *,
                          SortedSide, const void *, StageBufs, void *, float *, float *, int *,
                          cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace muse
