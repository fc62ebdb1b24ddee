// Tensor-core (tcgen05 / TMEM / TMA) refinement kernel for sm_100a.
#pragma once

#include "internal.h"

namespace muse {

// True when the tcgen05 refinement handles this configuration (bfloat16 inputs).
bool tc_supported(int dtype, int D, int Dv);

// vt: the transposed sorted values (run_sort_side_t).
cudaError_t run_refine_tc(const MuseTables &mt, int D, int Dv, int N, int P, SortedSide qs,
                          const int32_t *q_perm, SortedSide ks, const int32_t *k_offsets,
                          const void *vt, StageBufs b, void *O, float *part_o, float *part_lse,
                          int *status, cudaStream_t st);

}  // namespace muse
