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

// Retrieval remainder (pair form over each query's causal prefix minus its selected
// (cluster, block) pairs) into the partials part_o [P][N][Dv], part_lse [P][N] (token
// order); b.c0 / b.c1 / b.lse carry the remainder coefficients per sorted query row.
// kblk [P][N]: block of every sorted key; kgrp [P][N/8]: min | max << 16 of every 8.
cudaError_t run_refine_tc_ret(const MuseTables &mt, int D, int Dv, int N, int P, SortedSide qs,
                              const int32_t *q_perm, SortedSide ks, const int32_t *k_offsets,
                              const void *vt, StageBufs b, float *part_o, float *part_lse,
                              const unsigned short *kblk, const int *kgrp, const int32_t *pend,
                              const int32_t *sel, int S, int k1, int k2, int *status,
                              cudaStream_t st);

}  // namespace muse
