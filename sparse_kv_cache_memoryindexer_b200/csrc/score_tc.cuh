// Tensor-core (tcgen05) index score for n_h = 64, d_I = 128: not built yet in this revision.
#pragma once
#include "common.cuh"

namespace lsa {

inline bool tc_score_available() { return false; }

inline lsa_status launch_score_tc(const void *, const float *, const void *, const float *, int, const int64_t *,
                                  const int *, int, int64_t, int, float, float *, uint32_t *, int, cudaStream_t)
{
    return LSA_ERR_UNSUPPORTED;
}

}  // namespace lsa
