// conv1d_tc.cuh -- op B with the pointwise contraction on tcgen05 tensor cores.
#pragma once

#include "common.cuh"

namespace fcv {

inline bool conv1d_tc_supported(int, int, int, int) { return false; }

inline int launch_dwsep_conv1d_tc(const float*, const float*, const float*, const float*, int, int, int,
                                  int, int, int, int, int, float*, cudaStream_t)
{
    return FCV_ERR_UNSUPPORTED;
}

}  // namespace fcv
