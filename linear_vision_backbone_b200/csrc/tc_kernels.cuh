// tc_kernels.cuh -- tcgen05/TMEM path (placeholder until the tensor-core
// kernels land; every shape reports unsupported so the SIMT path runs).
#pragma once
#include "common.cuh"

namespace gtr {

inline bool tc_shape_supported(int, int, int, int) { return false; }
inline int tc_blocks_per_sm(int, int) { return 1; }

inline int launch_tc(int, int, const void*, const void*, const void*, const float*, const void*,
                     const float*, void*, float*, float*, int, int, int, int, int, int, int, int,
                     int, int, int, cudaStream_t) {
  return -2;
}

}  // namespace gtr
