// Tensor-core (tcgen05) chunked forward: not built yet; every call falls to the SIMT family.
#pragma once

#include "common.cuh"

namespace gdn {

inline bool tc_chunk_supported(int, int, int, bool) { return false; }

inline gdn_status tc_chunk_launch(const void*, const void*, const void*, const float*,
                                  const float*, const float*, void*, float*, int, int, int, int,
                                  float, cudaStream_t) {
  return GDN_ERR_UNSUPPORTED;
}

inline gdn_status tc_chunk_launch_f32out(const void*, const void*, const void*, const float*,
                                         const float*, const float*, float*, float*, int, int,
                                         int, int, float, cudaStream_t) {
  return GDN_ERR_UNSUPPORTED;
}

}  // namespace gdn
