// Tensor-core (tcgen05) chunk kernel: not yet wired in.
#pragma once

#include "common.cuh"

namespace comba {

inline bool tc_supported(int, int, int) { return false; }

inline int launch_chunk_tc(const void*, const void*, const void*, const float*, const float*,
                           const float*, const float*, void*, float*, int, int, int,
                           cudaStream_t) {
    return COMBA_EUNSUPPORTED;
}

}  // namespace comba
