// Shared device helpers for the Comba kernels (single translation unit: comba.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace comba {

// Host side: guards the library's lazily initialised per-device state (kernel
// attributes, cached device properties, copy streams), so that threads making their
// first calls at the same time initialise it once.
inline std::mutex& init_mutex() {
    static std::mutex m;
    return m;
}

// Per-device status word.  Kernels latch the first device-side error here
// (atomicCAS from 0); comba_get_last_error() reads and clears it.
__device__ int g_status = 0;

__device__ __forceinline__ void latch_status(int code) { atomicCAS(&g_status, 0, code); }


__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace comba
