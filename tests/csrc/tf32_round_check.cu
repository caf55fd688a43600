// Device check: the chunk kernel's integer tf32 rounding against the hardware
// conversion cvt.rna.tf32.f32, on every non-NaN input bit pattern given.
#include <cstdint>
#include <cuda_runtime.h>
#include "tc_primitives.cuh"

__global__ void tf32_round_kernel(const uint32_t* in, uint32_t* mismatches, uint32_t* first_bad, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float x = __uint_as_float(in[i]);
        uint32_t hw;
        asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hw) : "f"(x));
        const uint32_t sw = comba::tc::f32_to_tf32(x);
        if (x != x) continue;   // NaN inputs are outside the claim
        if (hw != sw) {
            atomicAdd(mismatches, 1u);
            atomicCAS(first_bad, 0xffffffffu, in[i]);
        }
    }
}

extern "C" int tf32_round_check(const uint32_t* in, uint32_t* mismatches, uint32_t* first_bad, int n) {
    tf32_round_kernel<<<264, 256>>>(in, mismatches, first_bad, n);
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : -1;
}
