// Test-only kernel: builds tcgen05 operands in the 128B-swizzled shared-memory
// layouts the chunk kernel uses, issues the product's MMA helpers, and returns
// D = A B^T (plus an optional initial D) so a test can compare with a host GEMM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tc_primitives.cuh"

using namespace comba::tc;

namespace {

// element (r, k) of a K-major tile: rows at 128 B, K in 64-element atoms `atom` bytes apart
__device__ uint32_t kmaj(int r, int k, uint32_t atom) {
    return (k >> 6) * atom + sw128(r, (k & 63) >> 3) + (k & 7) * 2;
}
// element (m, k) of an MN-major tile: one 128 B row per k, 64-element M atoms `lbo` apart
__device__ uint32_t mnmaj(int m, int k, uint32_t lbo) {
    return (m >> 6) * lbo + sw128(k, (m & 63) >> 3) + (m & 7) * 2;
}

__global__ void umma_check_kernel(int mode, const float* A, const float* B, const float* D0,
                                  float* D, int* status) {
    extern __shared__ uint8_t raw[];
    const uint32_t r0 = smem_u32(raw);
    uint8_t* sm = raw + (((r0 + 1023u) & ~1023u) - r0);
    const uint32_t sb = smem_u32(sm);
    uint8_t* sa = sm;            // A tile, 32 KB
    uint8_t* sbt = sm + 32768;   // B tile, 32 KB
    __shared__ uint64_t bar;
    __shared__ uint32_t tslot;
    const int tid = threadIdx.x, warp = tid >> 5;
    // mode: 0 gram (A K 128x128, B K 64x128), 1 W^T (A MN lbo 16384, K=64; B K 64x64),
    //       2 N^T (A MN lbo 8192), 3 S W^T (A K 128x128; B MN N=64, K=128),
    //       4 state update (A K 128x128 hi|lo; B MN N=128 lbo 16384, K rows 64 wrapped),
    //       5 output (A K 128x128; B K 64x64 re-read; accumulate onto D0)
    int M = 128, N = 64, K = 128;
    if (mode == 1 || mode == 2) K = 64;
    if (mode == 4) N = 128;
    if (mode == 8 || mode == 9) {
        // bf16 with A in TMEM (two bf16 per column); B bf16 in smem:
        // 8: K-major, N = 64, K = 128 in two atoms 16 KB apart
        // 9: MN-major, N = 64 (one atom), K = 128 rows
        K = 128;
        N = 64;
        for (int e = tid; e < N * K; e += blockDim.x) {
            const int n = e / K, k = e % K;
            const uint32_t off = (mode == 8) ? kmaj(n, k, 16384) : mnmaj(n, k, 8192);
            *reinterpret_cast<__nv_bfloat16*>(sbt + off) = __float2bfloat16_rn(B[e]);
        }
    } else if (mode == 6 || mode == 7) {
        // tf32 with A in TMEM (fp32, lane = row, column = k); B fp32 in smem:
        // 6: K-major, N = 64, K = 64 in two 32-element atoms 8 KB apart
        // 7: K-major, N = 128, K = 64 in two 32-element atoms 16 KB apart
        K = 64;
        N = (mode == 7) ? 128 : 64;
        for (int e = tid; e < N * K; e += blockDim.x) {
            const int n = e / K, k = e % K;
            uint32_t off;
            if (mode == 6) off = (k >> 5) * 8192 + sw128(n, (k & 31) >> 2) + (k & 3) * 4;
            else off = (k >> 5) * 16384 + sw128(n, (k & 31) >> 2) + (k & 3) * 4;
            *reinterpret_cast<float*>(sbt + off) = B[e];
        }
    } else {
    for (int e = tid; e < M * K; e += blockDim.x) {
        const int m = e / K, k = e % K;
        uint32_t off;
        if (mode == 1) off = mnmaj(m, k, 16384);
        else if (mode == 2) off = mnmaj(m, k, 8192);
        else off = kmaj(m, k, 16384);
        *reinterpret_cast<__nv_bfloat16*>(sa + off) = __float2bfloat16_rn(A[e]);
    }
    const int Kb = (mode == 4 || mode == 5) ? 64 : K;   // stored B extent along K
    for (int e = tid; e < N * Kb; e += blockDim.x) {
        const int n = e / Kb, k = e % Kb;
        uint32_t off;
        if (mode == 3) off = mnmaj(n, k, 8192);
        else if (mode == 4) off = mnmaj(n, k, 16384);
        else off = kmaj(n, k, 16384);
        *reinterpret_cast<__nv_bfloat16*>(sbt + off) = __float2bfloat16_rn(B[n * K + k]);
    }
    }
    if (tid == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
    if (warp == 0) tmem_alloc(&tslot, 256);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    if (mode == 8 || mode == 9) {   // A (bf16 pairs) into TMEM columns 128..191
        for (int part = 0; part < 2; ++part) {
            float v[32];
            for (int e = 0; e < 32; ++e) {
                const int k = part * 64 + 2 * e;
                const uint32_t w = pack_bf16(A[tid * K + k], A[tid * K + k + 1]);
                v[e] = __uint_as_float(w);
            }
            tmem_st32(trow + 128 + part * 32, v);
        }
        tmem_st_wait();
        tc_fence_before();
    }
    if (mode == 6 || mode == 7) {   // A (fp32) into TMEM columns 128..191
        for (int part = 0; part < 2; ++part) {
            float v[32];
            for (int e = 0; e < 32; ++e) v[e] = A[tid * K + part * 32 + e];
            tmem_st32(trow + 128 + part * 32, v);
        }
        tmem_st_wait();
        tc_fence_before();
    }
    if (mode == 5) {
        for (int part = 0; part < N / 32; ++part) {
            float v[32];
            for (int e = 0; e < 32; ++e) v[e] = D0[tid * N + part * 32 + e];
            tmem_st32(trow + part * 32, v);
        }
        tmem_st_wait();
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 0) {   // one converged warp issues (one elected lane)
        tc_fence_after();
        const uint32_t a = sb, b = sb + 32768;
        switch (mode) {
            case 0: mma_ak_bk(tmem, a, 16384, b, 16384, idesc_bf16(128, 64, false, false), 8, 0); break;
            case 1: mma_amn_bk(tmem, a, 16384, b, idesc_bf16(128, 64, true, false), 4, 0); break;
            case 2: mma_amn_bk(tmem, a, 8192, b, idesc_bf16(128, 64, true, false), 4, 0); break;
            case 3: mma_ak_bmn(tmem, a, 16384, b, 8192, idesc_bf16(128, 64, false, true), 8, 8, 0); break;
            case 4: mma_ak_bmn(tmem, a, 16384, b, 16384, idesc_bf16(128, 128, false, true), 8, 4, 0); break;
            case 5: mma_ak_bk(tmem, a, 16384, b, 0, idesc_bf16(128, 64, false, false), 8, 1); break;
            case 6: mma_tf32_ta_bk(tmem, tmem + 128, b, 8192, idesc_tf32(128, 64, false, false), 8, 0); break;
            case 8: mma_bf16_ta_bk(tmem, tmem + 128, b, 16384, idesc_bf16(128, 64, false, false), 8, 0); break;
            case 9: mma_bf16_ta_bmn(tmem, tmem + 128, b, 8192, idesc_bf16(128, 64, false, true), 8, 0); break;
            case 7: mma_tf32_ta_bk(tmem, tmem + 128, b, 16384, idesc_tf32(128, 128, false, false), 8, 0); break;
        }
        mma_commit(&bar);
    }
    const bool done = mbar_wait(&bar, 0, 2000000000ull);
    if (!done && tid == 0) *status = 1;
    tc_fence_after();
    if (done) {
        for (int part = 0; part < N / 32; ++part) {
            float v[32];
            tmem_ld32(trow + part * 32, v);
            tmem_ld_wait();
            for (int e = 0; e < 32; ++e) D[tid * N + part * 32 + e] = v[e];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace

extern "C" int umma_layout_check(int mode, const float* A, const float* B, const float* D0, float* D,
                                 int* status) {
    const int smem = 65536 + 1024;
    if (cudaFuncSetAttribute(umma_check_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return -3;
    umma_check_kernel<<<1, 128, smem>>>(mode, A, B, D0, D, status);
    if (cudaGetLastError() != cudaSuccess) return -3;
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : -3;
}
