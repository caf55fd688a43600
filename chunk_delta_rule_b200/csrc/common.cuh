// Shared device helpers for the Comba kernels (single translation unit: comba.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace comba {

// Per-device status word.  Kernels latch the first device-side error here
// (atomicCAS from 0); comba_get_last_error() reads and clears it.
__device__ int g_status = 0;

__device__ __forceinline__ void latch_status(int code) { atomicCAS(&g_status, 0, code); }

// Optional phase tracing (compile with -DCOMBA_TRACE_PHASES): thread 0 and thread
// COMBA_TRACE_TID2 (default 128) of CTA 0 accumulate clock64() deltas between
// consecutive COMBA_PHASE marks in registers (each thread its own slots) and add
// them to a device array at COMBA_PHASE_END; threads 0 (state group), 128 (MMA-issue
// warp) and COMBA_TRACE_TID2 also record the absolute clock64() of every mark in
// loop iterations COMBA_TRACE_ITER .. + 3.  Off by default; the marks then compile
// to nothing.
#define COMBA_TRACE_SLOTS 32
#define COMBA_TRACE_TS_ITERS 4
#ifdef COMBA_TRACE_PHASES
#ifndef COMBA_TRACE_TID2
#define COMBA_TRACE_TID2 128
#endif
#ifndef COMBA_TRACE_ITER
#define COMBA_TRACE_ITER 10
#endif
#ifndef COMBA_TRACE_CTA
#define COMBA_TRACE_CTA 0
#endif
__device__ unsigned long long g_phase_cycles[COMBA_TRACE_SLOTS];
// [thread 0 | thread 128 | thread TID2][iteration ITER + k][mark]
__device__ long long g_phase_ts[3 * COMBA_TRACE_TS_ITERS * COMBA_TRACE_SLOTS];
#define COMBA_PHASE_BEGIN()                                   \
    long long comba_phase_t = clock64();                      \
    int comba_iter = 0;                                       \
    unsigned long long comba_phase_acc[COMBA_TRACE_SLOTS] = {}
#ifndef COMBA_TRACE_MASK
#define COMBA_TRACE_MASK 0xffffffffu
#endif
#define COMBA_PHASE(i)                                                        \
    do {                                                                      \
        if (!((COMBA_TRACE_MASK >> (i)) & 1u)) break;                         \
        const long long comba_phase_now = clock64();                          \
        comba_phase_acc[(i)] += (unsigned long long)(comba_phase_now - comba_phase_t); \
        comba_phase_t = comba_phase_now;                                      \
        const int comba_k = comba_iter - COMBA_TRACE_ITER;                    \
        const int comba_w = threadIdx.x == 0 ? 0 : threadIdx.x == 128 ? 1     \
                          : threadIdx.x == COMBA_TRACE_TID2 ? 2 : -1;         \
        if (comba_k >= 0 && comba_k < COMBA_TRACE_TS_ITERS && comba_w >= 0 && \
            blockIdx.x == COMBA_TRACE_CTA)                                    \
            g_phase_ts[(comba_w * COMBA_TRACE_TS_ITERS + comba_k) * COMBA_TRACE_SLOTS + (i)] = \
                comba_phase_now;                                              \
    } while (0)
#define COMBA_ITER_NEXT() (++comba_iter)
// per-CTA start / end (global timer, ns) of up to 1024 CTAs, and SM clock cycles
__device__ unsigned long long g_cta_ns[2 * 1024];
__device__ long long g_cta_clk[3 * 1024];
#define COMBA_CTA_MARK(k)                                                          \
    do {                                                                           \
        if (threadIdx.x == 0 && blockIdx.x < 1024) {                               \
            unsigned long long comba_t;                                            \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(comba_t));            \
            g_cta_ns[2 * blockIdx.x + (k)] = comba_t;                              \
            g_cta_clk[2 * blockIdx.x + (k)] = clock64();                           \
            if ((k) == 0) {                                                        \
                unsigned comba_sm;                                                 \
                asm volatile("mov.u32 %0, %%smid;" : "=r"(comba_sm));              \
                g_cta_clk[2048 + blockIdx.x] = comba_sm;                           \
            }                                                                      \
        }                                                                          \
    } while (0)
#define COMBA_COUNT(i) (++comba_phase_acc[(i)])
#define COMBA_PHASE_END()                                                     \
    do {                                                                      \
        if (blockIdx.x == COMBA_TRACE_CTA && (threadIdx.x == 0 || threadIdx.x == COMBA_TRACE_TID2)) \
            for (int comba_i = 0; comba_i < COMBA_TRACE_SLOTS; ++comba_i)     \
                g_phase_cycles[comba_i] += comba_phase_acc[comba_i];          \
    } while (0)
#else
#define COMBA_PHASE_BEGIN() do {} while (0)
#define COMBA_PHASE(i) do {} while (0)
#define COMBA_ITER_NEXT() do {} while (0)
#define COMBA_CTA_MARK(k) do {} while (0)
#define COMBA_COUNT(i) do {} while (0)
#define COMBA_PHASE_END() do {} while (0)
#endif

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
