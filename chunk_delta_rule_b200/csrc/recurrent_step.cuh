// Single-token Comba step for decoding (the recurrence at T = 1, state in place).
//
// For each (b, h) and each value row i of S (write-up, section
// "背景知识和相关工作": constant-size state, O(1) work per token):
//   p_i   = S_i . k                         (read-out at the key, old state)
//   S_i  <- alpha S_i - beta p_i k + beta v_i k
//   o_i   = S_i . (q - d_h k)               (post-update output correction)
// The step moves each state row through HBM exactly once in each direction,
// so it is bandwidth-bound: rows are streamed with 16-byte loads and stores
// (one warp per row group, each lane owns dk/32 consecutive columns), several
// rows in flight per warp, and the loads/stores are marked streaming because
// no state row is reused within the step.
#pragma once

#include "common.cuh"

namespace comba {

constexpr int kStepThreads = 256;
constexpr int kStepRowsInFlight = 4;

template <int PER> struct VecF;
template <> struct VecF<4> { using T = float4; };
template <> struct VecF<2> { using T = float2; };
template <> struct VecF<1> { using T = float; };

template <int PER>
__device__ __forceinline__ void vload(const float* p, float (&x)[PER]) {
    if constexpr (PER == 4) {
        const float4 t = __ldcs(reinterpret_cast<const float4*>(p));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else if constexpr (PER == 2) {
        const float2 t = __ldcs(reinterpret_cast<const float2*>(p));
        x[0] = t.x; x[1] = t.y;
    } else {
        x[0] = __ldcs(p);
    }
}

template <int PER>
__device__ __forceinline__ void vstore(float* p, const float (&x)[PER]) {
    if constexpr (PER == 4) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
    } else if constexpr (PER == 2) {
        __stcs(reinterpret_cast<float2*>(p), make_float2(x[0], x[1]));
    } else {
        __stcs(p, x[0]);
    }
}

// One CTA per (b, h); warp w owns rows w, w + 8, w + 16, ...
template <int DK>
__global__ void __launch_bounds__(kStepThreads)
recurrent_step_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      const __nv_bfloat16* __restrict__ v, const float* __restrict__ log_alpha,
                      const float* __restrict__ beta, const float* __restrict__ dvec,
                      float* __restrict__ S, __nv_bfloat16* __restrict__ out, int H, int dv, int Hqk) {
    constexpr int PER = DK / 32;
    __shared__ float o_s[128];
    const int bh = blockIdx.x;
    const int h = bh % H;
    // q / k of value head h: head h / (H / Hqk) of the batch row's Hqk heads
    const size_t qk = ((size_t)(bh / H) * Hqk + h / (H / Hqk)) * DK;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int nwarps = kStepThreads / 32;

    const float a = expf(log_alpha[bh]);
    const float bt = beta[bh];
    const float dh = dvec[h];
    float kr[PER], qt[PER];
#pragma unroll
    for (int p = 0; p < PER; ++p) {
        kr[p] = __bfloat162float(k[qk + lane * PER + p]);
        qt[p] = __bfloat162float(q[qk + lane * PER + p]) - dh * kr[p];
    }
    float* Sb = S + (size_t)bh * dv * DK + lane * PER;
    const __nv_bfloat16* vb = v + (size_t)bh * dv;

    for (int base = warp; base < dv; base += nwarps * kStepRowsInFlight) {
        float x[kStepRowsInFlight][PER];
        float vi[kStepRowsInFlight];
#pragma unroll
        for (int u = 0; u < kStepRowsInFlight; ++u) {
            const int i = base + u * nwarps;
            vi[u] = 0.f;
#pragma unroll
            for (int p = 0; p < PER; ++p) x[u][p] = 0.f;
            if (i < dv) {
                vload<PER>(Sb + (size_t)i * DK, x[u]);
                vi[u] = __bfloat162float(vb[i]);
            }
        }
        float pk[kStepRowsInFlight];
#pragma unroll
        for (int u = 0; u < kStepRowsInFlight; ++u) {
            float acc = 0.f;
#pragma unroll
            for (int p = 0; p < PER; ++p) acc = fmaf(x[u][p], kr[p], acc);
            pk[u] = acc;
        }
#pragma unroll
        for (int u = 0; u < kStepRowsInFlight; ++u) pk[u] = warp_sum(pk[u]);
        float ov[kStepRowsInFlight];
#pragma unroll
        for (int u = 0; u < kStepRowsInFlight; ++u) {
            const int i = base + u * nwarps;
            float acc = 0.f;
#pragma unroll
            for (int p = 0; p < PER; ++p) {
                x[u][p] = a * x[u][p] - bt * pk[u] * kr[p] + bt * vi[u] * kr[p];
                acc = fmaf(x[u][p], qt[p], acc);
            }
            ov[u] = acc;
            if (i < dv) vstore<PER>(Sb + (size_t)i * DK, x[u]);
        }
#pragma unroll
        for (int u = 0; u < kStepRowsInFlight; ++u) ov[u] = warp_sum(ov[u]);
        if (lane == 0) {
#pragma unroll
            for (int u = 0; u < kStepRowsInFlight; ++u) {
                const int i = base + u * nwarps;
                if (i < dv) o_s[i] = ov[u];
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < dv; i += kStepThreads)
        out[(size_t)bh * dv + i] = __float2bfloat16_rn(o_s[i]);
}

}  // namespace comba
