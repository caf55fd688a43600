// Sequence-segmented chunk forward for chains too few to fill the GPU (long T, small
// B*H): the state pass of each (b, h) chain is split into P contiguous segments that
// run as independent chains, joined by the segments' affine state transitions.
//
// The state recursion is affine in the state.  Over one segment, from a start state
// S, it ends in  S M + R  with  R = the end state from S = 0 (with the segment's V)
// and  M = the end state from S = I with V = 0 (dk x dk; dv = dk here).  So:
//   pass 1   one launch of the chunk kernel over the B*P segments twice stacked:
//            [segments from S = 0 | segments from S = I with V = 0], no outputs
//            -> R and M of every segment
//   compose  S_start(0) = S0,  S_start(p + 1) = S_start(p) M_p + R_p  (per chain)
//   pass 2   the chunk kernel over the B*P segments from S_start(p), with outputs;
//            the last segment's end state is the chain's S_final.
// A [B, T, H, d] tensor cut into P contiguous pieces of T/P tokens is the
// [B*P, T/P, H, d] tensor, so each pass is one plain launch of the chunk kernel.
// This is the write-up's "recurrent across blocks, parallel inside" form applied
// one level up (section "硬件高效的分块并行计算"), with the per-segment transition
// made explicit.
#pragma once

#include "chunk_tc.cuh"

namespace comba {
namespace seg {

constexpr int kD = 128;                        // dk = dv for the tensor-core path
constexpr size_t kStateFloats = (size_t)kD * kD;

// Number of segments per chain (1 = no split): the one minimising the estimated
// time in chunk-steps of one CTA, counting pass 1 (twice as many CTAs) and pass 2
// in waves of `sms` CTAs, and about two chunk-steps per compose step.  Segments are
// whole chunks and at least 8 chunks long.
inline int segment_count(int B, int T, int H, int sms) {
    if (T % 64 != 0 || sms <= 0) return 1;
    const long nch = T / 64, bh = (long)B * H;
    auto waves = [&](long ctas) { return (ctas + sms - 1) / sms; };
    const long plain = waves(bh) * nch;
    int best = 1;
    long best_cost = plain;
    for (int P = 2; P <= 64; P *= 2) {
        if (nch % P != 0 || nch / P < 8) break;
        const long cost = (waves(2 * bh * P) + waves(bh * P)) * (nch / P) + 2 * P;   // + compose
        if (cost < best_cost) { best_cost = cost; best = P; }
    }
    return (best > 1 && 4 * best_cost < 3 * plain) ? best : 1;
}

// Workspace: [2 B P H] start states of pass 1, [2 B P H] end states (R | M),
// [B P H] start states of pass 2, [B P H] end states of pass 2; fp32 dv x dk each.
inline size_t workspace_floats(int B, int H, int P) {
    return (P <= 1) ? 0 : (size_t)6 * B * P * H * kStateFloats;
}

// Start states of pass 1: zeros for the first n_half states, the identity for the rest.
__global__ void seg_init_kernel(float* S, long n_half) {
    const long total = 2 * n_half * (long)kStateFloats;
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
        const long blk = i / (long)kStateFloats, e = i % (long)kStateFloats;
        S[i] = (blk >= n_half && (e / kD) == (e % kD)) ? 1.f : 0.f;
    }
}

constexpr int kComposeThreads = 256;
constexpr int kComposeRows = 16;                              // state rows per CTA
constexpr int kComposeBlocks = kD / kComposeRows;             // CTAs per chain
constexpr size_t kComposeSmem = (size_t)(kComposeRows + kD) * kD * sizeof(float);   // S rows, M

// S_start(0) = S0 (or 0), S_start(p+1) = S_start(p) M_p + R_p, written for p = 0 .. P-1
// to Sst[(b P + p) H + h].  R_p, M_p sit in RM at stacked batch b P + p and B P + b P +
// p.  A row of S_start(p+1) depends only on the same row of S_start(p), so each chain's
// 128 rows are split over kComposeBlocks CTAs that never communicate: CTA
// (b H + h) kComposeBlocks + rb owns rows 16 rb .. 16 rb + 15, and thread t the 8
// columns 8 (t % 16) .. + 7 of row t / 16.  Every output element is the same fp32 FMA
// chain (R first, then k = 0 .. 127) whichever CTA computes it.
__global__ void __launch_bounds__(kComposeThreads)
seg_compose_kernel(const float* __restrict__ RM, const float* __restrict__ S0, float* __restrict__ Sst,
                   int B, int H, int P) {
    extern __shared__ __align__(16) float smem[];
    float* Sc = smem;                              // the CTA's rows of the current start state
    float* Mt = smem + kComposeRows * kD;          // this segment's transition, dk x dk
    const int chain = blockIdx.x / kComposeBlocks, rb = blockIdx.x % kComposeBlocks;
    const int b = chain / H, h = chain % H, tid = threadIdx.x;
    const int i = tid / 16, j0 = (tid % 16) * 8, row = rb * kComposeRows + i;
    const long BP = (long)B * P;
    const float* s0 = S0 ? S0 + ((size_t)b * H + h) * kStateFloats : nullptr;
    float sv[8];
    {
        const float4 a4 = s0 ? *reinterpret_cast<const float4*>(s0 + (size_t)row * kD + j0) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 b4 = s0 ? *reinterpret_cast<const float4*>(s0 + (size_t)row * kD + j0 + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        sv[0] = a4.x; sv[1] = a4.y; sv[2] = a4.z; sv[3] = a4.w;
        sv[4] = b4.x; sv[5] = b4.y; sv[6] = b4.z; sv[7] = b4.w;
    }
    for (int p = 0; p < P; ++p) {
        float* dst = Sst + ((size_t)(b * P + p) * H + h) * kStateFloats + (size_t)row * kD + j0;
        *reinterpret_cast<float4*>(dst) = make_float4(sv[0], sv[1], sv[2], sv[3]);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(sv[4], sv[5], sv[6], sv[7]);
        if (p + 1 == P) break;
        const float* Rp = RM + ((size_t)(b * P + p) * H + h) * kStateFloats;
        const float* Mp = RM + ((size_t)(BP + b * P + p) * H + h) * kStateFloats;
        __syncthreads();   // the previous product is done with Sc and Mt
#pragma unroll
        for (int c = 0; c < 8; ++c) Sc[i * kD + j0 + c] = sv[c];
        {   // M_p into shared memory: every 16-byte load issued before the stores
            constexpr int PER = (int)(kStateFloats / 4) / kComposeThreads;
            float4 m4[PER];
#pragma unroll
            for (int it = 0; it < PER; ++it)
                m4[it] = *reinterpret_cast<const float4*>(Mp + 4 * (size_t)(tid + it * kComposeThreads));
#pragma unroll
            for (int it = 0; it < PER; ++it)
                *reinterpret_cast<float4*>(Mt + 4 * (tid + it * kComposeThreads)) = m4[it];
        }
        float acc[8];
        {
            const float4 a4 = *reinterpret_cast<const float4*>(Rp + (size_t)row * kD + j0);
            const float4 b4 = *reinterpret_cast<const float4*>(Rp + (size_t)row * kD + j0 + 4);
            acc[0] = a4.x; acc[1] = a4.y; acc[2] = a4.z; acc[3] = a4.w;
            acc[4] = b4.x; acc[5] = b4.y; acc[6] = b4.z; acc[7] = b4.w;
        }
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < kD; ++k) {
            const float s = Sc[i * kD + k];
            const float4 ma = *reinterpret_cast<const float4*>(Mt + k * kD + j0);
            const float4 mb = *reinterpret_cast<const float4*>(Mt + k * kD + j0 + 4);
            acc[0] = fmaf(s, ma.x, acc[0]); acc[1] = fmaf(s, ma.y, acc[1]);
            acc[2] = fmaf(s, ma.z, acc[2]); acc[3] = fmaf(s, ma.w, acc[3]);
            acc[4] = fmaf(s, mb.x, acc[4]); acc[5] = fmaf(s, mb.y, acc[5]);
            acc[6] = fmaf(s, mb.z, acc[6]); acc[7] = fmaf(s, mb.w, acc[7]);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) sv[c] = acc[c];
    }
}

inline int sm_count() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lock(init_mutex());
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cached[dev] = n;
    }
    return cached[dev];
}

// The three steps above on `stream`; `ws` holds workspace_floats(B, H, P) floats.
// Returns 0 or a negative status as launch_chunk_tc.
inline int launch_segmented(const void* q, const void* k, const void* v, const float* log_alpha,
                            const float* beta, const float* d, const float* S0, void* out,
                            float* S_final, int B, int T, int H, int P, float* ws,
                            cudaStream_t stream) {
    const int Bs = B * P, Ts = T / P;
    const size_t n = (size_t)Bs * H * kStateFloats;
    float* S_in1 = ws;            // 2 n
    float* RM = ws + 2 * n;       // 2 n
    float* Sst = ws + 4 * n;      // n
    float* Sfin = ws + 5 * n;     // n
    seg_init_kernel<<<2 * Bs * H, 256, 0, stream>>>(S_in1, (long)Bs * H);
    if (cudaGetLastError() != cudaSuccess) return -3;
    if (int st = launch_chunk_tc(q, k, v, log_alpha, beta, d, S_in1, nullptr, RM, Bs, Ts, H, stream, 2 * Bs))
        return st;
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -3;
    std::unique_lock<std::mutex> lock(init_mutex());
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(seg_compose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kComposeSmem) != cudaSuccess)
            return -3;
        attr_set[dev] = true;
    }
    lock.unlock();
    seg_compose_kernel<<<B * H * kComposeBlocks, kComposeThreads, kComposeSmem, stream>>>(RM, S0, Sst, B, H, P);
    if (cudaGetLastError() != cudaSuccess) return -3;
    if (int st = launch_chunk_tc(q, k, v, log_alpha, beta, d, Sst, out, Sfin, Bs, Ts, H, stream))
        return st;
    if (S_final) {   // the last segment's end state of each batch (H consecutive states)
        for (int b = 0; b < B; ++b)
            if (cudaMemcpyAsync(S_final + (size_t)b * H * kStateFloats,
                                Sfin + (size_t)(b * P + P - 1) * H * kStateFloats,
                                (size_t)H * kStateFloats * sizeof(float), cudaMemcpyDeviceToDevice,
                                stream) != cudaSuccess)
                return -3;
    }
    return 0;
}

}  // namespace seg
}  // namespace comba
