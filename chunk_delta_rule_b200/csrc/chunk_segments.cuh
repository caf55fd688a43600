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
constexpr size_t kComposeSmem = 2 * kStateFloats * sizeof(float);   // S and M tiles

// One CTA per (b, h) chain: S_start(0) = S0 (or 0), S_start(p+1) = S_start(p) M_p + R_p,
// written for p = 0 .. P-1 to Sst[(b P + p) H + h].  R_p, M_p sit in RM at stacked
// batch b P + p and B P + b P + p.  Each thread owns an 8 x 8 tile of the product.
__global__ void __launch_bounds__(kComposeThreads)
seg_compose_kernel(const float* __restrict__ RM, const float* __restrict__ S0, float* __restrict__ Sst,
                   int B, int H, int P) {
    extern __shared__ float smem[];
    float* Sc = smem;                  // current start state, row-major dv x dk
    float* Mt = smem + kStateFloats;   // this segment's transition, dk x dk
    const int b = blockIdx.x / H, h = blockIdx.x % H, tid = threadIdx.x;
    const long BP = (long)B * P;
    const float* s0 = S0 ? S0 + ((size_t)b * H + h) * kStateFloats : nullptr;
    for (int i = tid; i < (int)kStateFloats; i += kComposeThreads) Sc[i] = s0 ? s0[i] : 0.f;
    const int i0 = (tid / 16) * 8, j0 = (tid % 16) * 8;
    for (int p = 0; p < P; ++p) {
        __syncthreads();
        float* dst = Sst + ((size_t)(b * P + p) * H + h) * kStateFloats;
        for (int i = tid; i < (int)kStateFloats; i += kComposeThreads) dst[i] = Sc[i];
        if (p + 1 == P) break;
        const float* Rp = RM + ((size_t)(b * P + p) * H + h) * kStateFloats;
        const float* Mp = RM + ((size_t)(BP + b * P + p) * H + h) * kStateFloats;
        for (int i = tid; i < (int)kStateFloats; i += kComposeThreads) Mt[i] = Mp[i];
        __syncthreads();
        float acc[8][8];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[a][c] = Rp[(size_t)(i0 + a) * kD + j0 + c];
        for (int k = 0; k < kD; ++k) {
            float sv[8], mv[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) sv[a] = Sc[(i0 + a) * kD + k];
#pragma unroll
            for (int c = 0; c < 8; ++c) mv[c] = Mt[k * kD + j0 + c];
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(sv[a], mv[c], acc[a][c]);
        }
        __syncthreads();
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int c = 0; c < 8; ++c) Sc[(i0 + a) * kD + j0 + c] = acc[a][c];
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
    seg_compose_kernel<<<B * H, kComposeThreads, kComposeSmem, stream>>>(RM, S0, Sst, B, H, P);
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
