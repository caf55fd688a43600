// C ABI of the Comba chunk-wise forward, its backward and the decode step (declared
// in comba.h).
//
// The host side validates every argument before anything is enqueued, picks
// the kernel for the shape, launches on the caller's stream and returns a
// status.  It owns no device memory.
#include "comba.h"

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "chunk_simt.cuh"
#include "chunk_tc.cuh"
#include "chunk_segments.cuh"
#include "chunk_bwd.cuh"
#include "chunk_bwd_chain.cuh"
#include "recurrent_step.cuh"

namespace {

using comba::SimtSmem;

constexpr int kMaxDevices = 64;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Byte ranges [a, a + na) and [b, b + nb) intersect.
bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

struct ChunkArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *d, *S0;
    void* out;
    float* S_final;
    int B, T, H, dk, dv, chunk;
    size_t elt;  // bytes per q/k/v/out element
};

int validate_chunk(const ChunkArgs& a) {
    if (a.B < 0 || a.T < 0 || a.H < 0) return COMBA_EINVAL;
    if (a.dk < 16 || a.dk > 128 || a.dk % 16) return COMBA_EINVAL;
    if (a.dv < 16 || a.dv > 128 || a.dv % 16) return COMBA_EINVAL;
    if (a.chunk != 16 && a.chunk != 32 && a.chunk != 64) return COMBA_EINVAL;
    if (a.B == 0 || a.H == 0) return COMBA_OK;
    if (!a.d) return COMBA_EINVAL;
    if (a.T > 0 && (!a.q || !a.k || !a.v || !a.log_alpha || !a.beta || !a.out)) return COMBA_EINVAL;
    const size_t bth = (size_t)a.B * a.T * a.H;
    if (bth > (size_t)1 << 40) return COMBA_EINVAL;
    const size_t nqk = bth * a.dk * a.elt, nv = bth * a.dv * a.elt;
    const size_t ng = bth * sizeof(float), nd = (size_t)a.H * sizeof(float);
    const size_t ns = (size_t)a.B * a.H * a.dv * a.dk * sizeof(float);
    if (!aligned(a.q, 16) || !aligned(a.k, 16) || !aligned(a.v, 16) || !aligned(a.out, 16) ||
        !aligned(a.S0, 16) || !aligned(a.S_final, 16) || !aligned(a.log_alpha, 4) ||
        !aligned(a.beta, 4) || !aligned(a.d, 4))
        return COMBA_EINVAL;
    const void* ins[] = {a.q, a.k, a.v, a.log_alpha, a.beta, a.d, a.S0};
    const size_t nin[] = {nqk, nqk, nv, ng, ng, nd, ns};
    for (int i = 0; i < 7; ++i) {
        if (overlap(a.out, nv, ins[i], nin[i])) return COMBA_EINVAL;
        // S_final may alias S0 exactly (in-place carry), nothing else.
        if (i == 6 && a.S_final == a.S0) continue;
        if (overlap(a.S_final, ns, ins[i], nin[i])) return COMBA_EINVAL;
    }
    if (overlap(a.S_final, ns, a.out, nv)) return COMBA_EINVAL;
    return COMBA_OK;
}

int current_device(int* dev) {
    if (cudaGetDevice(dev) != cudaSuccess) return COMBA_ECUDA;
    if (*dev < 0 || *dev >= kMaxDevices) return COMBA_ECUDA;
    return COMBA_OK;
}

// T == 0: the final state is the initial one.
int empty_sequence(const ChunkArgs& a, cudaStream_t stream) {
    if (!a.S_final) return COMBA_OK;
    const size_t ns = (size_t)a.B * a.H * a.dv * a.dk * sizeof(float);
    cudaError_t e = a.S0 ? (a.S0 == a.S_final ? cudaSuccess
                                              : cudaMemcpyAsync(a.S_final, a.S0, ns,
                                                                cudaMemcpyDeviceToDevice, stream))
                         : cudaMemsetAsync(a.S_final, 0, ns, stream);
    return e == cudaSuccess ? COMBA_OK : COMBA_ECUDA;
}

// Packed sequences for launch_simt: cu_seqlens (device, nseq + 1 entries) over the
// token axis of a single batch; Hqk q / k heads.
struct Packing {
    const int* cu_seqlens = nullptr;
    int nseq = 0;
    int Hqk = 0;
    const float* A_log = nullptr;     // gated inputs (see comba_chunk_fwd_gated)
    const float* dt_bias = nullptr;
    float norm_eps = 0.f;
};

template <typename Tin>
int launch_simt(const ChunkArgs& a, cudaStream_t stream, Packing pk = Packing()) {
    static bool attr_set[kMaxDevices] = {};
    int dev;
    if (int st = current_device(&dev)) return st;
    std::unique_lock<std::mutex> lock(comba::init_mutex());
    const int dvt = (a.dv % 32 == 0) ? 32 : 16;
    const SimtSmem m = comba::simt_smem_layout(a.dk, dvt, a.chunk);
    const size_t smem = m.total * sizeof(float);
    auto kern = comba::chunk_fwd_simt_kernel<Tin>;
    if (!attr_set[dev]) {
        const SimtSmem mx = comba::simt_smem_layout(128, 32, 64);
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(mx.total * sizeof(float))) != cudaSuccess)
            return COMBA_ECUDA;
        attr_set[dev] = true;
    }
    lock.unlock();
    dim3 grid((a.dv + dvt - 1) / dvt, a.H, pk.cu_seqlens ? pk.nseq : a.B);
    kern<<<grid, comba::kSimtThreads, smem, stream>>>(
        static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
        a.log_alpha, a.beta, a.d, a.S0, static_cast<Tin*>(a.out), a.S_final, a.T, a.H, a.dk,
        a.dv, a.chunk, dvt, pk.cu_seqlens, pk.Hqk > 0 ? pk.Hqk : a.H, pk.A_log, pk.dt_bias, pk.norm_eps);
    return cudaGetLastError() == cudaSuccess ? COMBA_OK : COMBA_ECUDA;
}

}  // namespace

extern "C" int comba_chunk_fwd(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta, const float* d,
                               const float* S0, void* out, float* S_final, int B, int T, int H,
                               int dk, int dv, int chunk, comba_stream_t stream) {
    const ChunkArgs a{q, k, v, log_alpha, beta, d, S0, out, S_final, B, T, H, dk, dv, chunk, 2};
    if (int st = validate_chunk(a)) return st;
    if (B == 0 || H == 0) return COMBA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) return empty_sequence(a, s);
    if (comba::tc_supported(dk, dv, chunk)) return comba::launch_chunk_tc(a.q, a.k, a.v, a.log_alpha, a.beta, a.d, a.S0, a.out, a.S_final, B, T, H, s);
    return launch_simt<__nv_bfloat16>(a, s);
}

extern "C" int comba_chunk_fwd_stall_test(const void* q, const void* k, const void* v,
                                       const float* log_alpha, const float* beta, const float* d,
                                       const float* S0, void* out, float* S_final, int B, int T, int H,
                                       int dk, int dv, int chunk, unsigned long long timeout_ns,
                                       int stall, comba_stream_t stream) {
    const ChunkArgs a{q, k, v, log_alpha, beta, d, S0, out, S_final, B, T, H, dk, dv, chunk, 2};
    if (int st = validate_chunk(a)) return st;
    if (!comba::tc_supported(dk, dv, chunk)) return COMBA_EUNSUPPORTED;
    if (B == 0 || H == 0) return COMBA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) return empty_sequence(a, s);
    return comba::launch_chunk_tc(q, k, v, log_alpha, beta, d, S0, out, S_final, B, T, H, s, -1, timeout_ns,
                                  nullptr, 0, 0, nullptr, nullptr, 0.f, stall != 0) == 0
               ? COMBA_OK : COMBA_ECUDA;
}

extern "C" int comba_chunk_fwd_varlen(const void* q, const void* k, const void* v,
                                      const float* log_alpha, const float* beta, const float* d,
                                      const float* S0, void* out, float* S_final,
                                      const int* cu_seqlens, int N, int total_T, int H, int Hqk,
                                      int dk, int dv, int chunk, comba_stream_t stream) {
    if (N < 0 || total_T < 0 || H < 0) return COMBA_EINVAL;
    if (dk < 16 || dk > 128 || dk % 16 || dv < 16 || dv > 128 || dv % 16) return COMBA_EINVAL;
    if (chunk != 16 && chunk != 32 && chunk != 64) return COMBA_EINVAL;
    if (N == 0 || H == 0) return COMBA_OK;
    if (Hqk < 1 || H % Hqk != 0 || !d || !cu_seqlens) return COMBA_EINVAL;
    if (total_T > 0 && (!q || !k || !v || !log_alpha || !beta || !out)) return COMBA_EINVAL;
    const size_t th = (size_t)total_T * H;
    if (th > (size_t)1 << 40) return COMBA_EINVAL;
    const size_t nqk = (size_t)total_T * Hqk * dk * 2, nv = th * dv * 2, ng = th * sizeof(float);
    const size_t nd = (size_t)H * sizeof(float), ns = (size_t)N * H * dv * dk * sizeof(float);
    const size_t ncu = ((size_t)N + 1) * sizeof(int);
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(S0, 16) ||
        !aligned(S_final, 16) || !aligned(log_alpha, 4) || !aligned(beta, 4) || !aligned(d, 4) ||
        !aligned(cu_seqlens, 4))
        return COMBA_EINVAL;
    const void* ins[] = {q, k, v, log_alpha, beta, d, S0, cu_seqlens};
    const size_t nin[] = {nqk, nqk, nv, ng, ng, nd, ns, ncu};
    for (int i = 0; i < 8; ++i) {
        if (overlap(out, nv, ins[i], nin[i])) return COMBA_EINVAL;
        if (i == 6 && S_final == S0) continue;   // in-place state carry
        if (overlap(S_final, ns, ins[i], nin[i])) return COMBA_EINVAL;
    }
    if (overlap(S_final, ns, out, nv)) return COMBA_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // one batch of total_T tokens; the kernels read each chain's bounds from cu_seqlens
    const ChunkArgs a{q, k, v, log_alpha, beta, d, S0, out, S_final, N, total_T, H, dk, dv, chunk, 2};
    if (total_T == 0) return empty_sequence(a, s);   // every sequence is empty
    if (comba::tc_supported(dk, dv, chunk))
        return comba::launch_chunk_tc(q, k, v, log_alpha, beta, d, S0, out, S_final, 1, total_T, H, s, -1,
                                      comba::kWaitTimeoutNs, cu_seqlens, N, Hqk);
    ChunkArgs a1 = a;
    a1.B = 1;
    return launch_simt<__nv_bfloat16>(a1, s, Packing{cu_seqlens, N, Hqk});
}

extern "C" int comba_chunk_fwd_gated(const void* q_raw, const void* k_raw, const void* v,
                                     const float* a_raw, const float* b_raw, const float* A_log,
                                     const float* dt_bias, const float* d, const float* S0, void* out,
                                     float* S_final, int B, int T, int H, int dk, int dv, int chunk,
                                     float norm_eps, comba_stream_t stream) {
    const ChunkArgs a{q_raw, k_raw, v, a_raw, b_raw, d, S0, out, S_final, B, T, H, dk, dv, chunk, 2};
    if (int st = validate_chunk(a)) return st;
    if (!(norm_eps >= 0.f)) return COMBA_EINVAL;
    if (B == 0 || H == 0) return COMBA_OK;
    if (!A_log || !aligned(A_log, 4) || !aligned(dt_bias, 4)) return COMBA_EINVAL;
    const size_t nv = (size_t)B * T * H * dv * 2, ns = (size_t)B * H * dv * dk * sizeof(float);
    if (overlap(out, nv, A_log, (size_t)H * 4) || overlap(out, nv, dt_bias, (size_t)H * 4) ||
        overlap(S_final, ns, A_log, (size_t)H * 4) || overlap(S_final, ns, dt_bias, (size_t)H * 4))
        return COMBA_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) return empty_sequence(a, s);
    if (comba::tc_supported(dk, dv, chunk))
        return comba::launch_chunk_tc(q_raw, k_raw, v, a_raw, b_raw, d, S0, out, S_final, B, T, H, s, -1,
                                      comba::kWaitTimeoutNs, nullptr, 0, 0, A_log, dt_bias, norm_eps);
    Packing pk;
    pk.A_log = A_log;
    pk.dt_bias = dt_bias;
    pk.norm_eps = norm_eps;
    return launch_simt<__nv_bfloat16>(a, s, pk);
}

extern "C" size_t comba_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk) {
    if (B <= 0 || H <= 0 || T <= 0 || !comba::tc_supported(dk, dv, chunk)) return 0;
    const int P = comba::seg::segment_count(B, T, H, comba::seg::sm_count());
    return comba::seg::workspace_floats(B, H, P) * sizeof(float);
}

extern "C" int comba_chunk_fwd_ws(const void* q, const void* k, const void* v,
                                  const float* log_alpha, const float* beta, const float* d,
                                  const float* S0, void* out, float* S_final, int B, int T, int H,
                                  int dk, int dv, int chunk, void* workspace, size_t workspace_bytes,
                                  comba_stream_t stream) {
    const ChunkArgs a{q, k, v, log_alpha, beta, d, S0, out, S_final, B, T, H, dk, dv, chunk, 2};
    if (int st = validate_chunk(a)) return st;
    if (B == 0 || H == 0) return COMBA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) return empty_sequence(a, s);
    if (!comba::tc_supported(dk, dv, chunk)) return launch_simt<__nv_bfloat16>(a, s);
    const int P = comba::seg::segment_count(B, T, H, comba::seg::sm_count());
    const size_t need = comba::seg::workspace_floats(B, H, P) * sizeof(float);
    if (P > 1 && workspace && workspace_bytes >= need) {
        if (!aligned(workspace, 16)) return COMBA_EINVAL;
        const size_t bth = (size_t)B * T * H;
        const void* bufs[] = {q, k, v, log_alpha, beta, d, S0, out, S_final};
        const size_t nb[] = {bth * dk * 2, bth * dk * 2, bth * dv * 2, bth * 4, bth * 4, (size_t)H * 4,
                             (size_t)B * H * dv * dk * 4, bth * dv * 2, (size_t)B * H * dv * dk * 4};
        for (int i = 0; i < 9; ++i)
            if (overlap(workspace, need, bufs[i], nb[i])) return COMBA_EINVAL;
        return comba::seg::launch_segmented(q, k, v, log_alpha, beta, d, S0, out, S_final, B, T, H, P,
                                            static_cast<float*>(workspace), s) == 0 ? COMBA_OK : COMBA_ECUDA;
    }
    return comba::launch_chunk_tc(a.q, a.k, a.v, a.log_alpha, a.beta, a.d, a.S0, a.out, a.S_final, B, T, H, s) == 0
               ? COMBA_OK : COMBA_ECUDA;
}

// Scratch of comba_chunk_fwd_noalloc: the segmented form's workspace for up to
// kNoallocChains segment-chains (B * P * H), in the module's static device memory.
constexpr size_t kNoallocChains = 128;
constexpr size_t kNoallocFloats = 6 * kNoallocChains * comba::seg::kStateFloats;
static __device__ __align__(256) float g_noalloc_ws[kNoallocFloats];

extern "C" int comba_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                       const float* log_alpha, const float* beta, const float* d,
                                       const float* S0, void* out, float* S_final, int B, int T,
                                       int H, int dk, int dv, int chunk, comba_stream_t stream) {
    void* ws = nullptr;
    if (cudaGetSymbolAddress(&ws, g_noalloc_ws) != cudaSuccess) return COMBA_ECUDA;
    return comba_chunk_fwd_ws(q, k, v, log_alpha, beta, d, S0, out, S_final, B, T, H, dk, dv, chunk, ws,
                              sizeof(g_noalloc_ws), stream);
}

extern "C" int comba_chunk_fwd_transition(const void* q, const void* k, const void* v,
                                          const float* log_alpha, const float* beta, const float* d,
                                          float* RM, int B, int T, int H, int dk, int dv, int chunk,
                                          comba_stream_t stream) {
    // the input rules of comba_chunk_fwd; RM (two states per chain) must not overlap an input
    if (B < 0 || T < 0 || H < 0) return COMBA_EINVAL;
    if (B == 0 || H == 0) return COMBA_OK;
    if (!comba::tc_supported(dk, dv, chunk)) return COMBA_EUNSUPPORTED;
    if (!RM || !aligned(RM, 16) || !d || !aligned(d, 4)) return COMBA_EINVAL;
    const size_t bph = (size_t)B * H, bth = (size_t)B * T * H;
    if (bth > (size_t)1 << 40 || 2 * bph > (size_t)1 << 31) return COMBA_EINVAL;
    const size_t nrm = 2 * bph * comba::seg::kStateFloats * sizeof(float);
    if (T > 0) {
        if (!q || !k || !v || !log_alpha || !beta) return COMBA_EINVAL;
        if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(log_alpha, 4) || !aligned(beta, 4))
            return COMBA_EINVAL;
    }
    const void* ins[] = {q, k, v, log_alpha, beta, d};
    const size_t nin[] = {bth * dk * 2, bth * dk * 2, bth * dv * 2, bth * 4, bth * 4, (size_t)H * 4};
    for (int i = 0; i < 6; ++i)
        if (overlap(RM, nrm, ins[i], nin[i])) return COMBA_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // RM starts as the stacked start states [0 | I]; the launch carries each in place to
    // its end state (CTAs of the second half see V = 0)
    comba::seg::seg_init_kernel<<<(unsigned)(2 * bph), 256, 0, s>>>(RM, (long)bph);
    if (cudaGetLastError() != cudaSuccess) return COMBA_ECUDA;
    if (T == 0) return COMBA_OK;
    return comba::launch_chunk_tc(q, k, v, log_alpha, beta, d, RM, nullptr, RM, B, T, H, s, 2 * B) == 0
               ? COMBA_OK : COMBA_ECUDA;
}

extern "C" int comba_chunk_fwd_f32(const float* q, const float* k, const float* v,
                                   const float* log_alpha, const float* beta, const float* d,
                                   const float* S0, float* out, float* S_final, int B, int T,
                                   int H, int dk, int dv, int chunk, comba_stream_t stream) {
    const ChunkArgs a{q, k, v, log_alpha, beta, d, S0, out, S_final, B, T, H, dk, dv, chunk, 4};
    if (int st = validate_chunk(a)) return st;
    if (B == 0 || H == 0) return COMBA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) return empty_sequence(a, s);
    return launch_simt<float>(a, s);
}

// ---------------------------------------------------------------- host buffers
namespace {

size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }

// Device regions of comba_chunk_fwd_host's workspace, in order.
struct HostLayout {
    size_t q, k, v, la, be, d, s0, out, sf, total;
};

HostLayout host_layout(int B, int T, int H, int dk, int dv) {
    const size_t bth = (size_t)B * T * H, ns = (size_t)B * H * dv * dk * sizeof(float);
    HostLayout L{};
    size_t o = 0;
    auto take = [&](size_t n) { const size_t at = o; o += round256(n); return at; };
    L.q = take(bth * dk * 2);
    L.k = take(bth * dk * 2);
    L.v = take(bth * dv * 2);
    L.la = take(bth * sizeof(float));
    L.be = take(bth * sizeof(float));
    L.d = take((size_t)H * sizeof(float));
    L.s0 = take(ns);
    L.out = take(bth * dv * 2);
    L.sf = take(ns);
    L.total = o;
    return L;
}

// Copy streams of one device, created on first use and kept for the process.
bool copy_streams(int dev, cudaStream_t* h2d, cudaStream_t* d2h) {
    static cudaStream_t s[kMaxDevices][2] = {};
    std::lock_guard<std::mutex> lock(comba::init_mutex());
    if (!s[dev][0]) {
        cudaStream_t a = nullptr, b = nullptr;
        if (cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking) != cudaSuccess) return false;
        if (cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking) != cudaSuccess) {
            cudaStreamDestroy(a);
            return false;
        }
        s[dev][0] = a;
        s[dev][1] = b;
    }
    *h2d = s[dev][0];
    *d2h = s[dev][1];
    return true;
}

}  // namespace

extern "C" size_t comba_chunk_fwd_host_workspace_size(int B, int T, int H, int dk, int dv) {
    if (B <= 0 || T <= 0 || H <= 0 || dk <= 0 || dv <= 0) return 0;
    return host_layout(B, T, H, dk, dv).total;
}

extern "C" int comba_chunk_fwd_host(const void* q, const void* k, const void* v,
                                    const float* log_alpha, const float* beta, const float* d,
                                    const float* S0, void* out, float* S_final, int B, int T, int H,
                                    int dk, int dv, int chunk, void* workspace, size_t workspace_bytes,
                                    int slices, comba_stream_t stream) {
    const ChunkArgs h{q, k, v, log_alpha, beta, d, S0, out, S_final, B, T, H, dk, dv, chunk, 2};
    if (int st = validate_chunk(h)) return st;
    if (B == 0 || H == 0) return COMBA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t ns = (size_t)B * H * dv * dk * sizeof(float);
    if (T == 0) {   // the final state is the initial one (or zero)
        if (!S_final) return COMBA_OK;
        if (S0) return cudaMemcpyAsync(S_final, S0, ns, cudaMemcpyHostToHost, s) == cudaSuccess ? COMBA_OK : COMBA_ECUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return COMBA_ECUDA;
        memset(S_final, 0, ns);
        return COMBA_OK;
    }
    const HostLayout L = host_layout(B, T, H, dk, dv);
    if (!workspace || workspace_bytes < L.total || !aligned(workspace, 256)) return COMBA_EINVAL;
    if (slices < 1) return COMBA_EINVAL;
    int dev;
    if (int st = current_device(&dev)) return st;
    cudaStream_t sh, sd;
    if (!copy_streams(dev, &sh, &sd)) return COMBA_ECUDA;
    char* w = static_cast<char*>(workspace);
    const int P = slices < B ? slices : B;
    // events: start, per slice in / out, done
    cudaEvent_t ev[2 * 64 + 2];
    const int nev = 2 * (P < 64 ? P : 64) + 2;
    for (int i = 0; i < nev; ++i)
        if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) {
            for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
            return COMBA_ECUDA;
        }
    int st = COMBA_OK;
    auto ok = [&](cudaError_t e) { if (e != cudaSuccess && st == COMBA_OK) st = COMBA_ECUDA; };
    // the copies start behind everything already on the caller's stream (an earlier
    // call may still be reading this workspace)
    ok(cudaEventRecord(ev[0], s));
    ok(cudaStreamWaitEvent(sh, ev[0], 0));
    ok(cudaMemcpyAsync(w + L.d, d, (size_t)H * sizeof(float), cudaMemcpyHostToDevice, sh));
    const int Pn = nev / 2 - 1;   // slices actually used (at most 64)
    const size_t th = (size_t)T * H;
    for (int p = 0; p < Pn && st == COMBA_OK; ++p) {
        const int b0 = (int)((long)B * p / Pn), b1 = (int)((long)B * (p + 1) / Pn), nb = b1 - b0;
        if (nb == 0) continue;
        auto h2d = [&](size_t at, const void* src, size_t per_b) {
            ok(cudaMemcpyAsync(w + at + b0 * per_b, static_cast<const char*>(src) + b0 * per_b, nb * per_b,
                               cudaMemcpyHostToDevice, sh));
        };
        h2d(L.q, q, th * dk * 2);
        h2d(L.k, k, th * dk * 2);
        h2d(L.v, v, th * dv * 2);
        h2d(L.la, log_alpha, th * sizeof(float));
        h2d(L.be, beta, th * sizeof(float));
        const size_t sb = (size_t)H * dv * dk * sizeof(float);
        if (S0) h2d(L.s0, S0, sb);
        ok(cudaEventRecord(ev[1 + 2 * p], sh));
        ok(cudaStreamWaitEvent(s, ev[1 + 2 * p], 0));
        const ChunkArgs a{w + L.q + b0 * th * dk * 2, w + L.k + b0 * th * dk * 2, w + L.v + b0 * th * dv * 2,
                          reinterpret_cast<const float*>(w + L.la + b0 * th * 4),
                          reinterpret_cast<const float*>(w + L.be + b0 * th * 4),
                          reinterpret_cast<const float*>(w + L.d),
                          S0 ? reinterpret_cast<const float*>(w + L.s0 + b0 * sb) : nullptr,
                          w + L.out + b0 * th * dv * 2,
                          S_final ? reinterpret_cast<float*>(w + L.sf + b0 * sb) : nullptr,
                          nb, T, H, dk, dv, chunk, 2};
        int lst;
        if (comba::tc_supported(dk, dv, chunk))
            lst = comba::launch_chunk_tc(a.q, a.k, a.v, a.log_alpha, a.beta, a.d, a.S0, a.out, a.S_final, nb, T, H, s);
        else
            lst = launch_simt<__nv_bfloat16>(a, s);
        if (lst != 0 && st == COMBA_OK) st = lst;
        ok(cudaEventRecord(ev[2 + 2 * p], s));
        ok(cudaStreamWaitEvent(sd, ev[2 + 2 * p], 0));
        ok(cudaMemcpyAsync(static_cast<char*>(out) + b0 * th * dv * 2, w + L.out + b0 * th * dv * 2,
                           nb * th * dv * 2, cudaMemcpyDeviceToHost, sd));
        if (S_final)
            ok(cudaMemcpyAsync(reinterpret_cast<char*>(S_final) + b0 * sb, w + L.sf + b0 * sb, nb * sb,
                               cudaMemcpyDeviceToHost, sd));
    }
    // the caller's stream completes once the results are in host memory
    ok(cudaEventRecord(ev[nev - 1], sd));
    ok(cudaStreamWaitEvent(s, ev[nev - 1], 0));
    for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
    return st;
}

extern "C" int comba_recurrent_step_grouped(const void* q, const void* k, const void* v,
                                            const float* log_alpha, const float* beta, const float* d,
                                            float* S, void* out, int B, int H, int Hqk, int dk, int dv,
                                            comba_stream_t stream) {
    if (B < 0 || H < 0) return COMBA_EINVAL;
    if (H > 0 && (Hqk < 1 || H % Hqk != 0)) return COMBA_EINVAL;
    if (dk != 32 && dk != 64 && dk != 128) return COMBA_EINVAL;
    if (dv < 16 || dv > 128 || dv % 16) return COMBA_EINVAL;
    if (B == 0 || H == 0) return COMBA_OK;
    if (!q || !k || !v || !log_alpha || !beta || !d || !S || !out) return COMBA_EINVAL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(S, 16) || !aligned(log_alpha, 4) || !aligned(beta, 4) || !aligned(d, 4))
        return COMBA_EINVAL;
    const size_t bh = (size_t)B * H;
    if (bh > (size_t)1 << 31) return COMBA_EINVAL;
    const size_t nqk = (size_t)B * Hqk * dk * 2, nv = bh * dv * 2, ng = bh * 4, ns = bh * dv * dk * 4;
    const void* ins[] = {q, k, v, log_alpha, beta, d};
    const size_t nin[] = {nqk, nqk, nv, ng, ng, (size_t)H * 4};
    for (int i = 0; i < 6; ++i)
        if (overlap(out, nv, ins[i], nin[i]) || overlap(S, ns, ins[i], nin[i])) return COMBA_EINVAL;
    if (overlap(out, nv, S, ns)) return COMBA_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    const auto* vb = static_cast<const __nv_bfloat16*>(v);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    const unsigned grid = (unsigned)bh;
    switch (dk) {
        case 32:
            comba::recurrent_step_kernel<32><<<grid, comba::kStepThreads, 0, s>>>(qb, kb, vb, log_alpha, beta, d, S, ob, H, dv, Hqk);
            break;
        case 64:
            comba::recurrent_step_kernel<64><<<grid, comba::kStepThreads, 0, s>>>(qb, kb, vb, log_alpha, beta, d, S, ob, H, dv, Hqk);
            break;
        default:
            comba::recurrent_step_kernel<128><<<grid, comba::kStepThreads, 0, s>>>(qb, kb, vb, log_alpha, beta, d, S, ob, H, dv, Hqk);
            break;
    }
    return cudaGetLastError() == cudaSuccess ? COMBA_OK : COMBA_ECUDA;
}

extern "C" int comba_recurrent_step(const void* q, const void* k, const void* v,
                                    const float* log_alpha, const float* beta, const float* d,
                                    float* S, void* out, int B, int H, int dk, int dv,
                                    comba_stream_t stream) {
    return comba_recurrent_step_grouped(q, k, v, log_alpha, beta, d, S, out, B, H, H, dk, dv, stream);
}

namespace {

struct BwdArgs {
    const void *q, *k, *v, *dout;
    const float *log_alpha, *beta, *d, *S0, *dS_final;
    float *dq, *dk, *dv, *dlog_alpha, *dbeta, *dd, *dS0;
    int B, T, H, DK, DV;
    unsigned long long timeout_ns = comba::bwd::chain::kWaitNs;   // the state passes' per-wait limit
    int stall = 0;                                                 // their failure-path test
};

template <typename Tin, int DK, int DV>
int launch_bwd(const BwdArgs& a, float* wsp, cudaStream_t s) {
    namespace bw = comba::bwd;
    const long chains = (long)a.B * a.H;
    const int nch = (a.T + bw::kL - 1) / bw::kL;
    const bw::Workspace ws = bw::carve(wsp, chains, nch, DK, DV);
    const auto* q = static_cast<const Tin*>(a.q);
    const auto* k = static_cast<const Tin*>(a.k);
    const auto* v = static_cast<const Tin*>(a.v);
    const auto* o = static_cast<const Tin*>(a.dout);
    const size_t sp = bw::PrepSmem<Tin, DK, DV>::total * sizeof(float);
    const size_t ss = bw::StatesSmem<DK, DV>::total * sizeof(float);
    const size_t sd = bw::DStatesSmem<DK, DV>::total * sizeof(float);
    const size_t sg = bw::grads_smem_bytes<Tin, DK, DV>();
    if (cudaFuncSetAttribute(bw::bwd_prep_kernel<Tin, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sp) != cudaSuccess ||
        cudaFuncSetAttribute(bw::bwd_states_kernel<Tin, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)ss) != cudaSuccess ||
        cudaFuncSetAttribute(bw::bwd_dstates_kernel<Tin, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sd) != cudaSuccess ||
        cudaFuncSetAttribute(bw::bwd_grads_kernel<Tin, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sg) != cudaSuccess)
        return COMBA_ECUDA;
    if constexpr (bw::grads_tc<Tin, DK, DV>()) {
        // prep, then both state passes in one launch (2 x chains CTAs), then the grads
        if (cudaFuncSetAttribute(bw::chain::bwd_chain_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)bw::chain::kSmemBytes) != cudaSuccess)
            return COMBA_ECUDA;
        if (chains > 0 && nch > 0) {
            const dim3 grid((unsigned)nch, (unsigned)chains);
            bw::bwd_prep_kernel<Tin, DK, DV><<<grid, bw::kThreads, sp, s>>>(q, k, v, a.log_alpha, a.beta, a.d, o,
                                                                             ws, a.T, a.H, nch);
        }
        if (chains > 0)
            bw::chain::bwd_chain_tc_kernel<<<(unsigned)(2 * chains), bw::chain::kThreads, bw::chain::kSmemBytes, s>>>(
                ws, a.S0, a.dS_final, a.dS0, (int)chains, nch, a.timeout_ns, a.stall);
    } else if (chains > 0 && nch > 0) {
        const dim3 grid((unsigned)nch, (unsigned)chains);
        bw::bwd_prep_kernel<Tin, DK, DV><<<grid, bw::kThreads, sp, s>>>(q, k, v, a.log_alpha, a.beta, a.d, o, ws,
                                                                         a.T, a.H, nch);
        bw::bwd_states_kernel<Tin, DK, DV><<<(unsigned)(chains * (DV / bw::kRows)), bw::kThreads, ss, s>>>(k, a.log_alpha, a.beta, a.S0,
                                                                                       ws, a.T, a.H, nch);
    }
    if (!bw::grads_tc<Tin, DK, DV>() && chains > 0)
        bw::bwd_dstates_kernel<Tin, DK, DV><<<(unsigned)(chains * (DV / bw::kRows)), bw::kThreads, sd, s>>>(
            k, a.log_alpha, a.beta, a.dS_final, a.dS0, ws, a.T, a.H, nch);
    if (chains > 0 && nch > 0) {
        const dim3 grid((unsigned)nch, (unsigned)chains);
        bw::bwd_grads_kernel<Tin, DK, DV><<<grid, bw::kThreads, sg, s>>>(q, k, v, a.log_alpha, a.beta, a.d, o, a.dq,
                                                                          a.dk, a.dv, a.dlog_alpha, a.dbeta, ws,
                                                                          a.T, a.H, nch);
    }
    if (a.dd && a.H > 0)
        bw::bwd_dd_sum_kernel<<<(unsigned)a.H, bw::kThreads, 0, s>>>(ws.ddp, a.dd, a.B, a.H, nch);
    return cudaGetLastError() == cudaSuccess ? COMBA_OK : COMBA_ECUDA;
}

template <typename Tin, int DK>
int launch_bwd_dv(const BwdArgs& a, float* ws, cudaStream_t s) {
    switch (a.DV) {
        case 32: return launch_bwd<Tin, DK, 32>(a, ws, s);
        case 64: return launch_bwd<Tin, DK, 64>(a, ws, s);
        default: return launch_bwd<Tin, DK, 128>(a, ws, s);
    }
}

template <typename Tin>
int launch_bwd_dk(const BwdArgs& a, float* ws, cudaStream_t s) {
    switch (a.DK) {
        case 32: return launch_bwd_dv<Tin, 32>(a, ws, s);
        case 64: return launch_bwd_dv<Tin, 64>(a, ws, s);
        default: return launch_bwd_dv<Tin, 128>(a, ws, s);
    }
}

bool bwd_dim(int x) { return x == 32 || x == 64 || x == 128; }

}  // namespace

extern "C" size_t comba_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv) {
    if (B < 0 || T < 0 || H < 0 || !bwd_dim(dk) || !bwd_dim(dv)) return 0;
    const int nch = (T + comba::bwd::kL - 1) / comba::bwd::kL;
    return comba::bwd::workspace_floats((long)B * H, nch, dk, dv) * sizeof(float);
}

static int chunk_bwd_impl(const void* q, const void* k, const void* v, const float* log_alpha,
                          const float* beta, const float* d, const float* S0, const void* dout,
                          const float* dS_final, float* dq, float* dk, float* dv, float* dlog_alpha,
                          float* dbeta, float* dd, float* dS0, int B, int T, int H, int dk_, int dv_,
                          int dtype, void* workspace, size_t workspace_bytes, comba_stream_t stream,
                          unsigned long long timeout_ns, int stall) {
    if (B < 0 || T < 0 || H < 0 || !bwd_dim(dk_) || !bwd_dim(dv_)) return COMBA_EINVAL;
    if (dtype != COMBA_BF16 && dtype != COMBA_F32) return COMBA_EINVAL;
    const size_t elt = (dtype == COMBA_BF16) ? 2 : 4;
    const long chains = (long)B * H;
    if (chains > 65535) return COMBA_EUNSUPPORTED;
    const size_t bth = (size_t)B * T * H;
    if (bth > (size_t)1 << 40) return COMBA_EINVAL;
    if (chains == 0 && !(dd && H > 0)) return COMBA_OK;
    const size_t need = comba_chunk_bwd_workspace_size(B, T, H, dk_, dv_);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return COMBA_EINVAL;
    if (bth > 0 && (!q || !k || !v || !dout || !log_alpha || !beta || !dq || !dk || !dv || !dlog_alpha || !dbeta))
        return COMBA_EINVAL;
    if (chains > 0 && !d) return COMBA_EINVAL;
    const void* ins[] = {q, k, v, dout, log_alpha, beta, d, S0, dS_final};
    const size_t nqk = bth * dk_ * elt, nv = bth * dv_ * elt, ng = bth * 4, nh = (size_t)H * 4;
    const size_t ns = (size_t)chains * dv_ * dk_ * 4;
    const size_t nin[] = {nqk, nqk, nv, nv, ng, ng, nh, ns, ns};
    const void* outs[] = {dq, dk, dv, dlog_alpha, dbeta, dd, dS0, workspace};
    const size_t nout[] = {bth * dk_ * 4, bth * dk_ * 4, bth * dv_ * 4, ng, ng, nh, ns, need};
    // rows of q, k, v, dout and the state matrices are read with 16-byte vector loads
    for (int i = 0; i < 9; ++i)
        if (!aligned(ins[i], (i < 4 || i >= 7) ? 16 : 4)) return COMBA_EINVAL;
    for (int i = 0; i < 8; ++i) {
        if (!aligned(outs[i], 4)) return COMBA_EINVAL;
        for (int j = 0; j < 9; ++j)
            if (overlap(outs[i], nout[i], ins[j], nin[j])) return COMBA_EINVAL;
        for (int j = i + 1; j < 8; ++j)
            if (overlap(outs[i], nout[i], outs[j], nout[j])) return COMBA_EINVAL;
    }
    const BwdArgs a{q, k, v, dout, log_alpha, beta, d, S0, dS_final, dq, dk, dv, dlog_alpha, dbeta, dd, dS0,
                    B, T, H, dk_, dv_, timeout_ns, stall};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    float* ws = static_cast<float*>(workspace);
    return dtype == COMBA_BF16 ? launch_bwd_dk<__nv_bfloat16>(a, ws, s) : launch_bwd_dk<float>(a, ws, s);
}

extern "C" int comba_chunk_bwd(const void* q, const void* k, const void* v, const float* log_alpha,
                               const float* beta, const float* d, const float* S0, const void* dout,
                               const float* dS_final, float* dq, float* dk, float* dv, float* dlog_alpha,
                               float* dbeta, float* dd, float* dS0, int B, int T, int H, int dk_, int dv_,
                               int dtype, void* workspace, size_t workspace_bytes, comba_stream_t stream) {
    return chunk_bwd_impl(q, k, v, log_alpha, beta, d, S0, dout, dS_final, dq, dk, dv, dlog_alpha, dbeta, dd, dS0,
                          B, T, H, dk_, dv_, dtype, workspace, workspace_bytes, stream,
                          comba::bwd::chain::kWaitNs, 0);
}

extern "C" int comba_chunk_bwd_stall_test(const void* q, const void* k, const void* v, const float* log_alpha,
                                          const float* beta, const float* d, const float* S0, const void* dout,
                                          const float* dS_final, float* dq, float* dk, float* dv,
                                          float* dlog_alpha, float* dbeta, float* dd, float* dS0, int B, int T,
                                          int H, int dk_, int dv_, int dtype, void* workspace,
                                          size_t workspace_bytes, unsigned long long timeout_ns, int stall,
                                          comba_stream_t stream) {
    if (dtype != COMBA_BF16 || dk_ != 128 || dv_ != 128) return COMBA_EUNSUPPORTED;
    return chunk_bwd_impl(q, k, v, log_alpha, beta, d, S0, dout, dS_final, dq, dk, dv, dlog_alpha, dbeta, dd, dS0,
                          B, T, H, dk_, dv_, dtype, workspace, workspace_bytes, stream, timeout_ns, stall);
}

extern "C" int comba_state_compose(const float* RM, const float* S0, float* S_start, int B, int H, int P,
                                   comba_stream_t stream) {
    if (B < 0 || H < 0 || P < 1) return COMBA_EINVAL;
    if (B == 0 || H == 0) return COMBA_OK;
    if (!RM || !S_start) return COMBA_EINVAL;
    if (!aligned(RM, 16) || !aligned(S0, 16) || !aligned(S_start, 16)) return COMBA_EINVAL;
    const size_t st = comba::seg::kStateFloats * sizeof(float);
    const size_t bph = (size_t)B * P * H;
    if (bph > (size_t)1 << 31 || (size_t)B * H * comba::seg::kComposeBlocks > (size_t)0x7fffffff) return COMBA_EINVAL;
    if (overlap(S_start, bph * st, RM, 2 * bph * st) || overlap(S_start, bph * st, S0, (size_t)B * H * st))
        return COMBA_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaFuncSetAttribute(comba::seg::seg_compose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)comba::seg::kComposeSmem) != cudaSuccess)
        return COMBA_ECUDA;
    comba::seg::seg_compose_kernel<<<(unsigned)(B * H * comba::seg::kComposeBlocks), comba::seg::kComposeThreads,
                                        comba::seg::kComposeSmem, s>>>(
        RM, S0, S_start, B, H, P);
    return cudaGetLastError() == cudaSuccess ? COMBA_OK : COMBA_ECUDA;
}

namespace {

// Reads and clears the current device's status word with copies ordered on `s`.
int read_clear_status(cudaStream_t s) {
    int h = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbolAsync(&h, comba::g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemcpyToSymbolAsync(comba::g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return COMBA_ECUDA;
    return h;
}

}  // namespace

extern "C" int comba_get_last_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return COMBA_ECUDA;
    return read_clear_status(nullptr);
}

extern "C" int comba_get_last_error_stream(comba_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return COMBA_ECUDA;
    return read_clear_status(s);
}

extern "C" const char* comba_status_string(int status) {
    switch (status) {
        case COMBA_OK: return "ok";
        case COMBA_EINVAL: return "invalid argument (pointer, size, alignment or aliasing)";
        case COMBA_EUNSUPPORTED: return "unsupported shape";
        case COMBA_ECUDA: return "CUDA runtime error";
        case COMBA_ETIMEOUT: return "device-side bounded wait gave up";
        case COMBA_EDEVICE: return "device-side inconsistency";
        default: return "unknown status";
    }
}

extern "C" int comba_version(void) { return 100; }
