// Tensor-core chunk-wise Comba forward for bf16 inputs, dk = dv = 128, chunk 64.
//
// One CTA (8 warps) owns one (b, h) chain and walks its chunks in order.
// Thread t owns TMEM lane t % 128 and half of that lane's columns.  Per chunk
// (chunk-start state S, local tokens r, s, g_r = sum_{i<=r} log_alpha_i, g_0 = 0;
// the write-up's "block-recurrent, intra-block parallel" form with a single
// inverse for the intermediates W and U, section "硬件高效的分块并行计算"):
//
//   1. gates (prefetched one chunk ahead): g by warp-shuffle scan, e^{g_r},
//      e^{-g_r}, e^{g_L - g_r}, c_r = beta_r e^{g_{r-1}}
//   2. Gram MMA G = [K; Q] K^T (bf16 -> TMEM), issued during the previous chunk
//   3. K K^T staged in the P operand; A_rs = beta_r e^{g_{r-1}-g_s}(K K^T)_rs (s < r);
//      then, concurrently: P_rs = e^{g_r-g_s}(Q K^T - d K K^T)_rs (s <= r) in
//      place (fp32 operand), Qh = diag(e^g)(Q - d K) over Q and (D K)^T with
//      D = diag(e^{g_L - g}) (fp32, K-major) on half the warps; the 16 x 16
//      diagonal blocks of Tinv = (I + A)^{-1} by substitution on the others
//   4. off-diagonal blocks of Tinv by distance, warp-level tf32 MMAs per 8-column slab
//   5. Tc = Tinv diag(c); Eb = (Tinv - I) diag(beta) + diag(hi(beta)) (bf16),
//      diag(lo(beta)) (bf16), so that beta = hi + lo to 16 bits
//   6. MMAs W^T = K^T Tc^T,  X^T = V^T Eb^T + V^T diag(lo)^T  (= U~^T)
//   7. -W^T -> bf16 operand
//   8. MMAs X^T += S (-W)^T, O^T = S Qh^T (bf16, S from its bf16 copy);
//      then, reading X^T straight from TMEM as a tf32 operand,
//      S += X^T (D K) and O^T += X^T P^T; then the next chunk's Gram MMA
//   9. S -> bf16 operand, S master *= e^{g_L} of the next chunk; O^T -> TMA store
//
// The leading beta V term of U~ = beta V + (Tinv - I) beta V is carried to
// 16 bits (hi + lo bf16 diagonals against the exact bf16 V), and the state
// master stays fp32 throughout.  Within a chunk e^{g_r - g_s} is formed as
// e^{g_r} e^{-g_s} when the chunk's total log-decay is above -80 (both factors
// stay normal fp32 numbers); otherwise each entry takes exp2 of the difference.  A ragged last chunk is zero-filled by TMA and
// its gates padded with log_alpha = 0, beta = 0, which leaves the state and
// the valid outputs exact.
#pragma once

#include "common.cuh"
#include "tc_primitives.cuh"

namespace comba {
namespace tck {

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 256;

// TMEM columns (fp32, 128 lanes)
constexpr uint32_t TM_G = 0;     // Gram (lanes 0-63 K K^T, 64-127 Q K^T), then W^T
constexpr uint32_t TM_X = 64;    // X^T (lane = value index i, column = token r)
constexpr uint32_t TM_O = 128;   // O^T accumulator
constexpr uint32_t TM_S = 256;   // fp32 state master (lane i, column j)
constexpr uint32_t TM_COLS = 512;

// Shared memory (bytes from a 1024-aligned base).
constexpr uint32_t SM_KQ0 = 0;        // [K;Q] stage 0: 2 K-atoms x 128 rows x 128 B (bf16)
constexpr uint32_t SM_KQ1 = 32768;    // stage 1
constexpr uint32_t SM_V = 65536;      // V: 2 dv-atoms x 64 tokens x 128 B
constexpr uint32_t SM_S = 81920;      // S bf16: 2 K-atoms x 128 rows
constexpr uint32_t SM_W = 114688;     // -W bf16, MN-major: 128 rows (j) x 64 tokens
constexpr uint32_t SM_P = 131072;     // P fp32, K-major: 2 atoms (32 s) x 64 rows (K K^T first)
constexpr uint32_t SM_DK = 147456;    // (D K)^T fp32, K-major: 2 atoms (32 r) x 128 rows (j); out staging
constexpr uint32_t SM_F1 = 180224;    // fp32 64x64: A; then Tc (bf16) | Eb (bf16)
constexpr uint32_t SM_F2 = 196608;    // fp32 64x64: Tinv (upper blocks: scratch)
constexpr uint32_t SM_BLO = 212992;   // bf16 64x64 K-major: diag(lo(beta)), zero elsewhere
constexpr uint32_t SM_MISC = 221184;  // gates, barriers
constexpr uint32_t SM_END = SM_MISC + 2048;
constexpr uint32_t kSmemBytes = SM_END + 1024;

constexpr uint32_t KQ_ATOM = 16384;
constexpr uint32_t V_ATOM = 8192;
constexpr uint32_t OP_ATOM = 16384;
constexpr uint32_t F32_ATOM = 8192;   // 64 rows x 128 B
constexpr uint32_t DKT_ATOM = 16384;  // 128 rows x 128 B

constexpr uint32_t ID_G = tc::idesc_bf16(128, 64, false, false);    // [K;Q] K^T
constexpr uint32_t ID_WN = tc::idesc_bf16(128, 64, true, false);    // K^T Tc^T, V^T Eb^T
constexpr uint32_t ID_SW = tc::idesc_bf16(128, 64, false, true);    // S (-W)^T (W MN-major)
constexpr uint32_t ID_SQ = tc::idesc_bf16(128, 64, false, false);   // S Qh^T
constexpr uint32_t ID_SU = tc::idesc_tf32(128, 128, false, false);  // X^T (D K), (D K)^T K-major
constexpr uint32_t ID_XP = tc::idesc_tf32(128, 64, false, false);   // X^T P^T

constexpr float kLog2e = 1.4426950408889634f;

// fp32 64 x 64 scratch with an XOR swizzle on the column; byte address in a buffer.
__device__ __forceinline__ int fidx(int r, int s) { return r * 64 + (s ^ (r & 31)); }
__device__ __forceinline__ uint32_t faddr(uint32_t base, int r, int s) {
    return base + 4u * (uint32_t)fidx(r, s);
}

// c[16 x 8] += A-block(FA at ra, ca: 16 x 16) * B-slab(FB at rb, cb: 16 x 8), one warp, tf32.
__device__ __forceinline__ void slab_mma(float (&c)[4], uint32_t FA, int ra, int ca, uint32_t FB,
                                         int rb, int cb, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        uint32_t a[4], bb[2];
        a[0] = tc::f32_to_tf32(tc::lds_f32(faddr(FA, ra + g, ca + 8 * kk + t)));
        a[1] = tc::f32_to_tf32(tc::lds_f32(faddr(FA, ra + g + 8, ca + 8 * kk + t)));
        a[2] = tc::f32_to_tf32(tc::lds_f32(faddr(FA, ra + g, ca + 8 * kk + t + 4)));
        a[3] = tc::f32_to_tf32(tc::lds_f32(faddr(FA, ra + g + 8, ca + 8 * kk + t + 4)));
        bb[0] = tc::f32_to_tf32(tc::lds_f32(faddr(FB, rb + 8 * kk + t, cb + g)));
        bb[1] = tc::f32_to_tf32(tc::lds_f32(faddr(FB, rb + 8 * kk + t + 4, cb + g)));
        tc::mma_sync_tf32(c, a, bb);
    }
}

__device__ __forceinline__ void slab_store(uint32_t F, int r0, int c0, const float (&c)[4],
                                           float scale, int lane) {
    const int g = lane >> 2, t = lane & 3;
    tc::sts_f32(faddr(F, r0 + g, c0 + 2 * t), scale * c[0]);
    tc::sts_f32(faddr(F, r0 + g, c0 + 2 * t + 1), scale * c[1]);
    tc::sts_f32(faddr(F, r0 + g + 8, c0 + 2 * t), scale * c[2]);
    tc::sts_f32(faddr(F, r0 + g + 8, c0 + 2 * t + 1), scale * c[3]);
}

// Diagonal 16 x 16 block `blk` of (I + A)^{-1} (A strictly lower, fp32 at F1)
// into F2: one warp, lane j < 16 owns column j, right-looking substitution.
// Inside block `blk`, fidx(16 blk + r, 16 blk + s) = (16 blk + r) 64 + 32 (blk >> 1)
// + (s ^ r), so every A offset below is a compile-time constant.
__device__ __forceinline__ void diag_block_inverse(uint32_t F1, uint32_t F2, int blk, int lane) {
    const uint32_t base = 4u * (uint32_t)(16 * blk * 64 + 32 * (blk >> 1));
    const uint32_t Ab = F1 + base;
    const int j = lane & 15;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
    for (int s = 0; s < 15; ++s) {
        const float xs = x[s];
#pragma unroll
        for (int r = s + 1; r < 16; ++r)
            x[r] = fmaf(-tc::lds_f32(Ab + 4u * (uint32_t)(r * 64 + (s ^ r))), xs, x[r]);
    }
    if (lane < 16) {
        const uint32_t Tb = F2 + base;
#pragma unroll
        for (int r = 0; r < 16; ++r) tc::sts_f32(Tb + 4u * (uint32_t)(r * 64 + (j ^ r)), x[r]);
    }
}

// Off-diagonal blocks of (I + A)^{-1} by distance, T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj,
// one warp per 16 x 8 slab (warp 2j + slab); M_ij is staged in the upper block (j, i).
__device__ __forceinline__ void offdiag_inverse(uint32_t F1, uint32_t F2, int tid) {
    const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
    for (int dist = 1; dist <= 3; ++dist) {
        if (warp < 2 * (4 - dist)) {
            const int j = warp >> 1, nt = warp & 1, i = j + dist;
            float m[4] = {0.f, 0.f, 0.f, 0.f};
            for (int kb = j; kb < i; ++kb)
                slab_mma(m, F1, 16 * i, 16 * kb, F2, 16 * kb, 16 * j + 8 * nt, lane);
            slab_store(F2, 16 * j, 16 * i + 8 * nt, m, 1.f, lane);
            __syncwarp();
            float r2[4] = {0.f, 0.f, 0.f, 0.f};
            slab_mma(r2, F2, 16 * i, 16 * i, F2, 16 * j, 16 * i + 8 * nt, lane);
            slab_store(F2, 16 * i, 16 * j + 8 * nt, r2, -1.f, lane);
        }
        __syncthreads();
    }
}

// Exact-exponential fallbacks for a chunk whose total log-decay is at or
// below -80 (e^{-g} would leave the normal fp32 range): each entry takes exp2
// of its own exponent difference.  Kept out of line: they are rarely taken.
__device__ __noinline__ void a_row_exact(uint32_t F1, uint32_t gram_taddr, int r, int s0, float br,
                                         float gpr, uint32_t G2) {
    float gv[32];
    tc::tmem_ld32(gram_taddr, gv);
    tc::tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int s = s0 + e;
        const float v = br * exp2f(gpr - tc::lds_f32(G2 + 4u * s)) * gv[e];
        tc::sts_f32(faddr(F1, r, s), (s < r) ? v : 0.f);
    }
}

__device__ __noinline__ void p_row_exact(uint32_t prow, uint32_t gram_taddr, int r, int s0,
                                         float dh, uint32_t G2) {
    float gv[32];
    tc::tmem_ld32(gram_taddr, gv);
    tc::tmem_ld_wait();
    const float gr = tc::lds_f32(G2 + 4u * r);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int s = s0 + e;
        const uint32_t pa = prow + tc::sw128(r, e >> 2) + 4u * (e & 3);
        const float v = exp2f(gr - tc::lds_f32(G2 + 4u * s)) * fmaf(-dh, tc::lds_f32(pa), gv[e]);
        tc::sts_f32(pa, (s <= r) ? v : 0.f);
    }
}

// All threads wait on `bar`; a timeout is latched and makes every thread see
// `false` after the barrier.
__device__ __noinline__ bool cta_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                      volatile int* abort_flag) {
    if (!tc::mbar_wait(bar, parity, timeout_ns)) {
        *abort_flag = 1;
        latch_status(-4 /* COMBA_ETIMEOUT */);
    }
    __syncthreads();
    return *abort_flag == 0;
}

__device__ __forceinline__ uint4 pack8_bf16(const float* v) {
    uint4 w;
    w.x = tc::pack_bf16(v[0], v[1]);
    w.y = tc::pack_bf16(v[2], v[3]);
    w.z = tc::pack_bf16(v[4], v[5]);
    w.w = tc::pack_bf16(v[6], v[7]);
    return w;
}

// Gram MMA of chunk n by one thread: waits for the chunk's q/k tiles, then
// G = [K; Q] K^T into TMEM, committed to bars[5].
__device__ __noinline__ bool issue_gram_mma(uint64_t* bars, uint32_t sb, uint32_t tmem, int n,
                                            uint64_t timeout_ns) {
    if (!tc::mbar_wait(&bars[n & 1], (n >> 1) & 1, timeout_ns)) return false;
    const uint32_t kq_a = sb + ((n & 1) ? SM_KQ1 : SM_KQ0);
    tc::tc_fence_after();
    tc::mma_ak_bk(tmem + TM_G, kq_a, KQ_ATOM, kq_a, KQ_ATOM, ID_G, 8, 0);
    tc::mma_commit(&bars[5]);
    return true;
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const float* __restrict__ log_alpha, const float* __restrict__ beta,
                    const float* __restrict__ dvec, const float* S0, float* S_final, int T, int H,
                    unsigned long long timeout_ns) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sb = tc::smem_u32(sm);

    // gate tables (64 fp32 each), by shared address
    const uint32_t G2 = sb + SM_MISC;        // g_r log2(e)
    const uint32_t GP2 = G2 + 256;           // g_{r-1} log2(e)
    const uint32_t BT = G2 + 512;            // beta_r
    const uint32_t CS = G2 + 768;            // beta_r e^{g_{r-1}}
    const uint32_t EG = G2 + 1024;           // e^{g_r}
    const uint32_t ED = G2 + 1280;           // e^{g_L - g_r}
    const uint32_t IEG = G2 + 1536;          // e^{-g_r} (when the chunk allows)
    const uint32_t RED = G2 + 1792;          // [0..1] scan carries, [2..3] next-chunk sums
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM_MISC + 1856);  // kq0, kq1, v, mma, mma1, gram
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t F1 = sb + SM_F1, F2 = sb + SM_F2;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = tid & 127;          // TMEM lane
    const int half = tid >> 7;          // column half of that lane
    const int b = blockIdx.x / H, h = blockIdx.x % H;
    const float dh = dvec[h];
    const int nchunks = (T + kC - 1) / kC;
    const uint32_t trow = (uint32_t)((warp & 3) * 32) << 16;

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) tc::mbar_init(&bars[i], 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_v);
        tc::prefetch_tmap(&tm_o);
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, TM_COLS);
    for (int i = tid; i < 8192 / 16; i += kThreads)   // diag(lo(beta)): zero off the diagonal
        tc::sts_u32x4(sb + SM_BLO + 16u * i, make_uint4(0u, 0u, 0u, 0u));
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + trow;    // this thread's TMEM lane, column 0

    auto load_kq = [&](int n) {
        uint8_t* dst = sm + ((n & 1) ? SM_KQ1 : SM_KQ0);
        uint64_t* bar = &bars[n & 1];
        tc::mbar_arrive_expect_tx(bar, 32768);
        const int t0 = n * kC;
        tc::tma_load_4d(dst, &tm_k, bar, 0, h, t0, b);
        tc::tma_load_4d(dst + 8192, &tm_q, bar, 0, h, t0, b);
        tc::tma_load_4d(dst + KQ_ATOM, &tm_k, bar, 64, h, t0, b);
        tc::tma_load_4d(dst + KQ_ATOM + 8192, &tm_q, bar, 64, h, t0, b);
    };
    auto load_v = [&](int n) {
        tc::mbar_arrive_expect_tx(&bars[2], 16384);
        const int t0 = n * kC;
        tc::tma_load_4d(sm + SM_V, &tm_v, &bars[2], 0, h, t0, b);
        tc::tma_load_4d(sm + SM_V + V_ATOM, &tm_v, &bars[2], 64, h, t0, b);
    };
    auto issue_gram = [&](int n) -> bool { return issue_gram_mma(bars, sb, tmem, n, timeout_ns); };
    auto gate = [&](const float* p, int t) -> float {
        return (t < T) ? p[((size_t)b * T + t) * H + h] : 0.f;
    };

    if (tid == 0) {
        load_kq(0);
        if (nchunks > 1) load_kq(1);
        load_v(0);
        if (!issue_gram(0)) {
            *abort_flag = 1;
            latch_status(-4);
        }
    }
    // Gates of chunk 0 (threads 0..63), and their total for the initial decay.
    float la_c = 0.f, bt_c = 0.f, la_n = 0.f, bt_n = 0.f;
    if (tid < 64) {
        la_c = gate(log_alpha, tid);
        bt_c = gate(beta, tid);
        const float w = warp_sum(la_c);
        if (lane == 0) tc::sts_f32(RED + 8u + 4u * warp, w);
    }
    __syncthreads();
    const float eL0 = __expf(tc::lds_f32(RED + 8u) + tc::lds_f32(RED + 12u));

    // Initial state: fp32 master (decayed for chunk 0) into TMEM, bf16 copy.
    {
        const float* s0row = S0 ? S0 + ((size_t)blockIdx.x * kD + row) * kD + half * 64 : nullptr;
        const uint32_t sbase = sb + SM_S + half * OP_ATOM;
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 t4 = s0row ? *reinterpret_cast<const float4*>(s0row + part * 32 + e)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                v[e] = t4.x; v[e + 1] = t4.y; v[e + 2] = t4.z; v[e + 3] = t4.w;
            }
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                tc::sts_u32x4(sbase + tc::sw128(row, part * 4 + c4), pack8_bf16(v + c4 * 8));
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= eL0;
            tc::tmem_st32(tl + TM_S + half * 64 + part * 32, v);
        }
        tc::tmem_st_wait();
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    uint32_t mma_phase = 0, mma1_phase = 0;
    bool ok = *abort_flag == 0;
    COMBA_PHASE_BEGIN();
    for (int n = 0; n < nchunks && ok; ++n) {
        const int t0 = n * kC;
        const int st = n & 1;
        const uint32_t kq_a = sb + (st ? SM_KQ1 : SM_KQ0);
        const bool last = (n + 1 == nchunks);

        // ---- 1. gates ------------------------------------------------------------
        if (tid < 64) {
            if (!last) {   // prefetch the next chunk's gates
                la_n = gate(log_alpha, t0 + kC + tid);
                bt_n = gate(beta, t0 + kC + tid);
            }
            float x = la_c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            if (lane == 31) tc::sts_f32(RED + 4u * warp, x);
            tc::sts_f32(G2 + 4u * tid, x);
        }
        if (tid == 0) tc::bulk_wait_read0();   // previous out tile has left SM_DK
        __syncthreads();
        const float carry = tc::lds_f32(RED);
        const float gL = carry + tc::lds_f32(RED + 4u);
        const bool fast = gL > -80.f;           // e^{-g} stays a normal fp32 number
        if (tid < 64) {
            const float g = tc::lds_f32(G2 + 4u * tid) + (tid >= 32 ? carry : 0.f);
            const float gp = g - la_c;
            tc::sts_f32(BT + 4u * tid, bt_c);
            tc::sts_f32(CS + 4u * tid, bt_c * __expf(gp));
            tc::sts_f32(EG + 4u * tid, __expf(g));
            tc::sts_f32(IEG + 4u * tid, fast ? __expf(-g) : 0.f);
            tc::sts_f32(ED + 4u * tid, __expf(gL - g));
            tc::sts_f32(GP2 + 4u * tid, gp * kLog2e);
            tc::sts_f32(G2 + 4u * tid, g * kLog2e);
        }
        COMBA_PHASE(0);

        // ---- 2. Gram of this chunk (issued earlier) -----------------------------------
        if (!cta_wait(&bars[st], (n >> 1) & 1, timeout_ns, abort_flag)) { ok = false; break; }
        if (!cta_wait(&bars[5], n & 1, timeout_ns, abort_flag)) { ok = false; break; }
        tc::tc_fence_after();
        COMBA_PHASE(1);

        // ---- 3. K K^T -> P buffer, A -> F1; then P/Qh/(DK)^T || diagonal inverse -------
        {
            float gv[32];
            tc::tmem_ld32(tl + TM_G + half * 32, gv);
            tc::tmem_ld_wait();
            const int s0 = half * 32;
            const uint32_t prow = sb + SM_P + half * F32_ATOM;
            if (row < 64) {
                const int r = row;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    tc::sts_f32x4(prow + tc::sw128(r, c),
                                  make_float4(gv[4 * c], gv[4 * c + 1], gv[4 * c + 2], gv[4 * c + 3]));
                if (fast) {
                    const float cr = tc::lds_f32(CS + 4u * r);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 ig = tc::lds_f32x4(IEG + 4u * (s0 + 4 * c));
                        const float iv[4] = {ig.x, ig.y, ig.z, ig.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int s = s0 + 4 * c + e;
                            tc::sts_f32(faddr(F1, r, s), (s < r) ? cr * iv[e] * gv[4 * c + e] : 0.f);
                        }
                    }
                } else {
                    a_row_exact(F1, tl + TM_G + half * 32, r, s0, tc::lds_f32(BT + 4u * r),
                                tc::lds_f32(GP2 + 4u * r), G2);
                }
                if (!last && tid < 64) {   // total log-decay of the next chunk
                    const float w = warp_sum(la_n);
                    if (lane == 0) tc::sts_f32(RED + 8u + 4u * warp, w);
                }
            }
            __syncthreads();
            COMBA_PHASE(9);
            if (row >= 64) {
                // P in place over K K^T (row r, columns s0 .. s0 + 31)
                const int r = row - 64;
                const float er = tc::lds_f32(EG + 4u * r);
                if (fast) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t pa = prow + tc::sw128(r, c);
                        const float4 kk = tc::lds_f32x4(pa);
                        const float4 ig = tc::lds_f32x4(IEG + 4u * (s0 + 4 * c));
                        const int s = s0 + 4 * c;
                        float4 p;
                        p.x = (s + 0 <= r) ? er * ig.x * fmaf(-dh, kk.x, gv[4 * c + 0]) : 0.f;
                        p.y = (s + 1 <= r) ? er * ig.y * fmaf(-dh, kk.y, gv[4 * c + 1]) : 0.f;
                        p.z = (s + 2 <= r) ? er * ig.z * fmaf(-dh, kk.z, gv[4 * c + 2]) : 0.f;
                        p.w = (s + 3 <= r) ? er * ig.w * fmaf(-dh, kk.w, gv[4 * c + 3]) : 0.f;
                        tc::sts_f32x4(pa, p);
                    }
                } else {
                    p_row_exact(prow, tl + TM_G + half * 32, r, s0, dh, G2);
                }
                // Qh (over Q) and (D K)^T for row r, key columns 64 half .. 64 half + 63
                const float edr = tc::lds_f32(ED + 4u * r);
                const uint32_t dka = sb + SM_DK + (r >> 5) * DKT_ATOM + (r & 3) * 4;
                const uint32_t rc = (r & 31) >> 2;
#pragma unroll 2
                for (int c = 0; c < 8; ++c) {
                    const uint32_t off = kq_a + half * KQ_ATOM + tc::sw128(r, c);
                    const uint4 kw = tc::lds_u32x4(off);
                    uint4 qw = tc::lds_u32x4(off + 8192);
                    const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kw);
                    __nv_bfloat162* q2 = reinterpret_cast<__nv_bfloat162*>(&qw);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 kf = __bfloat1622float2(k2[e]);
                        const float2 qf = __bfloat1622float2(q2[e]);
                        q2[e] = __floats2bfloat162_rn(er * fmaf(-dh, kf.x, qf.x), er * fmaf(-dh, kf.y, qf.y));
                        const int j = 64 * half + 8 * c + 2 * e;
                        tc::sts_f32(dka + tc::sw128(j, rc), edr * kf.x);
                        tc::sts_f32(dka + tc::sw128(j + 1, rc), edr * kf.y);
                    }
                    tc::sts_u32x4(off + 8192, qw);
                }
            } else {
                // warps 0, 1, 4, 5 -> diagonal blocks 0, 1, 2, 3
                diag_block_inverse(F1, F2, (warp & 1) + 2 * half, lane);
            }
            __syncthreads();
        }
        COMBA_PHASE(2);

        // ---- 4. off-diagonal blocks of the inverse -----------------------------------
        offdiag_inverse(F1, F2, tid);
        COMBA_PHASE(3);

        // ---- 5. Tc, Eb (+ diag hi(beta)) over F1; diag lo(beta) ---------------------------
        {
            const int r = tid & 63, qq = tid >> 6;   // row, quarter of the columns
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                const int c = 2 * qq + c2;
                float tcv[8], ebv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = c * 8 + e;
                    const float t = tc::lds_f32(faddr(F2, r, s));
                    const float cv = tc::lds_f32(CS + 4u * s), bv = tc::lds_f32(BT + 4u * s);
                    tcv[e] = (s <= r) ? t * cv : 0.f;
                    ebv[e] = (s < r) ? t * bv : ((s == r) ? bv : 0.f);
                }
                tc::sts_u32x4(F1 + tc::sw128(r, c), pack8_bf16(tcv));
                tc::sts_u32x4(F1 + 8192 + tc::sw128(r, c), pack8_bf16(ebv));
            }
            if (tid < 64) {
                const float bv = tc::lds_f32(BT + 4u * tid);
                const float bh = __bfloat162float(__float2bfloat16_rn(bv));
                const __nv_bfloat16 lo = __float2bfloat16_rn(bv - bh);
                tc::sts_u16(sb + SM_BLO + tc::sw128(tid, tid >> 3) + (tid & 7) * 2,
                            *reinterpret_cast<const unsigned short*>(&lo));
            }
        }
        tc::fence_proxy_async_smem();
        COMBA_PHASE(4);

        // ---- 6. W^T = K^T Tc^T;  X^T = V^T Eb^T + V^T diag(lo)^T ---------------------------
        if (!cta_wait(&bars[2], n & 1, timeout_ns, abort_flag)) { ok = false; break; }
        if (tid == 0) {
            tc::tc_fence_after();
            tc::mma_amn_bk(tmem + TM_G, kq_a, KQ_ATOM, F1, ID_WN, 4, 0);
            tc::mma_amn_bk(tmem + TM_X, sb + SM_V, V_ATOM, F1 + 8192, ID_WN, 4, 0);
            tc::mma_amn_bk(tmem + TM_X, sb + SM_V, V_ATOM, sb + SM_BLO, ID_WN, 4, 1);
            tc::mma_commit(&bars[3]);
        }
        if (!cta_wait(&bars[3], mma_phase, timeout_ns, abort_flag)) { ok = false; break; }
        mma_phase ^= 1;
        tc::tc_fence_after();
        if (tid == 0 && !last) {
            tc::fence_proxy_async_smem();
            load_v(n + 1);
        }
        COMBA_PHASE(5);

        // ---- 7. -W operand (MN-major: row j holds -W[0..63][j]) ------------------------------
        {
            float w[32];
            tc::tmem_ld32(tl + TM_G + half * 32, w);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = -w[e];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                tc::sts_u32x4(sb + SM_W + tc::sw128(row, half * 4 + c4), pack8_bf16(w + c4 * 8));
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        COMBA_PHASE(6);

        // ---- 8. X^T += S (-W)^T, O^T = S Qh^T; S += X^T (D K), O^T += X^T P^T; next Gram ------
        if (tid == 0) {
            tc::tc_fence_after();
            tc::mma_ak_bmn(tmem + TM_X, sb + SM_S, OP_ATOM, sb + SM_W, 8192, ID_SW, 8, 8, 1);
            tc::mma_commit(&bars[4]);
            tc::mma_ak_bk(tmem + TM_O, sb + SM_S, OP_ATOM, kq_a + 8192, KQ_ATOM, ID_SQ, 8, 0);
            bool good = tc::mbar_wait(&bars[4], mma1_phase, timeout_ns);
            COMBA_PHASE(10);
            if (good) {
                tc::tc_fence_after();
                tc::mma_tf32_ta_bk(tmem + TM_S, tmem + TM_X, sb + SM_DK, DKT_ATOM, ID_SU, 8, 1);
                tc::mma_tf32_ta_bk(tmem + TM_O, tmem + TM_X, sb + SM_P, F32_ATOM, ID_XP, 8, 1);
                tc::mma_commit(&bars[3]);
                COMBA_PHASE(11);
                if (!last) good = issue_gram(n + 1);          // TM_G is free again
                COMBA_PHASE(12);
            }
            if (!good) {
                *abort_flag = 1;
                latch_status(-4);
            }
        }
        mma1_phase ^= 1;
        if (!cta_wait(&bars[3], mma_phase, timeout_ns, abort_flag)) { ok = false; break; }
        mma_phase ^= 1;
        tc::tc_fence_after();
        if (tid == 0 && n + 2 < nchunks) {   // stage st is free: its Qh was read by the MMAs above
            tc::fence_proxy_async_smem();
            load_kq(n + 2);
        }
        COMBA_PHASE(7);

        // ---- 9. S -> bf16 operand, decay for the next chunk; output tile -------------------
        {
            const float eLn = last ? 1.f : __expf(tc::lds_f32(RED + 8u) + tc::lds_f32(RED + 12u));
            float* sfrow = (last && S_final)
                               ? S_final + ((size_t)blockIdx.x * kD + row) * kD + half * 64
                               : nullptr;
            const uint32_t sbase = sb + SM_S + half * OP_ATOM;
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
                float v[32];
                tc::tmem_ld32(tl + TM_S + half * 64 + part * 32, v);
                tc::tmem_ld_wait();
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                    tc::sts_u32x4(sbase + tc::sw128(row, part * 4 + c4), pack8_bf16(v + c4 * 8));
                if (sfrow) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(sfrow + part * 32 + e) =
                            make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                } else if (!last) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] *= eLn;
                    tc::tmem_st32(tl + TM_S + half * 64 + part * 32, v);
                }
            }
            // O^T row i (value index) -> out tile [token][i], two 64-wide boxes
            const uint32_t ot = sb + SM_DK + (row >> 6) * 8192 + (row & 7) * 2;
            const int oc = (row & 63) >> 3;
            float o[32];
            tc::tmem_ld32(tl + TM_O + half * 32, o);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const __nv_bfloat16 ob = __float2bfloat16_rn(o[e]);
                tc::sts_u16(ot + tc::sw128(half * 32 + e, oc), *reinterpret_cast<const unsigned short*>(&ob));
            }
            tc::tmem_st_wait();
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc::tma_store_4d(&tm_o, sm + SM_DK, 0, h, t0, b);
            tc::tma_store_4d(&tm_o, sm + SM_DK + 8192, 64, h, t0, b);
            tc::bulk_commit();
        }
        la_c = la_n;
        bt_c = bt_n;
        COMBA_PHASE(8);
    }

    COMBA_PHASE_END();
    if (tid == 0) tc::bulk_wait0();
    if (!ok) tc::mbar_wait(&bars[3], mma_phase, timeout_ns);
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, TM_COLS);
}

}  // namespace tck

// ---------------------------------------------------------------- host side
inline bool tc_supported(int dk, int dv, int chunk) { return dk == 128 && dv == 128 && chunk == 64; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [B, T, H, 128] bf16 viewed as 4-D (d, h, t, b); box = 64 x 1 x 64 x 1, 128B swizzle.
inline bool make_tmap_bthd(CUtensorMap* map, const void* ptr, int B, int T, int H) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {128 * 2, (cuuint64_t)H * 128 * 2, (cuuint64_t)T * H * 128 * 2};
    const cuuint32_t box[4] = {64, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;   // 2 s per wait

inline int launch_chunk_tc(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* d, const float* S0, void* out,
                           float* S_final, int B, int T, int H, cudaStream_t stream,
                           unsigned long long timeout_ns = kWaitTimeoutNs) {
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -3;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(tck::chunk_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tck::kSmemBytes) != cudaSuccess)
            return -3;
        attr_set[dev] = true;
    }
    CUtensorMap tq, tk, tv, to;
    if (!make_tmap_bthd(&tq, q, B, T, H) || !make_tmap_bthd(&tk, k, B, T, H) ||
        !make_tmap_bthd(&tv, v, B, T, H) || !make_tmap_bthd(&to, out, B, T, H))
        return -3;
    tck::chunk_fwd_tc_kernel<<<(unsigned)(B * H), tck::kThreads, tck::kSmemBytes, stream>>>(
        tq, tk, tv, to, log_alpha, beta, d, S0, S_final, T, H, timeout_ns);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace comba
