// Tensor-core chunk-wise Comba forward for bf16 inputs, dk = dv = 128, chunk 64.
//
// One CTA (8 warps) owns one (b, h) chain and walks its chunks in order.
// Thread t owns TMEM lane t % 128 and half of that lane's columns.  Per chunk
// (chunk-start state S, local tokens r, s, g_r = sum_{i<=r} log_alpha_i, g_0 = 0;
// the write-up's "block-recurrent, intra-block parallel" form with a single
// inverse for the intermediates W and U, section "硬件高效的分块并行计算"):
//
//   1. gates (prefetched one chunk ahead): g by warp-shuffle scan, e^{g_r},
//      e^{g_L - g_r}, c_r = beta_r e^{g_{r-1}}
//   2. Gram MMA      G = [K; Q] K^T                                  (bf16 -> TMEM)
//   3. P_rs = e^{g_r-g_s}(Q K^T - d K K^T)_rs (s <= r) as an fp32 operand;
//      A_rs = beta_r e^{g_{r-1}-g_s}(K K^T)_rs (s < r)
//   4. Tinv = (I + A)^{-1}: 16 x 16 diagonal blocks by forward substitution,
//      off-diagonal blocks by distance with warp-level tf32 MMAs
//   5. Tc = Tinv diag(c), Eb = (Tinv - I) diag(beta) (bf16); Qh = diag(e^g)(Q - d K)
//      over Q; (D K)^T with D = diag(e^{g_L - g}) (fp32 operand, K-major)
//   6. X^T <- beta V^T (TMEM store); MMAs W^T = K^T Tc^T, X^T += V^T Eb^T
//   7. -W^T -> bf16 operand
//   8. MMAs X^T += S (-W)^T, O^T = S Qh^T (bf16, S from its bf16 copy);
//      then, reading X^T straight from TMEM as a tf32 operand,
//      S += X^T (D K) and O^T += X^T P^T
//   9. S -> bf16 operand, S master *= e^{g_L} of the next chunk; O^T -> TMA store
//
// The leading beta V term of U~ = beta V + (Tinv - I) beta V and the state
// master stay fp32 throughout.  A ragged last chunk is zero-filled by TMA and
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
constexpr uint32_t SM_P = 131072;     // P fp32, K-major: 2 atoms (32 s) x 64 rows
constexpr uint32_t SM_DK = 147456;    // (D K)^T fp32, K-major: 2 atoms (32 r) x 128 rows (j); out staging
constexpr uint32_t SM_F1 = 180224;    // fp32 64x64: K K^T, then A; then Tc (bf16) | Eb (bf16)
constexpr uint32_t SM_F2 = 196608;    // fp32 64x64: Tinv (upper blocks: scratch)
constexpr uint32_t SM_MISC = 212992;  // gates, barriers
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

// fp32 64 x 64 scratch with an XOR swizzle on the column.
__device__ __forceinline__ int fidx(int r, int s) { return r * 64 + (s ^ (r & 31)); }

// C[16 x 16] += A-block(FA at ra, ca) * B-block(FB at rb, cb), one warp, tf32.
__device__ __forceinline__ void blk_mma(float (&c)[2][4], const float* FA, int ra, int ca,
                                        const float* FB, int rb, int cb, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        uint32_t a[4];
        a[0] = tc::f32_to_tf32(FA[fidx(ra + g, ca + 8 * kk + t)]);
        a[1] = tc::f32_to_tf32(FA[fidx(ra + g + 8, ca + 8 * kk + t)]);
        a[2] = tc::f32_to_tf32(FA[fidx(ra + g, ca + 8 * kk + t + 4)]);
        a[3] = tc::f32_to_tf32(FA[fidx(ra + g + 8, ca + 8 * kk + t + 4)]);
#pragma unroll
        for (int nn = 0; nn < 2; ++nn) {
            uint32_t b[2];
            b[0] = tc::f32_to_tf32(FB[fidx(rb + 8 * kk + t, cb + 8 * nn + g)]);
            b[1] = tc::f32_to_tf32(FB[fidx(rb + 8 * kk + t + 4, cb + 8 * nn + g)]);
            tc::mma_sync_tf32(c[nn], a, b);
        }
    }
}

__device__ __forceinline__ void blk_store(float* F, int r0, int c0, const float (&c)[2][4],
                                          float scale, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nn = 0; nn < 2; ++nn) {
        F[fidx(r0 + g, c0 + 8 * nn + 2 * t)] = scale * c[nn][0];
        F[fidx(r0 + g, c0 + 8 * nn + 2 * t + 1)] = scale * c[nn][1];
        F[fidx(r0 + g + 8, c0 + 8 * nn + 2 * t)] = scale * c[nn][2];
        F[fidx(r0 + g + 8, c0 + 8 * nn + 2 * t + 1)] = scale * c[nn][3];
    }
}

// (I + A)^{-1} for strictly lower A (64 x 64 fp32 in F1) into F2 (lower triangle
// with the unit diagonal; the upper 16 x 16 blocks of F2 are used as scratch).
__device__ __forceinline__ void unit_lower_inverse(const float* __restrict__ F1, float* F2,
                                                   int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    if (warp < 4) {
        // Diagonal block `warp`, column j per lane, right-looking substitution.
        const int o = 16 * warp;
        const int j = lane & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int s = 0; s < 15; ++s) {
            const float xs = x[s];
#pragma unroll
            for (int r = s + 1; r < 16; ++r) x[r] = fmaf(-F1[fidx(o + r, o + s)], xs, x[r]);
        }
        if (lane < 16) {
#pragma unroll
            for (int r = 0; r < 16; ++r) F2[fidx(o + r, o + j)] = x[r];
        }
    }
    __syncthreads();
    // Off-diagonal blocks by distance: T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj
    // (warp j computes block (j + dist, j); M_ij is staged in upper block (j, i)).
#pragma unroll
    for (int dist = 1; dist <= 3; ++dist) {
        if (warp < 4 - dist) {
            const int j = warp, i = warp + dist;
            float m[2][4] = {};
            for (int kb = j; kb < i; ++kb) blk_mma(m, F1, 16 * i, 16 * kb, F2, 16 * kb, 16 * j, lane);
            blk_store(F2, 16 * j, 16 * i, m, 1.f, lane);
            __syncwarp();
            float r2[2][4] = {};
            blk_mma(r2, F2, 16 * i, 16 * i, F2, 16 * j, 16 * i, lane);
            blk_store(F2, 16 * i, 16 * j, r2, -1.f, lane);
        }
        __syncthreads();
    }
}

// All threads wait on `bar`; a timeout is latched and makes every thread see
// `false` after the barrier.
__device__ __forceinline__ bool cta_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
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

__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const float* __restrict__ log_alpha, const float* __restrict__ beta,
                    const float* __restrict__ dvec, const float* S0, float* S_final, int T, int H,
                    unsigned long long timeout_ns) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sb = tc::smem_u32(sm);

    float* g2_s = reinterpret_cast<float*>(sm + SM_MISC);  // g_r log2(e)
    float* gp2_s = g2_s + 64;                               // g_{r-1} log2(e)
    float* bt_s = g2_s + 128;                               // beta_r
    float* c_s = g2_s + 192;                                // beta_r e^{g_{r-1}}
    float* eg_s = g2_s + 256;                               // e^{g_r}
    float* ed_s = g2_s + 320;                               // e^{g_L - g_r}
    float* red_s = g2_s + 384;                              // [0..1] scan carries, [2..3] sums
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM_MISC + 1600);  // kq0, kq1, v, mma, mma1
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* F1 = reinterpret_cast<float*>(sm + SM_F1);
    float* F2 = reinterpret_cast<float*>(sm + SM_F2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = tid & 127;          // TMEM lane
    const int half = tid >> 7;          // column half of that lane
    const int b = blockIdx.x / H, h = blockIdx.x % H;
    const float dh = dvec[h];
    const int nchunks = (T + kC - 1) / kC;
    const uint32_t trow = (uint32_t)((warp & 3) * 32) << 16;

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) tc::mbar_init(&bars[i], 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_v);
        tc::prefetch_tmap(&tm_o);
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, TM_COLS);
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
    auto gate = [&](const float* p, int t) -> float {
        return (t < T) ? p[((size_t)b * T + t) * H + h] : 0.f;
    };
    // Sum over the 64 gates held by threads 0..63 (warps 0 and 1); all threads call.
    auto sum64 = [&](float x, int slot) -> float {
        if (tid < 64) {
            x = warp_sum(x);
            if (lane == 0) red_s[2 + warp] = x;
        }
        __syncthreads();
        const float r = red_s[2] + red_s[3];
        (void)slot;
        return r;
    };

    if (tid == 0) {
        load_kq(0);
        if (nchunks > 1) load_kq(1);
        load_v(0);
    }
    // Gates of chunk 0 and, one chunk ahead, of chunk 1 (threads 0..63).
    float la_c = 0.f, bt_c = 0.f, la_n = 0.f, bt_n = 0.f;
    if (tid < 64) {
        la_c = gate(log_alpha, tid);
        bt_c = gate(beta, tid);
    }
    const float eL0 = __expf(sum64(la_c, 0));

    // Initial state: fp32 master (decayed for chunk 0) into TMEM, bf16 copy.
    {
        const float* s0row = S0 ? S0 + ((size_t)blockIdx.x * kD + row) * kD + half * 64 : nullptr;
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 t4 = s0row ? *reinterpret_cast<const float4*>(s0row + part * 32 + e)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                v[e] = t4.x; v[e + 1] = t4.y; v[e + 2] = t4.z; v[e + 3] = t4.w;
            }
            uint8_t* base = sm + SM_S + half * OP_ATOM;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                *reinterpret_cast<uint4*>(base + tc::sw128(row, part * 4 + c4)) = pack8_bf16(v + c4 * 8);
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
    bool ok = true;
    COMBA_PHASE_BEGIN();
    for (int n = 0; n < nchunks && ok; ++n) {
        const int t0 = n * kC;
        const int st = n & 1;
        uint8_t* kq = sm + (st ? SM_KQ1 : SM_KQ0);
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
            if (lane == 31) red_s[warp] = x;
            g2_s[tid] = x;     // inclusive within the warp for now
        }
        if (tid == 0) tc::bulk_wait_read0();   // previous out tile has left SM_DK
        __syncthreads();
        if (tid < 64) {
            const float g = g2_s[tid] + (tid >= 32 ? red_s[0] : 0.f);
            const float gL = red_s[0] + red_s[1];
            const float gp = g - la_c;
            bt_s[tid] = bt_c;
            c_s[tid] = bt_c * __expf(gp);
            eg_s[tid] = __expf(g);
            ed_s[tid] = __expf(gL - g);
            gp2_s[tid] = gp * kLog2e;
            __syncwarp();
            g2_s[tid] = g * kLog2e;
        }
        COMBA_PHASE(0);

        // ---- 2. Gram MMA ------------------------------------------------------------
        if (!cta_wait(&bars[st], (n >> 1) & 1, timeout_ns, abort_flag)) { ok = false; break; }
        if (tid == 0) {
            tc::tc_fence_after();
            tc::mma_ak_bk(tmem + TM_G, kq_a, KQ_ATOM, kq_a, KQ_ATOM, ID_G, 8, 0);
            tc::mma_commit(&bars[3]);
        }
        if (!cta_wait(&bars[3], mma_phase, timeout_ns, abort_flag)) { ok = false; break; }
        mma_phase ^= 1;
        tc::tc_fence_after();
        COMBA_PHASE(1);

        // ---- 3. P (fp32 operand) and A ----------------------------------------------
        {
            float gv[32];
            tc::tmem_ld32(tl + TM_G + half * 32, gv);
            tc::tmem_ld_wait();
            const int s0 = half * 32;
            if (row < 64) {
#pragma unroll
                for (int e = 0; e < 32; ++e) F1[fidx(row, s0 + e)] = gv[e];
            }
            __syncthreads();
            if (row >= 64) {
                const int r = row - 64;
                const float gr = g2_s[r];
                uint8_t* prow = sm + SM_P + half * F32_ATOM;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float p[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = s0 + c * 4 + e;
                        p[e] = (s <= r) ? exp2f(gr - g2_s[s]) * (gv[c * 4 + e] - dh * F1[fidx(r, s)]) : 0.f;
                    }
                    *reinterpret_cast<float4*>(prow + tc::sw128(r, c)) = make_float4(p[0], p[1], p[2], p[3]);
                }
            } else {
                const float br = bt_s[row], gpr = gp2_s[row];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int s = s0 + e;
                    gv[e] = (s < row) ? br * exp2f(gpr - g2_s[s]) * gv[e] : 0.f;
                }
            }
            __syncthreads();
            if (row < 64) {
#pragma unroll
                for (int e = 0; e < 32; ++e) F1[fidx(row, s0 + e)] = gv[e];
            }
            __syncthreads();
        }
        COMBA_PHASE(2);

        // ---- 4. inverse -------------------------------------------------------------------
        unit_lower_inverse(F1, F2, tid);
        COMBA_PHASE(3);

        // ---- 5. Tc, Eb (bf16, over F1), Qh (over Q), D K (fp32) ----------------------------
        {
            const int r = tid & 63, qq = tid >> 6;   // row, quarter of the columns
            // Tc, Eb: columns 16 qq .. 16 qq + 15 -> chunks 2 qq, 2 qq + 1
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                const int c = 2 * qq + c2;
                float tcv[8], ebv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = c * 8 + e;
                    const float t = (s <= r) ? F2[fidx(r, s)] : 0.f;
                    tcv[e] = t * c_s[s];
                    ebv[e] = (s < r) ? t * bt_s[s] : 0.f;
                }
                *reinterpret_cast<uint4*>(sm + SM_F1 + tc::sw128(r, c)) = pack8_bf16(tcv);
                *reinterpret_cast<uint4*>(sm + SM_F1 + 8192 + tc::sw128(r, c)) = pack8_bf16(ebv);
            }
            // Qh and D K for key columns 32 qq .. 32 qq + 31 (K atom qq / 2, chunks 4 (qq % 2) ..)
            const float er = eg_s[r], edr = ed_s[r];
            const uint32_t atom = (qq >> 1) * KQ_ATOM;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const int c = (qq & 1) * 4 + c4;
                const uint32_t off = atom + tc::sw128(r, c);
                const uint4 kw = *reinterpret_cast<const uint4*>(kq + off);
                uint4 qw = *reinterpret_cast<const uint4*>(kq + 8192 + off);
                const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kw);
                __nv_bfloat162* q2 = reinterpret_cast<__nv_bfloat162*>(&qw);
                float dk[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kf = __bfloat1622float2(k2[e]);
                    const float2 qf = __bfloat1622float2(q2[e]);
                    q2[e] = __floats2bfloat162_rn(er * (qf.x - dh * kf.x), er * (qf.y - dh * kf.y));
                    dk[2 * e] = edr * kf.x;
                    dk[2 * e + 1] = edr * kf.y;
                }
                *reinterpret_cast<uint4*>(kq + 8192 + off) = qw;
                // (D K)^T, K-major fp32: row j = 32 qq + 8 c4 + e, token r in atom r / 32
                uint8_t* dka = sm + SM_DK + (r >> 5) * DKT_ATOM + (r & 3) * 4;
                const uint32_t rc = (r & 31) >> 2;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    *reinterpret_cast<float*>(dka + tc::sw128(32 * qq + 8 * c4 + e, rc)) = dk[e];
            }
        }
        tc::fence_proxy_async_smem();
        COMBA_PHASE(4);

        // ---- 6. X^T <- beta V^T; W^T = K^T Tc^T; X^T += V^T Eb^T ---------------------------
        if (!cta_wait(&bars[2], n & 1, timeout_ns, abort_flag)) { ok = false; break; }
        {
            const uint8_t* vt = sm + SM_V + (row >> 6) * V_ATOM;
            const int vc = (row & 63) >> 3, ve = row & 7;
            float bv[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int r = half * 32 + e;
                const float vv = __bfloat162float(
                    *reinterpret_cast<const __nv_bfloat16*>(vt + tc::sw128(r, vc) + ve * 2));
                bv[e] = bt_s[r] * vv;
            }
            tc::tmem_st32(tl + TM_X + half * 32, bv);
            tc::tmem_st_wait();
        }
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc::tc_fence_after();
            tc::mma_amn_bk(tmem + TM_G, kq_a, KQ_ATOM, sb + SM_F1, ID_WN, 4, 0);
            tc::mma_amn_bk(tmem + TM_X, sb + SM_V, V_ATOM, sb + SM_F1 + 8192, ID_WN, 4, 1);
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
                *reinterpret_cast<uint4*>(sm + SM_W + tc::sw128(row, half * 4 + c4)) = pack8_bf16(w + c4 * 8);
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        COMBA_PHASE(6);

        // ---- 8. X^T += S (-W)^T, O^T = S Qh^T; then S += X^T (D K), O^T += X^T P^T ---------
        if (tid == 0) {
            tc::tc_fence_after();
            tc::mma_ak_bmn(tmem + TM_X, sb + SM_S, OP_ATOM, sb + SM_W, 8192, ID_SW, 8, 8, 1);
            tc::mma_ak_bk(tmem + TM_O, sb + SM_S, OP_ATOM, kq_a + 8192, KQ_ATOM, ID_SQ, 8, 0);
            tc::mma_commit(&bars[4]);
            const bool done1 = tc::mbar_wait(&bars[4], mma1_phase, timeout_ns);
            if (done1) {
                tc::tc_fence_after();
                if (n + 2 < nchunks) {
                    tc::fence_proxy_async_smem();
                    load_kq(n + 2);
                }
                tc::mma_tf32_ta_bk(tmem + TM_S, tmem + TM_X, sb + SM_DK, DKT_ATOM, ID_SU, 8, 1);
                tc::mma_tf32_ta_bk(tmem + TM_O, tmem + TM_X, sb + SM_P, F32_ATOM, ID_XP, 8, 1);
                tc::mma_commit(&bars[3]);
            } else {
                *abort_flag = 1;
                latch_status(-4);
            }
        }
        mma1_phase ^= 1;
        if (!cta_wait(&bars[3], mma_phase, timeout_ns, abort_flag)) { ok = false; break; }
        mma_phase ^= 1;
        tc::tc_fence_after();
        COMBA_PHASE(7);

        // ---- 9. S -> bf16 operand, decay for the next chunk; output tile -------------------
        {
            const float eLn = last ? 1.f : __expf(sum64(la_n, 1));
            float* sfrow = (last && S_final)
                               ? S_final + ((size_t)blockIdx.x * kD + row) * kD + half * 64
                               : nullptr;
            uint8_t* base = sm + SM_S + half * OP_ATOM;
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
                float v[32];
                tc::tmem_ld32(tl + TM_S + half * 64 + part * 32, v);
                tc::tmem_ld_wait();
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                    *reinterpret_cast<uint4*>(base + tc::sw128(row, part * 4 + c4)) = pack8_bf16(v + c4 * 8);
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
            uint8_t* ot = sm + SM_DK + (row >> 6) * 8192;
            const int oc = (row & 63) >> 3, oe = row & 7;
            float o[32];
            tc::tmem_ld32(tl + TM_O + half * 32, o);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e)
                *reinterpret_cast<__nv_bfloat16*>(ot + tc::sw128(half * 32 + e, oc) + oe * 2) =
                    __float2bfloat16_rn(o[e]);
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
