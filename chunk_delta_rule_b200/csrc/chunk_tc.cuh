// Tensor-core chunk-wise Comba forward for bf16 inputs, dk = dv = 128, chunk 64.
//
// One CTA owns one (b, h) chain and walks its chunks in order, in the write-up's
// "block-recurrent, intra-block parallel" form with a single inverse for the
// intermediates W and U (section "硬件高效的分块并行计算").  Per chunk (chunk-start
// state S, local tokens r, s, g_r = sum_{i<=r} log_alpha_i):
//
//   A_rs = beta_r e^{g_{r-1} - g_s} (k_r . k_s)  (s < r),   Tinv = (I + A)^{-1}
//   W = Tinv diag(beta e^{g_{r-1}}) K,   U~ = Tinv diag(beta) V,   X = U~ - W S^T
//   P_rs = e^{g_r - g_s} (q_r - d k_r) . k_s  (s <= r)
//   O = diag(e^g)(Q - d K) S^T + P X,    S <- e^{g_L} S + (X diag(e^{g_L - g}))^T K
//
// Three warp-specialised roles run different chunks at once and hand buffers
// over through mbarriers:
//   prep group (7 warps): gate tables (one chunk ahead), A and P from the Gram
//     products, the 16 x 16 diagonal inverse blocks by substitution, then Tinv
//     by block forward substitution in 8-column strips on warp MMAs, written out
//     as Tc = Tinv diag(c) and Eb = Tinv diag(beta) (bf16);
//   MMA-issue warp: every tcgen05 MMA (Gram, W^T / U~^T, X and O against the state,
//     the state update and the intra-chunk output), in a fixed order per chunk;
//   state group (4 warps, TMEM lane = value index): -W and Qh operands, X' = X
//     diag(e^{g_L - g}) as bf16 hi + lo, the O readout, the bf16 copy and decay of
//     the fp32 state master in TMEM, and the out tile's TMA store.
// The leading beta V term of U~ is carried to 16 bits (hi + lo bf16 diagonals
// against the exact bf16 V).  Within a chunk e^{g_r - g_s} is formed as
// e^{g_r} e^{-g_s} when the chunk's total log-decay is above -80 (both factors stay
// normal fp32 numbers); otherwise each entry takes exp2 of the difference.  A ragged
// last chunk is zero-filled by TMA and its gates padded with log_alpha = 0,
// beta = 0, which leaves the state and the valid outputs exact.
#pragma once

#include "common.cuh"
#include "tc_primitives.cuh"

namespace comba {
namespace tck {

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 384;        // warps 0-3: state group; warp 4: MMA issue; warps 5-11: prep
constexpr int kStateThreads = 128;
constexpr int kCtlWarp = 4;
constexpr int kPrepThreads = 224;
constexpr int kPrepBase = 160;       // first thread of the prep group
constexpr int BAR_PREP = 1;          // named barrier ids: the prep group
constexpr int BAR_STATE = 2;         // the state group
constexpr int BAR_KK = 3;            // K K^T staged (3 warps arrive) -> P warps (3 warps wait)
constexpr int BAR_GATES = 4;         // the two gate warps
constexpr int kKKThreads = 192;

// TMEM columns (fp32, 128 lanes)
constexpr uint32_t TM_G = 0;     // Gram of even chunks (lanes 0-63 K K^T, 64-127 Q K^T), then W^T
constexpr uint32_t TM_G1 = 320;  // the same for odd chunks
constexpr uint32_t TM_X = 64;    // X^T (lane = value index i, column = token r), fp32
constexpr uint32_t TM_XH = 128;  // (X diag(e^{g_L - g}))^T as bf16 hi (32 columns) and lo (32)
constexpr uint32_t TM_O = 192;   // O^T accumulator
constexpr uint32_t TM_SB = 256;  // bf16 copy of S, two per column (MMA A operand)
constexpr uint32_t TM_S = 384;   // fp32 state master (lane i, column j)
constexpr uint32_t TM_COLS = 512;

// Shared memory (bytes from a 1024-aligned base).
constexpr int kKQStages = 3;          // q/k tiles in flight: chunk c in stage c % 3
constexpr uint32_t SM_KQ0 = 0;        // [K;Q] stages: 2 K-atoms x 128 rows x 128 B (bf16) each
constexpr uint32_t KQ_STAGE = 32768;
constexpr uint32_t SM_V = 98304;      // V: 2 dv-atoms x 64 tokens x 128 B; once the W / U~ MMAs
                                      // have read it, -W bf16, MN-major: 128 rows (j) x 64 tokens
constexpr uint32_t SM_W = 114688;     // out tile staging (two 64-wide boxes)
constexpr uint32_t SM_P0 = 131072;    // P fp32, K-major: 2 atoms (32 s) x 64 rows; even chunks
constexpr uint32_t SM_P1 = 147456;    // odd chunks (K K^T is staged here first, P formed in place)
constexpr uint32_t SM_F1 = 163840;    // Tc (bf16) | Eb (bf16), K-major, operands of the W / U~ MMAs
constexpr uint32_t SM_F2 = 180224;    // fp32 16x16 blocks: -A and the diagonal blocks of Tinv
constexpr uint32_t SM_BLO = 196608;   // bf16 64x64 K-major: diag(lo(beta)), zero elsewhere
constexpr uint32_t SM_QH = 204800;    // Qh bf16, K-major like Q: 2 atoms (64 j) x 64 tokens
constexpr uint32_t SM_MISC = 221184;  // gate tables, barriers
constexpr uint32_t SM_END = SM_MISC + 8192;
constexpr uint32_t kSmemBytes = SM_END + 1024;

constexpr uint32_t KQ_ATOM = 16384;
constexpr uint32_t QH_ATOM = 8192;
constexpr uint32_t V_ATOM = 8192;
constexpr uint32_t OP_ATOM = 16384;
constexpr uint32_t F32_ATOM = 8192;   // 64 rows x 128 B

constexpr uint32_t ID_G = tc::idesc_bf16(128, 64, false, false);    // [K;Q] K^T
constexpr uint32_t ID_WN = tc::idesc_bf16(128, 64, true, false);    // K^T Tc^T, V^T Eb^T
constexpr uint32_t ID_SW = tc::idesc_bf16(128, 64, false, true);    // S (-W)^T (W MN-major)
constexpr uint32_t ID_SQ = tc::idesc_bf16(128, 64, false, false);   // S Qh^T
constexpr uint32_t ID_SK = tc::idesc_bf16(128, 128, false, true);   // X'^T K (K MN-major)
constexpr uint32_t ID_XP = tc::idesc_tf32(128, 64, false, false);   // X^T P^T

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint4 pack8_bf16(const float* v) {
    uint4 w;
    w.x = tc::pack_bf16(v[0], v[1]);
    w.y = tc::pack_bf16(v[2], v[3]);
    w.z = tc::pack_bf16(v[4], v[5]);
    w.w = tc::pack_bf16(v[6], v[7]);
    return w;
}

// ---- the inverse Tinv = (I + A)^{-1} of one chunk (prep group) ----
// Scratch F2 (fp32) is a 4 x 4 grid of 16 x 16 blocks, block (R, C) at float
// offset 256 (4 R + C).  Its lower blocks hold -A (off-diagonal blocks rounded to
// tf32, the precision of the warp MMAs that read them; diagonal blocks exact), and
// four of the unused upper slots hold the diagonal inverse blocks T_ii.  Inside a
// block, element (r, c) sits at 16 r + (c ^ bsw(r)), bsw(r) = 8 (bit 1 of r) +
// 4 (bit 2 of r): conflict-free for a row of four floats per lane (16-byte
// accesses, eight rows per phase), for the m16n8k8 A fragment (rows g, g + 8,
// columns t, t + 4), the B fragment (rows t, t + 4, column g) and accumulator pairs
// (rows g, g + 8, columns 2t, 2t + 1).
__device__ __forceinline__ int bsw(int r) { return ((r & 2) << 2) | (r & 4); }
__device__ __forceinline__ int boff(int r, int c) { return 16 * r + (c ^ bsw(r)); }
__device__ __forceinline__ int blk_off(int R, int C) { return 256 * (4 * R + C); }
__device__ __forceinline__ int td_off(int i) { return 256 * (i < 3 ? i + 1 : 6); }   // T_ii slots
__device__ __forceinline__ float tf32_round(float x) { return __uint_as_float(tc::f32_to_tf32(x)); }

// -A of row r over columns 32 ch .. 32 ch + 31 (a[], zero for s >= r) into its
// blocks of F2; an upper block of the pair is skipped.
__device__ __forceinline__ void store_neg_a(float* F2p, int r, int ch, const float (&a)[32]) {
    const int R = r >> 4, rr = r & 15;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
        const int C = 2 * ch + cb;
        if (C > R) continue;
        float* row = F2p + blk_off(R, C) + 16 * rr;
        const bool off = (C < R);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float x = -a[16 * cb + 4 * c4 + e];
                v[e] = off ? tf32_round(x) : x;
            }
            *reinterpret_cast<float4*>(row + ((4 * c4) ^ bsw(rr))) = make_float4(v[0], v[1], v[2], v[3]);
        }
    }
}

// Diagonal block T_bb = (I + A_bb)^{-1}, column j of it per lane (16 lanes per
// block): x_r = [r = j] + sum_{s<r} (-A)_rs x_s for r = 0 .. 15 (left-looking
// substitution; row r of -A_bb read as 16-byte broadcasts), into the T_bb slot.
// Entries above the diagonal come out exactly zero.
__device__ __forceinline__ void diag_block_inverse(float* F2p, int b, int j) {
    const float* Ab = F2p + blk_off(b, b);
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int c4 = 0; 4 * c4 < r; ++c4) {
            const float4 v = *reinterpret_cast<const float4*>(Ab + 16 * r + ((4 * c4) ^ bsw(r)));
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (4 * c4 + e < r) acc = fmaf(vv[e], x[4 * c4 + e], acc);
        }
        x[r] = acc;
    }
    float* Tb = F2p + td_off(b);
#pragma unroll
    for (int r = 0; r < 16; ++r) Tb[boff(r, j)] = x[r];
}

// A 16 x 8 accumulator tile C (c0 = C[g][2t], c1 = C[g][2t+1], c2 = C[g+8][2t],
// c3 = C[g+8][2t+1]) as the B operand of a K = 16 product: tf32 b = {C[t][g],
// C[t+4][g], C[8+t][g], C[12+t][g]} (two m16n8k8 steps), by shuffles.
__device__ __forceinline__ void acc_to_bfrag(const float (&c)[4], uint32_t (&b)[4], int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int s0 = 4 * t + (g >> 1), s1 = s0 + 16;
    const bool odd = (g & 1) != 0;
    const float v00 = __shfl_sync(0xffffffffu, c[0], s0), v01 = __shfl_sync(0xffffffffu, c[1], s0);
    const float v10 = __shfl_sync(0xffffffffu, c[0], s1), v11 = __shfl_sync(0xffffffffu, c[1], s1);
    const float v20 = __shfl_sync(0xffffffffu, c[2], s0), v21 = __shfl_sync(0xffffffffu, c[3], s0);
    const float v30 = __shfl_sync(0xffffffffu, c[2], s1), v31 = __shfl_sync(0xffffffffu, c[3], s1);
    b[0] = tc::f32_to_tf32(odd ? v01 : v00);
    b[1] = tc::f32_to_tf32(odd ? v11 : v10);
    b[2] = tc::f32_to_tf32(odd ? v21 : v20);
    b[3] = tc::f32_to_tf32(odd ? v31 : v30);
}

// One strip w (columns 8 w .. 8 w + 7, inside block column j = w / 2) of Tinv by
// block forward substitution down the strip, from (I + A) Tinv = I:
//   T_j = the strip of T_jj,   T_i = T_ii (-A_ij T_j - ... - A_i,i-1 T_i-1)  (i > j),
// each product on m16n8k8 tf32 warp MMAs (the strip's blocks so far kept as B
// fragments).  Writes the strip's 64 rows of Tc = Tinv diag(c) and
// Eb = Tinv diag(beta) (bf16, K-major 128B-swizzled at F1 and F1 + 8192), zero
// above block row j.  CS / BT: shared addresses of c and beta.
__device__ __forceinline__ void strip_inverse(const float* F2p, uint32_t F1, int w, int lane, uint32_t CS,
                                              uint32_t BT, uint32_t IK = 0) {
    const int j = w >> 1, co = 8 * (w & 1);
    const int g = lane >> 2, t = lane & 3;
    const int oa0 = boff(g, t), oa1 = boff(g, t + 4), oa2 = boff(g, 8 + t), oa3 = boff(g, 12 + t);
    const int ob0 = boff(t, co + g), ob1 = boff(t + 4, co + g);
    const int s0 = 8 * w + 2 * t;
    float c0 = tc::lds_f32(CS + 4u * s0), c1 = tc::lds_f32(CS + 4u * (s0 + 1));
    if (IK) {   // normalised k: W = Tinv diag(c / |k|) K
        c0 *= tc::lds_f32(IK + 4u * s0);
        c1 *= tc::lds_f32(IK + 4u * (s0 + 1));
    }
    const float e0 = tc::lds_f32(BT + 4u * s0), e1 = tc::lds_f32(BT + 4u * (s0 + 1));
    // rows 16 i + g (+ 8) of this strip: 128B-swizzled chunk w of each row
    const uint32_t orow = F1 + (uint32_t)g * 128u + ((uint32_t)(w ^ g) << 4) + 4u * (uint32_t)t;
    auto out = [&](int i, float x0, float x1, float x2, float x3) {
        const uint32_t o = orow + 2048u * (uint32_t)i;
        tc::sts_u32(o, tc::pack_bf16(x0 * c0, x1 * c1));
        tc::sts_u32(o + 8192, tc::pack_bf16(x0 * e0, x1 * e1));
        tc::sts_u32(o + 1024, tc::pack_bf16(x2 * c0, x3 * c1));
        tc::sts_u32(o + 1024 + 8192, tc::pack_bf16(x2 * e0, x3 * e1));
    };
    const float* Tj = F2p + td_off(j);
    uint32_t tb[3][4];
    {
        const float2 u = *reinterpret_cast<const float2*>(Tj + boff(g, co + 2 * t));
        const float2 v = *reinterpret_cast<const float2*>(Tj + boff(g, co + 2 * t) + 128);
        const uint32_t q0 = tc::f32_to_tf32(Tj[ob0]), q1 = tc::f32_to_tf32(Tj[ob1]);
        const uint32_t q2 = tc::f32_to_tf32(Tj[ob0 + 128]), q3 = tc::f32_to_tf32(Tj[ob1 + 128]);
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            tb[k][0] = q0; tb[k][1] = q1; tb[k][2] = q2; tb[k][3] = q3;
        }
#pragma unroll
        for (int i = 0; i < 3; ++i)
            if (i < j) out(i, 0.f, 0.f, 0.f, 0.f);
        out(j, u.x, u.y, v.x, v.y);
    }
#pragma unroll
    for (int i = 1; i < 4; ++i) {
        if (i <= j) continue;
        float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < i; ++k) {
            if (k < j) continue;
            const float* Ab = F2p + blk_off(i, k);
            tc::mma_sync_tf32(p, __float_as_uint(Ab[oa0]), __float_as_uint(Ab[oa0 + 128]),
                              __float_as_uint(Ab[oa1]), __float_as_uint(Ab[oa1 + 128]), tb[k][0], tb[k][1]);
            tc::mma_sync_tf32(p, __float_as_uint(Ab[oa2]), __float_as_uint(Ab[oa2 + 128]),
                              __float_as_uint(Ab[oa3]), __float_as_uint(Ab[oa3 + 128]), tb[k][2], tb[k][3]);
        }
        uint32_t pb[4];
        acc_to_bfrag(p, pb, lane);
        const float* Ti = F2p + td_off(i);
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        tc::mma_sync_tf32(x, tc::f32_to_tf32(Ti[oa0]), tc::f32_to_tf32(Ti[oa0 + 128]), tc::f32_to_tf32(Ti[oa1]),
                          tc::f32_to_tf32(Ti[oa1 + 128]), pb[0], pb[1]);
        tc::mma_sync_tf32(x, tc::f32_to_tf32(Ti[oa2]), tc::f32_to_tf32(Ti[oa2 + 128]), tc::f32_to_tf32(Ti[oa3]),
                          tc::f32_to_tf32(Ti[oa3 + 128]), pb[2], pb[3]);
        out(i, x[0], x[1], x[2], x[3]);
        if (i < 3) acc_to_bfrag(x, tb[i], lane);
    }
}

// Gram [K;Q] K^T of one chunk's q/k stage into a TMEM buffer, committed to `bar`
// (the MMA-issue warp; one out-of-line copy for its three call sites).
__device__ __noinline__ void gram_mma(uint32_t d, uint32_t kq, uint64_t* bar) {
    tc::tc_fence_after();
    tc::mma_ak_bk(d, kq, KQ_ATOM, kq, KQ_ATOM, ID_G, 8, 0);
    tc::mma_commit(bar);
}

// Exact-exponential forms for a chunk whose total log-decay is at or below -80
// (e^{-g} would leave the normal fp32 range): each entry takes exp2 of its own
// exponent difference.  Out of line, they are never on the common path.
//   a_rows_exact: A_rs = beta_r 2^{g'_{r-1} - g'_s} (K K^T)_rs (s < r) for row r over
//   columns 32 ch .. + 31, from the Gram in TMEM, stored as -A into F2's blocks
//   (g' = g log2 e)
//   (ikt: shared address of 1 / |k| per token when q and k are normalised in the
//   kernel, else 0)
template <bool kNorm>
__device__ __noinline__ void a_rows_exact(float* F2p, uint32_t gram_taddr, int r, int ch, uint32_t ts,
                                          uint32_t ikt) {
    float a[32];
    tc::tmem_ld32(gram_taddr, a);
    tc::tmem_ld_wait();
    float br = tc::lds_f32(ts + 512 + 4u * r);
    const float gpr = tc::lds_f32(ts + 256 + 4u * r);
    if constexpr (kNorm) br *= tc::lds_f32(ikt + 4u * r);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int s = 32 * ch + e;
        float v = br * exp2f(gpr - tc::lds_f32(ts + 4u * s)) * a[e];
        if constexpr (kNorm) v *= tc::lds_f32(ikt + 4u * s);
        a[e] = (s < r) ? v : 0.f;
    }
    store_neg_a(F2p, r, ch, a);
}
//   p_row_exact: P_rs = 2^{g'_r - g'_s} (Q K^T - d K K^T)_rs (s <= r) for row r over
//   columns 32 ch .. + 31, in place over the staged K K^T row
//   (ikt as above; iq: 1 / |q_r|, 1 when not normalised)
template <bool kNorm>
__device__ __noinline__ void p_row_exact(uint32_t prow, uint32_t gram_taddr, int r, int ch, float dh,
                                         uint32_t ts, uint32_t ikt, float iq) {
    float gv[32];
    tc::tmem_ld32(gram_taddr, gv);
    tc::tmem_ld_wait();
    const float gr = tc::lds_f32(ts + 4u * r);
    const float dk = kNorm ? dh * tc::lds_f32(ikt + 4u * r) : dh;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int s = 32 * ch + e;
        const uint32_t pa = prow + tc::sw128(r, e >> 2) + 4u * (e & 3);
        float v;
        if constexpr (kNorm)
            v = exp2f(gr - tc::lds_f32(ts + 4u * s)) * tc::lds_f32(ikt + 4u * s) *
                fmaf(-dk, tc::lds_f32(pa), iq * gv[e]);
        else
            v = exp2f(gr - tc::lds_f32(ts + 4u * s)) * fmaf(-dh, tc::lds_f32(pa), gv[e]);
        tc::sts_f32(pa, (s <= r) ? v : 0.f);
    }
}

__device__ __forceinline__ void fail(volatile int* gabort) {
    *gabort = 1;
    latch_status(-4 /* COMBA_ETIMEOUT */);
}

// kPacked: chains are packed variable-length sequences (cu_seqlens) whose q / k heads
// may be shared by groups of value heads.  kGated: the inputs are raw projections --
// q and k rows are L2-normalised in the kernel and log_alpha / beta hold raw gate
// projections a, b (log-decay -exp(A_log_h) softplus(a + dt_bias_h), beta sigmoid(b)).
// The plain instantiation compiles without either path.
template <bool kPacked, bool kGated>
__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const float* __restrict__ log_alpha, const float* __restrict__ beta,
                    const float* __restrict__ dvec, const float* S0, float* S_final, int T, int H,
                    int b_split, int no_out, unsigned long long timeout_ns,
                    const int* __restrict__ cu_seqlens, int qk_group, unsigned short* out_raw,
                    const float* __restrict__ A_log, const float* __restrict__ dt_bias, float norm_eps,
                    int stall) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = tc::smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sb = tc::smem_u32(sm);

    // Prep gate tables, two sets (chunk c uses set c & 1; the next chunk's set is
    // built while the current one is in use), 64 fp32 each, by shared address:
    //   +0 g_r log2(e), +256 g_{r-1} log2(e), +512 beta_r, +768 beta_r e^{g_{r-1}},
    //   +1024 e^{g_r}, +1280 e^{-g_r} (when the chunk allows), +1536 the chunk's
    //   "fast" flag (total log-decay above -80), +1792 1 / |k_r| (normalised q, k only)
    auto tset = [&](int c) -> uint32_t { return sb + SM_MISC + 2048u * (uint32_t)(c & 1); };
    const uint32_t RED = sb + SM_MISC + 4096;   // gate warps: [0..1] scan carries
    const uint32_t SRED = RED + 16;             // state group: [0..1] scan carries
    // state group, per chunk parity: e^{g_L - g_r} (SED) and e^{g_r} (SEG) of a chunk
    auto sed = [&](int c) -> uint32_t { return sb + SM_MISC + 4352u + 512u * (uint32_t)(c & 1); };
    auto seg = [&](int c) -> uint32_t { return sed(c) + 256u; };
    // gated inputs: the state group's 1 / |k_r| of a chunk (per parity), and its
    // partial row sums of squares exchanged between the two threads of a row
    auto sik = [&](int c) -> uint32_t { return sb + SM_MISC + 5376u + 256u * (uint32_t)(c & 1); };
    const uint32_t XCH = sb + SM_MISC + 7168;
    // barriers: q/k stages, v, gram per TMEM buffer, wn (W^T, U~^T in TMEM), mma1 (X),
    // mma2, the P buffers (MMA2 has read them), mma1 (O).  Each is arrived on once per
    // phase (by a commit, a TMA transaction count or one thread after its group's
    // named barrier): many arrivals on one barrier serialise in the shared-memory pipe.
    // The MMA-issue warp waits on three hand-overs: the prep group's Tc / Eb / diag(lo)
    // of a chunk (WNREADY), the state group's -W operand and S copies (WREADY) and its
    // bf16 X' (SPLIT).
    enum { B_KQ0 = 0, B_V = 3, B_GRAM0 = 4, B_GRAM1 = 5, B_WN = 6, B_MMA1 = 7, B_MMA2 = 8,
           B_PBUF0 = 9, B_PBUF1 = 10, B_MMA1B = 11, B_WNREADY = 12, B_WREADY = 13, B_SPLIT = 14,
           B_DRAIN = 15, NBARS = 16 };
    // Waits that drain in-flight copies and MMAs before the CTA exits (after a wait has
    // given up, say) get at least this long.
    const unsigned long long drain_ns = timeout_ns > 100000000ull ? timeout_ns : 100000000ull;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM_MISC + 6144);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
    volatile int* gabort = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t F1 = sb + SM_F1;
    float* F2p = reinterpret_cast<float*>(sm + SM_F2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // CTAs of batch index >= b_split solve the same chain of batch (index - b_split)
    // with V = 0 (a stacked launch that also yields each chain's state transition);
    // S0 and S_final are indexed by the CTA.  no_out: the outputs are not written.
    const int bcta = blockIdx.x / H, h = blockIdx.x % H;
    const bool vzero = bcta >= b_split;
    const int b = vzero ? bcta - b_split : bcta;
    const bool want_out = (no_out == 0);
    const float dh = dvec[h];
    // gated inputs: a token's raw gate projections become its log-decay and beta where
    // they are consumed; tokens past the end stay neutral (log-decay 0, beta 0)
    const float gA = kGated ? -__expf(A_log[h]) : 0.f;
    const float gdt = (kGated && dt_bias) ? dt_bias[h] : 0.f;
    auto to_la = [&](float raw, bool valid) -> float {
        if constexpr (kGated) {
            const float x = raw + gdt;
            return valid ? gA * (fmaxf(x, 0.f) + log1pf(__expf(-fabsf(x)))) : 0.f;
        } else {
            return raw;
        }
    };
    auto to_bt = [&](float raw, bool valid) -> float {
        if constexpr (kGated) return valid ? 1.f / (1.f + __expf(-raw)) : 0.f;
        else return raw;
    };
    // The chain's tokens along the tensor maps' token axis (extent T): rows 0 .. T-1 of
    // batch b, or, for packed sequences (cu_seqlens), rows cu_seqlens[b] ..
    // cu_seqlens[b+1]-1 of the single batch.  Its q / k head is h / qk_group.
    int tok0 = 0, Tc = T, bm = b;
    if constexpr (kPacked) {
        const int s0 = cu_seqlens[b], s1 = cu_seqlens[b + 1];
        bm = 0;
        if (s0 < 0 || s1 < s0 || s1 > T) {   // malformed bounds: the sequence is skipped
            if (tid == 0) latch_status(-1 /* COMBA_EINVAL */);
            Tc = 0;
        } else {
            tok0 = s0;
            Tc = s1 - s0;
        }
    }
    const int hq = kPacked ? h / qk_group : h;
    // a packed sequence's ragged last tile is written with plain stores (a TMA store
    // would write into the next sequence's rows)
    const bool clip_tail = kPacked && (Tc % kC != 0);
    const int nchunks = (Tc + kC - 1) / kC;
    const uint32_t trow = (uint32_t)((warp & 3) * 32) << 16;

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i)
            tc::mbar_init(&bars[i], 1);
        *gabort = 0;
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

    auto kq_stage = [&](int n) -> uint32_t { return SM_KQ0 + KQ_STAGE * (uint32_t)(n % kKQStages); };
    auto kq_bar = [&](int n) -> uint64_t* { return &bars[B_KQ0 + n % kKQStages]; };
    auto kq_par = [&](int n) -> uint32_t { return (uint32_t)(n / kKQStages) & 1u; };
    auto load_kq = [&](int n) {
        uint8_t* dst = sm + kq_stage(n);
        uint64_t* bar = kq_bar(n);
        tc::mbar_arrive_expect_tx(bar, 32768);
        const int t0 = tok0 + n * kC;
        tc::tma_load_4d(dst, &tm_k, bar, 0, hq, t0, bm);
        tc::tma_load_4d(dst + 8192, &tm_q, bar, 0, hq, t0, bm);
        tc::tma_load_4d(dst + KQ_ATOM, &tm_k, bar, 64, hq, t0, bm);
        tc::tma_load_4d(dst + KQ_ATOM + 8192, &tm_q, bar, 64, hq, t0, bm);
    };
    auto load_v = [&](int n) {
        tc::mbar_arrive_expect_tx(&bars[B_V], 16384);
        const int t0 = tok0 + n * kC;
        tc::tma_load_4d(sm + SM_V, &tm_v, &bars[B_V], 0, h, t0, bm);
        tc::tma_load_4d(sm + SM_V + V_ATOM, &tm_v, &bars[B_V], 64, h, t0, bm);
    };
    // One token's gate value.  The load is issued where it is written (volatile) and
    // consumed a phase later, so its latency stays hidden; a plain load may be sunk
    // by the compiler to its use, past the waits in between.
    auto gate = [&](const float* p, int t) -> float {
        float v = 0.f;
        if (t < Tc) {
            const float* a = p + ((size_t)bm * T + tok0 + t) * H + h;
            asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(a));
        }
        return v;
    };

    if (kPacked && nchunks == 0) {
        // an empty chain (a zero-length packed sequence): S_final = S0 (or zero)
        if (warp < 4 && S_final) {
            const size_t ro = ((size_t)blockIdx.x * kD + tid) * kD;
            for (int e = 0; e < kD; e += 4)
                *reinterpret_cast<float4*>(S_final + ro + e) =
                    S0 ? *reinterpret_cast<const float4*>(S0 + ro + e) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    } else if (warp < 4) {
        // =============================== state group ===============================
        // Per chunk n: the -W operand from W^T (TMEM, the prep group's MMA) into the V
        // buffer; MMA1(n) X^T += S (-W)^T, O^T = S Qh^T; X' = X diag(e^{g_L - g}) as bf16
        // hi + lo; MMA2(n) S += X'^T K, O^T += X^T P^T; then S -> bf16 copy,
        // S *= e^{g_L(n+1)}, O^T -> out (staged, TMA store), and the Qh operand of
        // chunk n+1 from the group's own scan of its log-decays.
        const int row = tid;
        const bool issuer = (tid == 0);
        // Scan of chunk c's log-decays held by threads 0..63: writes e^{g_L - g_r} to
        // sed(c) and e^{g_r} to seg(c), and returns e^{g_L} to every thread of the group.
        auto state_gates = [&](float la, int c) -> float {
            float x = (tid < 64) ? to_la(la, c * kC + tid < Tc) : 0.f;
            if (tid < 64) {
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, off);
                    if (lane >= off) x += y;
                }
                if (lane == 31) tc::sts_f32(SRED + 4u * warp, x);
            }
            tc::named_barrier(BAR_STATE, kStateThreads);
            const float c0 = tc::lds_f32(SRED), gL = c0 + tc::lds_f32(SRED + 4u);
            if (tid < 64) {
                const float g = x + (tid >= 32 ? c0 : 0.f);
                tc::sts_f32(sed(c) + 4u * tid, __expf(gL - g));
                tc::sts_f32(seg(c) + 4u * tid, __expf(g));
            }
            return __expf(gL);
        };
        // Qh = diag(e^g)(Q - d K) of chunk c (bf16, K-major like Q), from its q/k tiles.
        auto state_qh = [&](int c) -> bool {
            const bool okc = tc::mbar_wait(kq_bar(c), kq_par(c), timeout_ns);
            const uint32_t kqc = sb + kq_stage(c);
            const int r = tid & 63, jh = tid >> 6;
            const float egr = tc::lds_f32(seg(c) + 4u * r);
            float fq = egr, fk = egr * dh;   // Qh row = fq q - fk k
            if constexpr (kGated) {
                // gated inputs: |q_r|, |k_r| from this thread's half-rows and the partner
                // thread's (64 + r or r - 64) partial sums; 1 / |k_r| kept for the state update
                float sk = 0.f, sq = 0.f;
#pragma unroll 2
                for (int c8 = 0; c8 < 8; ++c8) {
                    const uint32_t off = kqc + jh * KQ_ATOM + tc::sw128(r, c8);
                    const uint4 kw = tc::lds_u32x4(off), qw = tc::lds_u32x4(off + 8192);
                    const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kw);
                    const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qw);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 kf = __bfloat1622float2(k2[e]), qf = __bfloat1622float2(q2[e]);
                        sk = fmaf(kf.x, kf.x, fmaf(kf.y, kf.y, sk));
                        sq = fmaf(qf.x, qf.x, fmaf(qf.y, qf.y, sq));
                    }
                }
                tc::sts_f32(XCH + 8u * (64u * jh + r), sk);
                tc::sts_f32(XCH + 8u * (64u * jh + r) + 4u, sq);
                tc::named_barrier(BAR_STATE, kStateThreads);
                sk += tc::lds_f32(XCH + 8u * (64u * (1 - jh) + r));
                sq += tc::lds_f32(XCH + 8u * (64u * (1 - jh) + r) + 4u);
                const float ik = rsqrtf(sk + norm_eps), iq = rsqrtf(sq + norm_eps);
                if (jh == 0) tc::sts_f32(sik(c) + 4u * r, ik);
                fq = egr * iq;
                fk = egr * dh * ik;
            }
#pragma unroll 2
            for (int c8 = 0; c8 < 8; ++c8) {
                const uint32_t off = kqc + jh * KQ_ATOM + tc::sw128(r, c8);
                const uint4 kw = tc::lds_u32x4(off);
                uint4 qw = tc::lds_u32x4(off + 8192);
                const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kw);
                __nv_bfloat162* q2 = reinterpret_cast<__nv_bfloat162*>(&qw);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kf = __bfloat1622float2(k2[e]);
                    const float2 qf = __bfloat1622float2(q2[e]);
                    if constexpr (kGated)
                        q2[e] = __floats2bfloat162_rn(fmaf(-fk, kf.x, fq * qf.x), fmaf(-fk, kf.y, fq * qf.y));
                    else
                        q2[e] = __floats2bfloat162_rn(egr * fmaf(-dh, kf.x, qf.x), egr * fmaf(-dh, kf.y, qf.y));
                }
                tc::sts_u32x4(sb + SM_QH + jh * QH_ATOM + tc::sw128(r, c8), qw);
            }
            tc::fence_proxy_async_smem();
            return okc;
        };
        bool ok = true;
        // the last q/k and V chunks loaded into this CTA's shared memory (the prep group
        // issues chunks 0 .. 2 and V of chunk 0 first)
        int kq_last = (nchunks < kKQStages ? nchunks : kKQStages) - 1;
        int v_last = vzero ? -1 : 0;
        // decays and Qh of chunk 0, initial state
        {
            const float la0 = (tid < 64) ? gate(log_alpha, tid) : 0.f;
            const float eL0 = state_gates(la0, 0);
            tc::named_barrier(BAR_STATE, kStateThreads);
            ok = state_qh(0) && ok;
            const float* s0row = S0 ? S0 + ((size_t)blockIdx.x * kD + row) * kD : nullptr;
#pragma unroll 1
            for (int pair = 0; pair < 2; ++pair) {
                float v0[32], v1[32], pk[32];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 a4 = s0row ? *reinterpret_cast<const float4*>(s0row + 64 * pair + e)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4 b4 = s0row ? *reinterpret_cast<const float4*>(s0row + 64 * pair + 32 + e)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
                    v0[e] = a4.x; v0[e + 1] = a4.y; v0[e + 2] = a4.z; v0[e + 3] = a4.w;
                    v1[e] = b4.x; v1[e + 1] = b4.y; v1[e + 2] = b4.z; v1[e + 3] = b4.w;
                }
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    pk[c] = __uint_as_float(tc::pack_bf16(v0[2 * c], v0[2 * c + 1]));
                    pk[16 + c] = __uint_as_float(tc::pack_bf16(v1[2 * c], v1[2 * c + 1]));
                }
                tc::tmem_st32(tl + TM_SB + 32 * pair, pk);
#pragma unroll
                for (int e = 0; e < 32; ++e) { v0[e] *= eL0; v1[e] *= eL0; }
                tc::tmem_st32(tl + TM_S + 64 * pair, v0);
                tc::tmem_st32(tl + TM_S + 64 * pair + 32, v1);
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            if (!ok) fail(gabort);
            ok = tc::named_barrier_all_ok(BAR_STATE, kStateThreads, ok);
        }
        // next chunk's log-decay (threads 0..63), loaded a chunk ahead of its scan
        float la_n = (tid < 64 && nchunks > 1) ? gate(log_alpha, kC + tid) : 0.f;
        for (int n = 0; n < nchunks && ok; ++n) {
            const int t0 = n * kC;
            const int stg = n & 1;
            const uint32_t tgn = stg ? TM_G1 : TM_G;
            const bool last = (n + 1 == nchunks);
            // ---- -W operand from W^T (lane = j, column = token) once the prep's MMAs are
            // done, into the V buffer (those MMAs have read V)
            ok = (*gabort == 0) && tc::mbar_wait(&bars[B_WN], n & 1, timeout_ns);
            tc::named_barrier(BAR_STATE, kStateThreads);
            tc::tc_fence_after();
            {
                float w0[32], w1[32];
                tc::tmem_ld32(tl + tgn, w0);
                tc::tmem_ld32(tl + tgn + 32, w1);
                tc::tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) { w0[e] = -w0[e]; w1[e] = -w1[e]; }
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    tc::sts_u32x4(sb + SM_V + tc::sw128(row, c4), pack8_bf16(w0 + c4 * 8));
                    tc::sts_u32x4(sb + SM_V + tc::sw128(row, 4 + c4), pack8_bf16(w1 + c4 * 8));
                }
            }
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            if (!ok) fail(gabort);
            if (!tc::named_barrier_all_ok(BAR_STATE, kStateThreads, ok && *gabort == 0)) break;
            if (issuer) tc::mbar_arrive(&bars[B_WREADY]);  // -W and the S copies are in: MMA1
            __syncwarp();
            // ---- while MMA1 runs: the next chunk's decays
            const float eLn = last ? 1.f : state_gates(la_n, n + 1);
            if (tid < 64 && n + 2 < nchunks) la_n = gate(log_alpha, t0 + 2 * kC + tid);
            // ---- X' = X diag(e^{g_L - g}) as bf16 hi + lo (operand of the state update)
            ok = ok && tc::mbar_wait(&bars[B_MMA1], n & 1, timeout_ns);
            tc::tc_fence_after();
            if (issuer && ok && n + 1 < nchunks && !vzero) {   // MMA1 has read -W
                load_v(n + 1);
                v_last = n + 1;
            }
            const uint32_t sedn = sed(n);
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float xv[32], hv[16], lv[16];
                tc::tmem_ld32(tl + TM_X + 32 * half, xv);
                tc::tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float4 d4 = tc::lds_f32x4(sedn + 4u * (32 * half + 4 * c));
                    if constexpr (kGated) {   // the state update reads the normalised k: X' columns / |k_s|
                        const float4 k4 = tc::lds_f32x4(sik(n) + 4u * (32 * half + 4 * c));
                        d4.x *= k4.x; d4.y *= k4.y; d4.z *= k4.z; d4.w *= k4.w;
                    }
                    const float a0 = xv[4 * c] * d4.x, a1 = xv[4 * c + 1] * d4.y;
                    const float a2 = xv[4 * c + 2] * d4.z, a3 = xv[4 * c + 3] * d4.w;
                    const uint32_t h01 = tc::pack_bf16(a0, a1), h23 = tc::pack_bf16(a2, a3);
                    hv[2 * c] = __uint_as_float(h01);
                    hv[2 * c + 1] = __uint_as_float(h23);
                    lv[2 * c] = __uint_as_float(tc::pack_bf16(a0 - __uint_as_float(h01 << 16),
                                                              a1 - __uint_as_float(h01 & 0xffff0000u)));
                    lv[2 * c + 1] = __uint_as_float(tc::pack_bf16(a2 - __uint_as_float(h23 << 16),
                                                                  a3 - __uint_as_float(h23 & 0xffff0000u)));
                }
                tc::tmem_st16(tl + TM_XH + 16 * half, hv);
                tc::tmem_st16(tl + TM_XH + 32 + 16 * half, lv);
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            if (!ok) fail(gabort);
            if (!tc::named_barrier_all_ok(BAR_STATE, kStateThreads, ok && *gabort == 0)) break;
            if (issuer) tc::mbar_arrive(&bars[B_SPLIT]);   // X' is in: MMA2
            __syncwarp();
            // ---- while MMA2 runs: Qh of the next chunk (MMA1 has read this chunk's)
            if (!last && want_out) {
                ok = ok && tc::mbar_wait(&bars[B_MMA1B], n & 1, timeout_ns);
                ok = state_qh(n + 1) && ok;
            }
            ok = ok && tc::mbar_wait(&bars[B_MMA2], n & 1, timeout_ns);
            if (issuer) tc::bulk_wait_read0();   // the previous out store has read its staging
            if (!ok) fail(gabort);
            if (!tc::named_barrier_all_ok(BAR_STATE, kStateThreads, ok && *gabort == 0)) break;
            tc::tc_fence_after();
            if (issuer && n + kKQStages < nchunks) {   // this chunk's q/k stage is read
                tc::fence_proxy_async_smem();
                load_kq(n + kKQStages);
                kq_last = n + kKQStages;
            }
            __syncwarp();
            // O^T row (value index) -> bf16 pairs of tokens
            uint32_t ob[32];
            if (want_out) {
                float o0[32], o1[32];
                tc::tmem_ld32(tl + TM_O, o0);
                tc::tmem_ld32(tl + TM_O + 32, o1);
                tc::tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    ob[c] = tc::pack_bf16(o0[2 * c], o0[2 * c + 1]);
                    ob[16 + c] = tc::pack_bf16(o1[2 * c], o1[2 * c + 1]);
                }
            }
            float* sfrow = (last && S_final) ? S_final + ((size_t)blockIdx.x * kD + row) * kD : nullptr;
#pragma unroll 1
            for (int pair = 0; pair < 2; ++pair) {
                float v0[32], v1[32];
                tc::tmem_ld32(tl + TM_S + 64 * pair, v0);
                tc::tmem_ld32(tl + TM_S + 64 * pair + 32, v1);
                tc::tmem_ld_wait();
                float pk[32];
                if (sfrow) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        *reinterpret_cast<float4*>(sfrow + 64 * pair + e) =
                            make_float4(v0[e], v0[e + 1], v0[e + 2], v0[e + 3]);
                        *reinterpret_cast<float4*>(sfrow + 64 * pair + 32 + e) =
                            make_float4(v1[e], v1[e + 1], v1[e + 2], v1[e + 3]);
                    }
                } else if (!last) {
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        pk[c] = __uint_as_float(tc::pack_bf16(v0[2 * c], v0[2 * c + 1]));
                        pk[16 + c] = __uint_as_float(tc::pack_bf16(v1[2 * c], v1[2 * c + 1]));
                    }
                    tc::tmem_st32(tl + TM_SB + 32 * pair, pk);
#pragma unroll
                    for (int e = 0; e < 32; ++e) { v0[e] *= eLn; v1[e] *= eLn; }
                    tc::tmem_st32(tl + TM_S + 64 * pair, v0);
                    tc::tmem_st32(tl + TM_S + 64 * pair + 32, v1);
                }
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            if (want_out) {
            // out tile [token][value index] in two 64-wide 128B-swizzled boxes, staged in
            // its own buffer, TMA store; a packed sequence's ragged last tile is copied
            // out row by row instead.  The barrier below also hands the new S copies to
            // the next MMA1.
            {
                const uint32_t ot = sb + SM_W + (row >> 6) * 8192 + (row & 7) * 2;
                const int oc = (row & 63) >> 3;
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    tc::sts_u16(ot + tc::sw128(2 * c, oc), (unsigned short)(ob[c] & 0xffffu));
                    tc::sts_u16(ot + tc::sw128(2 * c + 1, oc), (unsigned short)(ob[c] >> 16));
                }
            }
            tc::fence_proxy_async_smem();
            tc::named_barrier(BAR_STATE, kStateThreads);
            if (clip_tail && last) {
                const int rows = Tc - t0;   // 16-byte pieces: value indices 8c .. 8c+7 of row r
                for (int e = row; e < rows * 16; e += kStateThreads) {
                    const int r = e >> 4, c = e & 15;
                    const uint4 w = tc::lds_u32x4(sb + SM_W + (c >> 3) * 8192 + tc::sw128(r, c & 7));
                    *reinterpret_cast<uint4*>(out_raw + (((size_t)bm * T + tok0 + t0 + r) * H + h) * kD + 8 * c) = w;
                }
            } else if (issuer) {
                tc::tma_store_4d(&tm_o, sm + SM_W, 0, h, tok0 + t0, bm);
                tc::tma_store_4d(&tm_o, sm + SM_W + 8192, 64, h, tok0 + t0, bm);
                tc::bulk_commit();
            }
            }
        }
        if (issuer) {
            tc::bulk_wait0();
            // every q/k and V copy issued into this CTA's shared memory (the prep group's
            // first ones included) has landed before the CTA exits, also after a wait gave up
            for (int c = kq_last - kKQStages + 1; c <= kq_last; ++c)
                if (c >= 0) tc::mbar_wait(kq_bar(c), kq_par(c), drain_ns);
            if (v_last >= 0) tc::mbar_wait(&bars[B_V], v_last & 1, drain_ns);
        }
    } else if (warp == kCtlWarp) {
        // ============================ MMA-issue warp ===============================
        // All tensor-core MMAs.  Per chunk n: MMA1(n) (once the state group hands over
        // -W and the S copies), then O^T += X^T P^T (needs only X^T and P, so it runs
        // while the state group splits X'), then the state update (once it hands over
        // X').  Then W^T / U~^T of chunk n+1 (once the prep group hands over Tc / Eb)
        // and the Gram of chunk n+2 (into the TMEM buffer whose W^T the state group
        // has read), W^T / U~^T first unless the prep group is not done with chunk
        // n+1 yet.  The tensor pipe runs MMAs in issue order; every wait depends only
        // on MMAs issued before it, so no order of these can deadlock.
        bool ok = true;
        // waits are made warp-uniform before any issue (the issuing helpers use the full mask)
        auto issue_gram = [&](int c) -> bool {
            const bool okg = __all_sync(0xffffffffu, tc::mbar_wait(kq_bar(c), kq_par(c), timeout_ns)) != 0;
            if (okg)
                gram_mma(tmem + ((c & 1) ? TM_G1 : TM_G), sb + kq_stage(c), &bars[(c & 1) ? B_GRAM1 : B_GRAM0]);
            return okg;
        };
        // W^T = K^T Tc^T;  X^T = U~^T = V^T Eb^T + V^T diag(lo)^T  of chunk c (X^T of chunk
        // c-1 read by its O MMA, committed with its P buffer)
        auto issue_wn = [&](int c) -> bool {
            bool okw = tc::mbar_wait(&bars[B_WNREADY], c & 1, timeout_ns) &&
                             (vzero || tc::mbar_wait(&bars[B_V], c & 1, timeout_ns)) &&
                             (c == 0 || tc::mbar_wait(&bars[((c - 1) & 1) ? B_PBUF1 : B_PBUF0],
                                                      ((c - 1) >> 1) & 1, timeout_ns));
            okw = __all_sync(0xffffffffu, okw) != 0;
            if (okw) {
                tc::tc_fence_after();
                const uint32_t kqc = sb + kq_stage(c);
                tc::mma_amn_bk(tmem + ((c & 1) ? TM_G1 : TM_G), kqc, KQ_ATOM, F1, ID_WN, 4, 0);
                if (!vzero) {
                    tc::mma_amn_bk(tmem + TM_X, sb + SM_V, V_ATOM, F1 + 8192, ID_WN, 4, 0);
                    tc::mma_amn_bk(tmem + TM_X, sb + SM_V, V_ATOM, sb + SM_BLO, ID_WN, 4, 1);
                }
                tc::mma_commit(&bars[B_WN]);
            }
            return okw;
        };
        ok = issue_gram(0) && (nchunks < 2 || issue_gram(1)) && issue_wn(0);
        // stall: a wait on a phase that nothing completes before the drain below (the
        // failure-path test), so it runs out after timeout_ns
        if (ok && stall) ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars[B_DRAIN], 0, timeout_ns)) != 0;
        for (int n = 0; n < nchunks && ok; ++n) {
            const int stg = n & 1;
            const uint32_t kqn = sb + kq_stage(n);
            // ---- MMA1(n): X^T += S (-W)^T;  O^T = S Qh^T;  then O^T += X^T P^T
            ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars[B_WREADY], n & 1, timeout_ns)) != 0;
            if (!ok) break;
            tc::tc_fence_after();
            tc::mma_bf16_ta_bmn(tmem + TM_X, tmem + TM_SB, sb + SM_V, 8192, ID_SW, 8, vzero ? 0u : 1u);
            tc::mma_commit(&bars[B_MMA1]);
            if (want_out) tc::mma_bf16_ta_bk(tmem + TM_O, tmem + TM_SB, sb + SM_QH, QH_ATOM, ID_SQ, 8, 0);
            tc::mma_commit(&bars[B_MMA1B]);
            if (want_out) tc::mma_tf32_ta_bk(tmem + TM_O, tmem + TM_X, sb + (stg ? SM_P1 : SM_P0), F32_ATOM, ID_XP, 8, 1);
            tc::mma_commit(&bars[stg ? B_PBUF1 : B_PBUF0]);
            // ---- MMA2(n): S += X'^T K (bf16 hi + lo)
            ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars[B_SPLIT], n & 1, timeout_ns)) != 0;
            if (!ok) break;
            tc::tc_fence_after();
            tc::mma_bf16_ta_bmn(tmem + TM_S, tmem + TM_XH, kqn, KQ_ATOM, ID_SK, 4, 1);
            tc::mma_bf16_ta_bmn(tmem + TM_S, tmem + TM_XH + 32, kqn, KQ_ATOM, ID_SK, 4, 1);
            tc::mma_commit(&bars[B_MMA2]);
            // ---- W^T / U~^T of chunk n+1 and the Gram of chunk n+2
            bool need_wn = n + 1 < nchunks, need_gram = n + 2 < nchunks;
            if (need_wn && need_gram &&
                !__all_sync(0xffffffffu, tc::mbar_test(&bars[B_WNREADY], (n + 1) & 1) &&
                                         (vzero || tc::mbar_test(&bars[B_V], (n + 1) & 1)))) {
                ok = issue_gram(n + 2);
                need_gram = false;
            }
            if (ok && need_wn) ok = issue_wn(n + 1);
            if (ok && need_gram) ok = issue_gram(n + 2);
        }
        if (!ok) fail(gabort);
        // every MMA issued has completed before the CTA releases TMEM and exits
        __syncwarp();
        tc::mma_commit(&bars[B_DRAIN]);
        tc::mbar_wait(&bars[B_DRAIN], 0, drain_ns);
        __syncwarp();
    } else {
        // =============================== prep group ================================
        // Chunk m's operands for the MMA warp: the inverse's blocks, Tc / Eb, P and
        // diag(lo(beta)).  Seven warps; warp pw reads TMEM lanes 32 (warp & 3) .. + 31 of
        // the Gram (K K^T in lanes 0-63, Q K^T in lanes 64-127):
        //   pw 3, 0, 4: K K^T rows 0-31 x cols 0-31, rows 32-63 x cols 0-31, rows 32-63 x
        //               cols 32-63: K K^T staged for P, -A into F2; pw 3 and 4 then
        //               invert the diagonal blocks (0, 1) and (2, 3) of their rows
        //   pw 1, 2, 6: Q K^T of the same row/column blocks: P, once K K^T is staged
        //   pw 5:       P rows 0-31 x cols 32-63 are zero (s > r)
        //   pw 5, 0:    the next chunk's gate tables (tokens 0-31, 32-63)
        // then one 8-column strip of Tinv per warp (pw 4: strips 6 and 7), written out
        // as Tc / Eb, and diag(lo(beta)) (pw 4, 5).
        const int pt = tid - kPrepBase;
        const int pw = pt >> 5, q = warp & 3;
        const bool kk_warp = (pw == 0 || pw == 3 || pw == 4);
        const bool p_warp = (pw == 1 || pw == 2 || pw == 6);
        const int ch = (pw == 4 || pw == 6) ? 1 : 0;        // Gram column half
        const bool gate_warp = (pw == 5 || pw == 0);
        const bool issuer = (pt == 0);
        const int gtok = (pw == 5) ? lane : 32 + lane;     // gate warps: token of this thread
        float la_x = 0.f, bt_x = 0.f;                       // gate warps: next chunk's values
        // gate tables of chunk c into tset(c) from this thread's token values (gate warps)
        auto make_tables = [&](int c, float la, float bt) {
            la = to_la(la, c * kC + gtok < Tc);
            bt = to_bt(bt, c * kC + gtok < Tc);
            float x = la;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            if (lane == 31) tc::sts_f32(RED + (pw == 5 ? 0u : 4u), x);
            __syncwarp();
            tc::named_barrier(BAR_GATES, 64);
            const float c0 = tc::lds_f32(RED), gL = c0 + tc::lds_f32(RED + 4u);
            const bool fst = gL > -80.f;
            const float g = x + (pw == 0 ? c0 : 0.f), gp = g - la;
            const uint32_t ts = tset(c);
            tc::sts_f32(ts + 4u * gtok, g * kLog2e);
            tc::sts_f32(ts + 256 + 4u * gtok, gp * kLog2e);
            tc::sts_f32(ts + 512 + 4u * gtok, bt);
            tc::sts_f32(ts + 768 + 4u * gtok, bt * __expf(gp));
            tc::sts_f32(ts + 1024 + 4u * gtok, __expf(g));
            tc::sts_f32(ts + 1280 + 4u * gtok, fst ? __expf(-g) : 0.f);
            if (gtok == 0) asm volatile("st.shared.u32 [%0], %1;" ::"r"(ts + 1536), "r"(fst ? 1u : 0u) : "memory");
            __syncwarp();
            tc::named_barrier(BAR_GATES, 64);   // RED is reused by the next call
        };
        bool ok = true;
        if (issuer) {
            for (int c = 0; c < kKQStages && c < nchunks; ++c) load_kq(c);
            if (!vzero) load_v(0);
        }
        __syncwarp();
        if (gate_warp) {
            make_tables(0, gate(log_alpha, gtok), gate(beta, gtok));
            if (nchunks > 1) {
                la_x = gate(log_alpha, kC + gtok);
                bt_x = gate(beta, kC + gtok);
            }
        }
        ok = tc::named_barrier_all_ok(BAR_PREP, kPrepThreads, ok);
        for (int m = 0; m < nchunks && ok; ++m) {
            const bool last = (m + 1 == nchunks);
            const uint32_t ts = tset(m);
            const uint32_t tgm = (m & 1) ? TM_G1 : TM_G;
            const uint32_t pbm = sb + ((m & 1) ? SM_P1 : SM_P0);
            const bool fast = tc::lds_u32(ts + 1536) != 0u;
            ok = (*gabort == 0);
            // ================= phase 1: A, K K^T, P, diagonal inverse blocks =================
            if (kk_warp) {
                const int r = 32 * q + lane;          // row (token) of this thread
                ok = ok && tc::mbar_wait(&bars[(m & 1) ? B_GRAM1 : B_GRAM0], (m >> 1) & 1, timeout_ns) &&
                     (m < 2 || tc::mbar_wait(&bars[(m & 1) ? B_PBUF1 : B_PBUF0], ((m - 2) >> 1) & 1, timeout_ns));
                __syncwarp();
                tc::tc_fence_after();
                float a[32];
                tc::tmem_ld32(tl + tgm + 32 * ch, a);
                tc::tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    tc::sts_f32x4(pbm + ch * F32_ATOM + tc::sw128(r, c),
                                  make_float4(a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]));
                if constexpr (kGated) {
                    // normalised q, k: 1 / |k_r| from the Gram's diagonal (pw 3: rows 0-31,
                    // pw 4: rows 32-63) for the whole prep group; pw 0 reads it after them
                    if (pw != 0) {
                        float dg = 0.f;
#pragma unroll
                        for (int e = 0; e < 32; ++e) dg = (e == lane) ? a[e] : dg;
                        tc::sts_f32(ts + 1792 + 4u * r, rsqrtf(dg + norm_eps));
                    }
                    tc::tc_fence_before();
                    if (pw != 0) tc::named_barrier_arrive(BAR_KK, kKKThreads);
                    else tc::named_barrier(BAR_KK, kKKThreads);
                    __syncwarp();
                } else {
                    tc::tc_fence_before();
                    tc::named_barrier_arrive(BAR_KK, kKKThreads);
                }
                // A_rs = beta_r e^{g_{r-1} - g_s} (K K^T)_rs for s < r -> -A into F2
                if (fast) {
                    float cr = tc::lds_f32(ts + 768 + 4u * r);
                    if constexpr (kGated) cr *= tc::lds_f32(ts + 1792 + 4u * r);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float4 ig = tc::lds_f32x4(ts + 1280 + 4u * (32 * ch + 4 * c));
                        if constexpr (kGated) {
                            const float4 k4 = tc::lds_f32x4(ts + 1792 + 4u * (32 * ch + 4 * c));
                            ig.x *= k4.x; ig.y *= k4.y; ig.z *= k4.z; ig.w *= k4.w;
                        }
                        const float iv[4] = {ig.x, ig.y, ig.z, ig.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            a[4 * c + e] = (32 * ch + 4 * c + e < r) ? cr * iv[e] * a[4 * c + e] : 0.f;
                    }
                    store_neg_a(F2p, r, ch, a);
                } else {
                    a_rows_exact<kGated>(F2p, tl + tgm + 32 * ch, r, ch, ts, ts + 1792);
                }
                if (pw != 0) {   // diagonal blocks 0, 1 (pw 3) and 2, 3 (pw 4) from this warp's rows
                    __syncwarp();
                    diag_block_inverse(F2p, (pw == 4 ? 2 : 0) + (lane >> 4), lane & 15);
                }
            } else if (p_warp) {
                const int r = 32 * (q - 2) + lane;    // row (token) of this thread
                ok = ok && tc::mbar_wait(&bars[(m & 1) ? B_GRAM1 : B_GRAM0], (m >> 1) & 1, timeout_ns);
                __syncwarp();
                tc::tc_fence_after();
                float gv[32];
                tc::tmem_ld32(tl + tgm + 32 * ch, gv);
                // normalised q, k: 1 / |q_r| from this chunk's q row (while the K K^T warps work)
                float iq = 1.f;
                if constexpr (kGated) {
                    const uint32_t qrow = sb + kq_stage(m) + 8192;
                    float sq = 0.f;
#pragma unroll 4
                    for (int i = 0; i < 16; ++i) {
                        const uint4 w = tc::lds_u32x4(qrow + (i >> 3) * KQ_ATOM + tc::sw128(r, i & 7));
                        const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(e2[e]);
                            sq = fmaf(f.x, f.x, fmaf(f.y, f.y, sq));
                        }
                    }
                    iq = rsqrtf(sq + norm_eps);
                }
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                tc::named_barrier(BAR_KK, kKKThreads);
                // P_rs = e^{g_r - g_s} (Q K^T - d K K^T)_rs for s <= r, in place over K K^T
                // (normalised q, k: e^{g_r - g_s} / |k_s| (Q K^T / |q_r| - d K K^T / |k_r|)_rs)
                const uint32_t prow = pbm + ch * F32_ATOM;
                if (fast) {
                    const float er = tc::lds_f32(ts + 1024 + 4u * r);
                    const float dk = kGated ? dh * tc::lds_f32(ts + 1792 + 4u * r) : dh;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t pa = prow + tc::sw128(r, c);
                        const float4 kk = tc::lds_f32x4(pa);
                        float4 ig = tc::lds_f32x4(ts + 1280 + 4u * (32 * ch + 4 * c));
                        if constexpr (kGated) {
                            const float4 k4 = tc::lds_f32x4(ts + 1792 + 4u * (32 * ch + 4 * c));
                            ig.x *= k4.x; ig.y *= k4.y; ig.z *= k4.z; ig.w *= k4.w;
                        }
                        const int s = 32 * ch + 4 * c;
                        float4 pv;
                        if constexpr (kGated) {
                            pv.x = (s + 0 <= r) ? er * ig.x * fmaf(-dk, kk.x, iq * gv[4 * c + 0]) : 0.f;
                            pv.y = (s + 1 <= r) ? er * ig.y * fmaf(-dk, kk.y, iq * gv[4 * c + 1]) : 0.f;
                            pv.z = (s + 2 <= r) ? er * ig.z * fmaf(-dk, kk.z, iq * gv[4 * c + 2]) : 0.f;
                            pv.w = (s + 3 <= r) ? er * ig.w * fmaf(-dk, kk.w, iq * gv[4 * c + 3]) : 0.f;
                        } else {
                            pv.x = (s + 0 <= r) ? er * ig.x * fmaf(-dh, kk.x, gv[4 * c + 0]) : 0.f;
                            pv.y = (s + 1 <= r) ? er * ig.y * fmaf(-dh, kk.y, gv[4 * c + 1]) : 0.f;
                            pv.z = (s + 2 <= r) ? er * ig.z * fmaf(-dh, kk.z, gv[4 * c + 2]) : 0.f;
                            pv.w = (s + 3 <= r) ? er * ig.w * fmaf(-dh, kk.w, gv[4 * c + 3]) : 0.f;
                        }
                        tc::sts_f32x4(pa, pv);
                    }
                } else {
                    p_row_exact<kGated>(prow, tl + tgm + 32 * ch, r, ch, dh, ts, ts + 1792, iq);
                }
                tc::fence_proxy_async_smem();
            } else {   // pw 5
                ok = ok && (m < 2 || tc::mbar_wait(&bars[(m & 1) ? B_PBUF1 : B_PBUF0], ((m - 2) >> 1) & 1, timeout_ns));
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    tc::sts_u32x4(pbm + F32_ATOM + tc::sw128(lane, c), make_uint4(0u, 0u, 0u, 0u));
                tc::fence_proxy_async_smem();
            }
            // ================= phase 2: next chunk's gate tables (gate warps) =================
            if (gate_warp && !last) {
                make_tables(m + 1, la_x, bt_x);
                if (m + 2 < nchunks) {
                    la_x = gate(log_alpha, (m + 2) * kC + gtok);
                    bt_x = gate(beta, (m + 2) * kC + gtok);
                }
            }
            if (!ok) fail(gabort);
            if (!tc::named_barrier_all_ok(BAR_PREP, kPrepThreads, ok && *gabort == 0)) break;
            // ================= phase 3: the inverse's strips -> Tc / Eb ==========
            // F1 and diag(lo) are free once the previous chunk's W / U~ MMAs are done
            ok = ok && (m == 0 || tc::mbar_wait(&bars[B_WN], (m - 1) & 1, timeout_ns));
            __syncwarp();
            if (__all_sync(0xffffffffu, ok)) {   // warp-uniform: the strips use full-warp shuffles and MMAs
                // the two longest strips (0, 1) on warps of schedulers 0 and 1 (warp % 4),
                // the others spread so that each scheduler carries a similar MMA load
                const int strip = (pw == 3) ? 0 : (pw == 0) ? 1 : (pw <= 2) ? pw + 1 : (pw == 4) ? 6 : pw - 1;
                strip_inverse(F2p, F1, strip, lane, ts + 768, ts + 512, kGated ? ts + 1792 : 0u);
                if (pw == 4) strip_inverse(F2p, F1, 7, lane, ts + 768, ts + 512, kGated ? ts + 1792 : 0u);
            }
            if (pt >= 128 && pt < 192) {   // diag(lo(beta))
                const int e = pt - 128;
                const float bv = tc::lds_f32(ts + 512 + 4u * e);
                const float bh = __bfloat162float(__float2bfloat16_rn(bv));
                const __nv_bfloat16 lo = __float2bfloat16_rn(bv - bh);
                tc::sts_u16(sb + SM_BLO + tc::sw128(e, e >> 3) + (e & 7) * 2,
                            *reinterpret_cast<const unsigned short*>(&lo));
            }
            tc::fence_proxy_async_smem();
            if (!ok) fail(gabort);
            if (!tc::named_barrier_all_ok(BAR_PREP, kPrepThreads, ok && *gabort == 0)) break;
            if (issuer) tc::mbar_arrive(&bars[B_WNREADY]);   // Tc, Eb, diag(lo) of chunk m are in
            __syncwarp();
        }
    }

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
    // resolved once (a function-local static is initialised once even under concurrent calls)
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return nullptr;
    }();
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

// One CTA per (b, h) of Bc stacked batches over data with B batches (Bc defaults to B):
// stacked batches b >= B repeat data batch b - B with V = 0.  out == nullptr: no
// outputs are written.  Packed sequences: cu_seqlens (device, nseq + 1 entries) cuts
// the token axis of a single batch (B = 1, T = total tokens) into nseq chains, one
// CTA per (sequence, head).  Hqk: number of q / k heads (divides H; 0 means H).
inline int launch_chunk_tc(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* d, const float* S0, void* out,
                           float* S_final, int B, int T, int H, cudaStream_t stream,
                           int Bc = -1, unsigned long long timeout_ns = kWaitTimeoutNs,
                           const int* cu_seqlens = nullptr, int nseq = 0, int Hqk = 0,
                           const float* A_log = nullptr, const float* dt_bias = nullptr,
                           float norm_eps = 0.f, bool stall = false) {
    if (Bc < 0) Bc = B;
    if (Hqk <= 0) Hqk = H;
    if (H % Hqk != 0) return -1;
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -3;
    std::unique_lock<std::mutex> lock(init_mutex());
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(tck::chunk_fwd_tc_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tck::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(tck::chunk_fwd_tc_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tck::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(tck::chunk_fwd_tc_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tck::kSmemBytes) != cudaSuccess)
            return -3;
        attr_set[dev] = true;
    }
    lock.unlock();
    CUtensorMap tq, tk, tv, to;
    if (!make_tmap_bthd(&tq, q, B, T, Hqk) || !make_tmap_bthd(&tk, k, B, T, Hqk) ||
        !make_tmap_bthd(&tv, v, B, T, H) || !make_tmap_bthd(&to, out ? out : v, B, T, H))
        return -3;
    const int chains = cu_seqlens ? nseq : Bc;
    const int b_split = cu_seqlens ? nseq : B;
    if (cu_seqlens && A_log) return -2;   // packed sequences with gated inputs: not built
    auto kern = cu_seqlens ? tck::chunk_fwd_tc_kernel<true, false>
                           : (A_log ? tck::chunk_fwd_tc_kernel<false, true> : tck::chunk_fwd_tc_kernel<false, false>);
    kern<<<(unsigned)(chains * H), tck::kThreads, tck::kSmemBytes, stream>>>(
        tq, tk, tv, to, log_alpha, beta, d, S0, S_final, T, H, b_split, out ? 0 : 1, timeout_ns,
        cu_seqlens, H / Hqk, static_cast<unsigned short*>(out), A_log, dt_bias, norm_eps, stall ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace comba
