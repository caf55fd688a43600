// Tensor-core state passes of the chunk backward (bf16 inputs, dk = dv = 128).
//
// The backward needs, for every 32-token chunk c of a chain, its start state S_c and
// the gradient dS'_c at its end state.  Both are chain recurrences over the chunks:
//   forward  S_{c+1} = e^{g_L} S_c + X_c^T diag(e^{g_L - g}) K_c,   X_c = U~_c - W_c S_c^T
//   reverse  dS_c    = e^{g_L} dS'_c - (dS'_c K_c^T diag(e^{g_L - g})) W_c + dO_c^T G_c,
//            G_c = Gamma Q~_c - P_c W_c,  dS'_{c-1} = dS_c,  dS'_{last} = dS_final, dS0 = dS_0
// (the forward's affine chunk transition and its adjoint).  They do not depend on each
// other, so one launch runs both: CTA x < chains walks chain x forwards, CTA chains + x
// walks it backwards.  A CTA keeps the chain's state as an fp32 master in TMEM (lane =
// state row i, column j) and a bf16 copy of it (the A operand of the chunk's first
// product).  Per chunk:
//   forward  X'^T = S W^T            one M=128, N=32, K=128 MMA (W: K-major tile)
//            Xd^T = (U~^T - X'^T) diag(e^{g_L - g})  as bf16 hi + lo (state group)
//            S   += Xd^T K           two M=128, N=128, K=32 MMAs (K: MN-major tile)
//   reverse  Z    = dS' K^T          one M=128, N=32, K=128 MMA
//            dS  += dO^T G           two SS MMAs (dO and G hi / lo tiles, both MN-major),
//                                    once the master has been pre-scaled
//            -Z diag(e^{g_L - g}) as bf16 hi + lo; dS += that times W (two MMAs)
// with the master pre-scaled by the chunk's e^{g_L} when the state is read out.  Each
// state read out is stored (bf16, in the piece layout of stl::off) to the workspace
// for the grads kernel.
// The prep kernel leaves every operand in the workspace in the layout the MMAs read
// (bf16 32 x 128 tiles, U~ fp32, the decays), so a chunk's inputs are one or two untiled
// bulk copies into a two-stage ring.  Warps 0-3 (the state group) own the TMEM lanes;
// warp 4 issues the copies and the MMAs.  Every wait is bounded: one that runs out
// latches COMBA_ETIMEOUT, raises the CTA's abort flag and ends the walk, and the CTA
// drains its copies and MMAs before it releases TMEM.
#pragma once

#include "chunk_bwd.cuh"

namespace comba {
namespace bwd {
namespace chain {

constexpr int kThreads = 160;        // warps 0-3: state group; warp 4: copies and MMA issue
constexpr int kD = 128;              // dk = dv
constexpr size_t kDS = (size_t)kD * kD;   // floats of one state slot of the workspace
constexpr uint32_t TM_S = 0;         // fp32 master (128 columns)
constexpr uint32_t TM_SB = 128;      // bf16 copy, two per column (64 columns)
constexpr uint32_t TM_X = 192;       // X'^T or Z (32 columns: tokens)
constexpr uint32_t TM_XH = 224;      // Xd^T or -Zd as bf16 hi (16 columns) and lo (16)
constexpr uint32_t kCols = 256;

// One ring stage (bytes).  Forward: W | K tiles, U~ (fp32 [32][128]), decays.
// Reverse: W | K tiles, G hi | G lo | dO tiles, decays.
constexpr uint32_t ST_W = 0, ST_K = 8192, ST_U = 16384, ST_G = 16384, ST_GLO = 24576, ST_DO = 32768,
                   ST_DEC = 40960, ST_BYTES = 41984;
constexpr uint32_t SM_BARS = 2 * ST_BYTES;     // 8 mbarriers, the TMEM slot, the abort flag
constexpr uint32_t kSmemBytes = SM_BARS + 128 + 1024;   // + alignment slack
enum { B_FULL0 = 0, B_FULL1 = 1, B_SREADY = 2, B_SPLIT = 3, B_MMA1 = 4, B_MMA2 = 5, B_DRAIN = 6, B_MREADY = 7 };
static_assert(ST_DEC + 256 <= ST_BYTES && ST_BYTES % 1024 == 0, "ring stage layout");
static_assert(ST_G + kPrepDec + 256 == ST_DEC + 256 && ST_DO == ST_G + 2 * tile::kBytes,
              "the reverse walk's copy of the C slot lands G hi, G lo, dO and the decays in place");
static_assert(2 * kSmemBytes <= 228 * 1024 - 2 * 1024, "two state-pass CTAs per SM");

constexpr uint32_t ID_N32 = tc::idesc_bf16(128, 32, false, false);    // S W^T, dS' K^T
constexpr uint32_t ID_N128B = tc::idesc_bf16(128, 128, false, true);  // Xd^T K, Zd W (B MN-major)
constexpr uint32_t ID_N128AB = tc::idesc_bf16(128, 128, true, true);  // dO^T G
constexpr unsigned long long kWaitNs = 2000000000ull;   // the default per-wait limit

// Reading out the state row this thread owns (lane = row i) after a chunk's update,
// in two passes so the next chunk's first MMA waits only for the first:
//  copy_out: the bf16 copy (the next first MMA's A operand), unless `last`; returns
//            the row as 64 packed bf16 pairs in `pk`
//  store_out: the row to the workspace (bf16, piece layout) and, unless `last`, the
//            master pre-scaled by `eL` for the next update; or, with `f32`, the row as
//            fp32 (dS0)
__device__ __forceinline__ void copy_out(uint32_t tl, bool last, uint32_t (&pk)[64]) {
#pragma unroll
    for (int pair = 0; pair < 2; ++pair) {
        float v0[32], v1[32];
        tc::tmem_ld32(tl + TM_S + 64 * pair, v0);
        tc::tmem_ld32(tl + TM_S + 64 * pair + 32, v1);
        tc::tmem_ld_wait();
        float p[32];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            pk[32 * pair + c] = tc::pack_bf16(v0[2 * c], v0[2 * c + 1]);
            pk[32 * pair + 16 + c] = tc::pack_bf16(v1[2 * c], v1[2 * c + 1]);
            p[c] = __uint_as_float(pk[32 * pair + c]);
            p[16 + c] = __uint_as_float(pk[32 * pair + 16 + c]);
        }
        if (!last) tc::tmem_st32(tl + TM_SB + 32 * pair, p);
    }
}
__device__ __forceinline__ void store_out(uint32_t tl, int row, bool last, float eL, const uint32_t (&pk)[64],
                                          uint8_t* slot, float* f32) {
    if (slot) {
#pragma unroll
        for (int c = 0; c < 16; ++c)
            *reinterpret_cast<uint4*>(slot + stl::off(row, c)) =
                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    }
    if (last && !f32) return;
#pragma unroll 1
    for (int pair = 0; pair < 2; ++pair) {
        float v0[32], v1[32];
        tc::tmem_ld32(tl + TM_S + 64 * pair, v0);
        tc::tmem_ld32(tl + TM_S + 64 * pair + 32, v1);
        tc::tmem_ld_wait();
        if (f32) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                *reinterpret_cast<float4*>(f32 + 64 * pair + e) = make_float4(v0[e], v0[e + 1], v0[e + 2], v0[e + 3]);
                *reinterpret_cast<float4*>(f32 + 64 * pair + 32 + e) =
                    make_float4(v1[e], v1[e + 1], v1[e + 2], v1[e + 3]);
            }
        }
        if (!last) {
#pragma unroll
            for (int e = 0; e < 32; ++e) { v0[e] *= eL; v1[e] *= eL; }
            tc::tmem_st32(tl + TM_S + 64 * pair, v0);
            tc::tmem_st32(tl + TM_S + 64 * pair + 32, v1);
        }
    }
}

// the initial row (fp32 global, or zero) into the master (scaled by eL) and the bf16
// copy (if `need`), and stored as bf16 to the workspace slot
__device__ __forceinline__ void load_in(uint32_t tl, int row, const float* __restrict__ src, bool need, float eL,
                                        uint8_t* slot) {
#pragma unroll 1
    for (int pair = 0; pair < 2; ++pair) {
        float v0[32], v1[32], p[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
            const float4 a = src ? *reinterpret_cast<const float4*>(src + 64 * pair + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 b = src ? *reinterpret_cast<const float4*>(src + 64 * pair + 32 + e)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            v0[e] = a.x; v0[e + 1] = a.y; v0[e + 2] = a.z; v0[e + 3] = a.w;
            v1[e] = b.x; v1[e + 1] = b.y; v1[e + 2] = b.z; v1[e + 3] = b.w;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            p[c] = __uint_as_float(tc::pack_bf16(v0[2 * c], v0[2 * c + 1]));
            p[16 + c] = __uint_as_float(tc::pack_bf16(v1[2 * c], v1[2 * c + 1]));
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(slot + stl::off(row, 8 * pair + c)) =
                make_uint4(__float_as_uint(p[4 * c]), __float_as_uint(p[4 * c + 1]), __float_as_uint(p[4 * c + 2]),
                           __float_as_uint(p[4 * c + 3]));
        if (need) {
            tc::tmem_st32(tl + TM_SB + 32 * pair, p);
#pragma unroll
            for (int e = 0; e < 32; ++e) { v0[e] *= eL; v1[e] *= eL; }
            tc::tmem_st32(tl + TM_S + 64 * pair, v0);
            tc::tmem_st32(tl + TM_S + 64 * pair + 32, v1);
        }
    }
}

__global__ void __launch_bounds__(kThreads)
bwd_chain_tc_kernel(Workspace ws, const float* __restrict__ S0, const float* __restrict__ dS_final,
                    float* __restrict__ dS0, int chains, int nch, unsigned long long timeout_ns, int stall) {
    // draining what was issued waits at least 100 ms, whatever the per-wait limit
    const unsigned long long drain_ns = timeout_ns > 100000000ull ? timeout_ns : 100000000ull;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* sm = smem_raw + (base - tc::smem_u32(smem_raw));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM_BARS);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + SM_BARS + 64);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SM_BARS + 68);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool rev = blockIdx.x >= (unsigned)chains;
    const int bh = rev ? blockIdx.x - chains : blockIdx.x;
    // update steps: the forward needs S_0 .. S_{nch-1} (nch - 1 updates), the reverse
    // dS'_{nch-1} .. dS'_0 and dS0 (nch updates)
    const int nit = rev ? nch : (nch > 0 ? nch - 1 : 0);
    auto chunk_of = [&](int n) { return rev ? nch - 1 - n : n; };
    auto state_slot = [&](int c) {   // bf16 128 x 128 (piece layout) in chunk c's fp32 slot
        return reinterpret_cast<uint8_t*>((rev ? ws.dS : ws.S) + ((size_t)bh * nch + c) * kDS);
    };

    if (tid == 0) {
        for (int i = 0; i < 8; ++i) tc::mbar_init(&bars[i], (i == B_SREADY || i == B_SPLIT || i == B_MREADY) ? 128u : 1u);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 4) tc::tmem_alloc(tslot, kCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tslot);

    auto fail = [&]() {
        *abort_flag = 1;
        latch_status(-4 /* COMBA_ETIMEOUT */);
    };
    auto wait = [&](int b, uint32_t parity) -> bool {
        const bool ok = (*abort_flag == 0) && tc::mbar_wait(&bars[b], parity, timeout_ns);
        if (!ok) fail();
        return ok;
    };

    if (warp < 4) {
        // ================================ state group ================================
        const int row = tid;   // state row i = TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        auto stage = [&](int n) { return sm + (n & 1) * ST_BYTES; };
        auto eL_of = [&](int n) { return reinterpret_cast<const float*>(stage(n) + ST_DEC)[32]; };
        bool ok = true;
        {   // initial state: S0 (forward) or dS_final (reverse), stored for chunk 0 / nch - 1
            const float* src = rev ? dS_final : S0;
            src = src ? src + ((size_t)bh * kD + row) * kD : nullptr;
            if (nch == 0) {   // no chunks: dS0 = dS_final
                if (rev && dS0)
                    for (int j = 0; j < kD; j += 4)
                        *reinterpret_cast<float4*>(dS0 + ((size_t)bh * kD + row) * kD + j) =
                            src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                const bool need = nit > 0;
                if (need) ok = wait(B_FULL0, 0);
                load_in(tl, row, src, need && ok, need && ok ? eL_of(0) : 1.f, state_slot(chunk_of(0)));
                tc::tmem_st_wait();
                tc::tc_fence_before();
                if (need && ok) tc::mbar_arrive(&bars[B_SREADY]);
            }
        }
        for (int n = 0; n < nit && ok; ++n) {
            const uint8_t* st = stage(n);
            const float* dec = reinterpret_cast<const float*>(st + ST_DEC);
            // ---- Xd^T = (U~^T - X'^T) diag(dec)  or  -Z diag(dec), as bf16 hi + lo
            if (!(ok = wait(B_MMA1, n & 1))) break;
            tc::tc_fence_after();
            {
                float xv[32], hv[16], lv[16];
                tc::tmem_ld32(tl + TM_X, xv);
                tc::tmem_ld_wait();
                const float* U = reinterpret_cast<const float*>(st + ST_U);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float d0 = dec[2 * c], d1 = dec[2 * c + 1];
                    const float a0 = rev ? -d0 * xv[2 * c] : d0 * (U[(2 * c) * kD + row] - xv[2 * c]);
                    const float a1 = rev ? -d1 * xv[2 * c + 1] : d1 * (U[(2 * c + 1) * kD + row] - xv[2 * c + 1]);
                    const uint32_t h = tc::pack_bf16(a0, a1);
                    hv[c] = __uint_as_float(h);
                    lv[c] = __uint_as_float(tc::pack_bf16(a0 - __uint_as_float(h << 16), a1 - __uint_as_float(h & 0xffff0000u)));
                }
                tc::tmem_st16(tl + TM_XH, hv);
                tc::tmem_st16(tl + TM_XH + 16, lv);
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            tc::mbar_arrive(&bars[B_SPLIT]);
            // ---- the updated state: the bf16 copy first (it releases the next chunk's
            // first MMA), then the store and the pre-scaled master (before the next SPLIT)
            const bool more = n + 1 < nit;
            if (more && !(ok = wait((n + 1) & 1 ? B_FULL1 : B_FULL0, ((n + 1) >> 1) & 1))) break;
            if (!(ok = wait(B_MMA2, n & 1))) break;
            tc::tc_fence_after();
            const int c = chunk_of(n);
            uint8_t* slot = nullptr;
            float* f32 = nullptr;
            if (!rev) slot = state_slot(c + 1);
            else if (c > 0) slot = state_slot(c - 1);
            else if (dS0) f32 = dS0 + ((size_t)bh * kD + row) * kD;
            uint32_t pk[64];
            copy_out(tl, !more, pk);
            if (more) {
                tc::tmem_st_wait();
                tc::tc_fence_before();
                tc::mbar_arrive(&bars[B_SREADY]);
            }
            store_out(tl, row, !more, more ? eL_of(n + 1) : 1.f, pk, slot, f32);
            tc::tmem_st_wait();
            tc::tc_fence_before();
            if (rev && more) tc::mbar_arrive(&bars[B_MREADY]);   // the master is scaled: dO^T G may add
        }
    } else {
        // ========================== copies and MMA issue (warp 4) ===================
        auto load = [&](int n) {   // chunk of step n into stage n & 1 (lane 0)
            const int c = chunk_of(n);
            const size_t ci = (size_t)bh * nch + c;
            uint8_t* st = sm + (n & 1) * ST_BYTES;
            uint64_t* full = &bars[(n & 1) ? B_FULL1 : B_FULL0];
            const uint8_t* wk = reinterpret_cast<const uint8_t*>(ws.W + ci * kL * kD);
            const uint8_t* cs = reinterpret_cast<const uint8_t*>(ws.C + ci * kDS);
            if (!rev) {
                tc::mbar_arrive_expect_tx(full, 16384u + 16384u + 256u);
                tc::bulk_load(st + ST_W, wk, 16384u, full);
                tc::bulk_load(st + ST_U, ws.U + ci * kL * kD, 16384u, full);
                tc::bulk_load(st + ST_DEC, cs + kPrepDec, 256u, full);
            } else {
                tc::mbar_arrive_expect_tx(full, 16384u + kPrepDec + 256u);
                tc::bulk_load(st + ST_W, wk, 16384u, full);
                tc::bulk_load(st + ST_G, cs, kPrepDec + 256u, full);
            }
        };
        int issued = 0;   // steps whose copies were issued
        if (lane == 0)
            for (; issued < 2 && issued < nit; ++issued) load(issued);
        issued = __shfl_sync(0xffffffffu, issued, 0);
        bool ok = true;
        // stall: a wait on a phase that nothing completes before the drain below (the
        // failure-path test), so it runs out after timeout_ns and ends the walk
        if (stall) ok = __all_sync(0xffffffffu, wait(B_DRAIN, 0)) != 0;
        for (int n = 0; n < nit && ok; ++n) {
            const uint32_t st = base + (n & 1) * ST_BYTES;
            ok = __all_sync(0xffffffffu, wait((n & 1) ? B_FULL1 : B_FULL0, (n >> 1) & 1) && wait(B_SREADY, n & 1)) != 0;
            if (!ok) break;
            tc::tc_fence_after();
            // first product of the chunk; the reverse pass's dO^T G follows once the state
            // group has pre-scaled the master (the chunk before's readout), and runs while
            // the state group splits Z
            tc::mma_bf16_ta_bk(tmem + TM_X, tmem + TM_SB, st + (rev ? ST_K : ST_W), 4096, ID_N32, 8, 0);
            tc::mma_commit(&bars[B_MMA1]);
            if (rev) {
                if (n > 0) {
                    ok = __all_sync(0xffffffffu, wait(B_MREADY, (n - 1) & 1)) != 0;
                    if (!ok) break;
                    tc::tc_fence_after();
                }
                tc::mma_amn_bmn(tmem + TM_S, st + ST_DO, 4096, st + ST_G, 4096, ID_N128AB, 2, 1);
                tc::mma_amn_bmn(tmem + TM_S, st + ST_DO, 4096, st + ST_GLO, 4096, ID_N128AB, 2, 1);
            }
            ok = __all_sync(0xffffffffu, wait(B_SPLIT, n & 1)) != 0;
            if (!ok) break;
            tc::tc_fence_after();
            const uint32_t bmn = st + (rev ? ST_W : ST_K);
            tc::mma_bf16_ta_bmn(tmem + TM_S, tmem + TM_XH, bmn, 4096, ID_N128B, 2, 1);
            tc::mma_bf16_ta_bmn(tmem + TM_S, tmem + TM_XH + 16, bmn, 4096, ID_N128B, 2, 1);
            tc::mma_commit(&bars[B_MMA2]);
            // the stage is free once this chunk's MMAs have completed
            if (n + 2 < nit) {
                ok = __all_sync(0xffffffffu, wait(B_MMA2, n & 1)) != 0;
                if (!ok) break;
                if (lane == 0) load(n + 2);
                issued = n + 3;
                __syncwarp();
            }
        }
        // drain: every MMA issued and every copy issued has completed before TMEM and
        // the ring are released
        __syncwarp();
        tc::mma_commit(&bars[B_DRAIN]);
        tc::mbar_wait(&bars[B_DRAIN], 0, drain_ns);
        for (int m = (issued > 2 ? issued - 2 : 0); m < issued; ++m)
            tc::mbar_wait(&bars[(m & 1) ? B_FULL1 : B_FULL0], (m >> 1) & 1, drain_ns);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kCols);
    }
}

}  // namespace chain
}  // namespace bwd
}  // namespace comba
