// General chunk-wise Comba forward: fp32 FMA arithmetic, any supported shape.
//
// This kernel serves comba_chunk_fwd_f32 (fp32 inputs, where reduced-precision
// tensor-core products would not meet fp32 accuracy) and the bf16 entry point
// for shapes the tensor-core kernel does not cover.  One CTA owns one
// (b, h, dv-tile) chain slice and walks the chunks in order; inside a chunk
// all work is parallel over the CTA's threads.
//
// Chunk algebra (derived from the recurrence; the write-up, section
// "硬件高效的分块并行计算", gives the structure -- recurrent across chunks,
// parallel within, intermediates W and U from a single inverse -- but its
// formulas were lost).  With chunk-start state S, local positions r, s and
// g_r = sum_{i<=r} log_alpha_i (g_0 = 0):
//   A_rs = beta_r e^{g_{r-1}-g_s} (k_r.k_s), s < r      (strictly lower)
//   [W | U~] = (I + A)^{-1} [diag(beta_r e^{g_{r-1}}) K | diag(beta_r) V]
//   X = U~ - W S^T                                      (rows beta_r (v_r - S_{r-1} k_r))
//   P_rs = e^{g_r-g_s} (q_r.k_s - d k_r.k_s), s <= r
//   O = diag(e^{g_r}) (Q - d K) S^T + P X
//   S <- e^{g_L} S + X^T diag(e^{g_L-g_s}) K
// The inverse is applied by forward substitution on the right-hand sides, so
// every exponent formed is a difference g_a - g_b with a >= b (value <= 1).
#pragma once

#include "common.cuh"

namespace comba {

struct SimtSmem {
    int ldk, ldv, ldc, ldy, ldx;
    size_t k, q, s, v, kk, pp, y, x, g, gp, bt, es, total;  // float offsets
};

__host__ __device__ inline SimtSmem simt_smem_layout(int dk, int dvt, int C) {
    SimtSmem m;
    m.ldk = dk + 1;
    m.ldv = dvt + 1;
    m.ldc = C + 1;
    m.ldy = dk + dvt + 1;
    m.ldx = dvt + 1;
    size_t o = 0;
    m.k = o;  o += (size_t)C * m.ldk;
    m.q = o;  o += (size_t)C * m.ldk;
    m.s = o;  o += (size_t)dvt * m.ldk;
    m.v = o;  o += (size_t)C * m.ldv;
    m.kk = o; o += (size_t)C * m.ldc;
    m.pp = o; o += (size_t)C * m.ldc;
    m.y = o;  o += (size_t)C * m.ldy;
    m.x = o;  o += (size_t)C * m.ldx;
    m.g = o;  o += C;
    m.gp = o; o += C;
    m.bt = o; o += C;
    m.es = o; o += C;
    m.total = o;
    return m;
}

constexpr int kSimtThreads = 256;

template <typename Tin>
__global__ void __launch_bounds__(kSimtThreads)
chunk_fwd_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                      const Tin* __restrict__ v, const float* __restrict__ log_alpha,
                      const float* __restrict__ beta, const float* __restrict__ dvec,
                      const float* S0, Tin* __restrict__ out, float* S_final,
                      int T, int H, int dk, int dv, int C, int dvt,
                      const int* __restrict__ cu_seqlens, int Hqk,
                      const float* __restrict__ A_log, const float* __restrict__ dt_bias, float norm_eps) {
    extern __shared__ float sm[];
    const SimtSmem L_ = simt_smem_layout(dk, dvt, C);
    float* Ks = sm + L_.k;
    float* Qs = sm + L_.q;
    float* Ss = sm + L_.s;
    float* Vs = sm + L_.v;
    float* KK = sm + L_.kk;   // becomes A (strictly lower) in place
    float* PP = sm + L_.pp;
    float* Y = sm + L_.y;     // [W | U~] after the substitution
    float* Xs = sm + L_.x;
    float* gs = sm + L_.g;
    float* gps = sm + L_.gp;
    float* bs = sm + L_.bt;
    float* es = sm + L_.es;
    const int ldk = L_.ldk, ldv = L_.ldv, ldc = L_.ldc, ldy = L_.ldy, ldx = L_.ldx;

    const int tid = threadIdx.x, nt = blockDim.x;
    const int i0 = blockIdx.x * dvt;
    const int h = blockIdx.y, b = blockIdx.z;
    // The chain's tokens: rows b T .. b T + T - 1 of the token axis, or, for packed
    // sequences, rows cu_seqlens[b] .. cu_seqlens[b+1]-1 (T = total tokens); its q / k
    // head is h / (H / Hqk).
    size_t row0 = (size_t)b * T;
    int Tc = T;
    if (cu_seqlens) {
        const int s0 = cu_seqlens[b], s1 = cu_seqlens[b + 1];
        if (s0 < 0 || s1 < s0 || s1 > T) {   // malformed bounds: the sequence is skipped
            if (threadIdx.x == 0) latch_status(-1 /* COMBA_EINVAL */);
            Tc = 0;
        } else {
            row0 = (size_t)s0;
            Tc = s1 - s0;
        }
    }
    const int hq = h / (H / Hqk);
    // gated inputs (A_log != null): q and k rows are L2-normalised here and log_alpha /
    // beta hold raw gate projections a, b: log-decay -exp(A_log_h) softplus(a + dt_bias_h),
    // beta sigmoid(b)
    const float gA = A_log ? -expf(A_log[h]) : 0.f;
    const float gdt = (A_log && dt_bias) ? dt_bias[h] : 0.f;
    const int nv = min(dvt, dv - i0);
    const int ny = dk + nv;
    const float dh = dvec[h];
    const size_t state_off = ((size_t)b * H + h) * (size_t)dv * dk;

    for (int idx = tid; idx < nv * dk; idx += nt) {
        const int i = idx / dk, j = idx % dk;
        Ss[i * ldk + j] = S0 ? S0[state_off + (size_t)(i0 + i) * dk + j] : 0.f;
    }

    for (int c0 = 0; c0 < Tc; c0 += C) {
        const int L = min(C, Tc - c0);
        __syncthreads();
        for (int idx = tid; idx < L * dk; idx += nt) {
            const int r = idx / dk, j = idx % dk;
            const size_t off = ((row0 + c0 + r) * Hqk + hq) * dk + j;
            Ks[r * ldk + j] = to_f32(k[off]);
            Qs[r * ldk + j] = to_f32(q[off]);
        }
        for (int idx = tid; idx < L * nv; idx += nt) {
            const int r = idx / nv, i = idx % nv;
            Vs[r * ldv + i] = to_f32(v[((row0 + c0 + r) * H + h) * dv + i0 + i]);
        }
        if (tid < L) {
            const size_t o = (row0 + c0 + tid) * H + h;
            float la = log_alpha[o], bt = beta[o];
            if (A_log) {
                const float x = la + gdt;
                la = gA * (fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))));
                bt = 1.f / (1.f + expf(-bt));
            }
            gs[tid] = la;
            bs[tid] = bt;
        }
        __syncthreads();
        if (A_log) {   // L2-normalise the chunk's q and k rows in place
            for (int idx = tid; idx < 2 * L; idx += nt) {
                float* rowp = (idx < L ? Ks : Qs) + (idx % L) * ldk;
                float ss = 0.f;
                for (int j = 0; j < dk; ++j) ss = fmaf(rowp[j], rowp[j], ss);
                const float rs = rsqrtf(ss + norm_eps);
                for (int j = 0; j < dk; ++j) rowp[j] *= rs;
            }
            __syncthreads();
        }
        if (tid == 0) {  // within-chunk cumulative log-decay
            float acc = 0.f;
            for (int r = 0; r < L; ++r) {
                gps[r] = acc;
                acc += gs[r];
                gs[r] = acc;
            }
            for (int r = 0; r < L; ++r) es[r] = expf(acc - gs[r]);
        }
        __syncthreads();
        // Gram products of the chunk, lower triangle including the diagonal.
        for (int idx = tid; idx < L * L; idx += nt) {
            const int r = idx / L, s = idx % L;
            if (s > r) continue;
            float kk = 0.f, qk = 0.f;
            for (int j = 0; j < dk; ++j) {
                const float ks = Ks[s * ldk + j];
                kk = fmaf(Ks[r * ldk + j], ks, kk);
                qk = fmaf(Qs[r * ldk + j], ks, qk);
            }
            PP[r * ldc + s] = expf(gs[r] - gs[s]) * (qk - dh * kk);
            KK[r * ldc + s] = (s < r) ? bs[r] * expf(gps[r] - gs[s]) * kk : 0.f;
        }
        // Right-hand sides of the unit-lower-triangular system.
        for (int idx = tid; idx < L * ny; idx += nt) {
            const int r = idx / ny, c = idx % ny;
            Y[r * ldy + c] = (c < dk) ? bs[r] * expf(gps[r]) * Ks[r * ldk + c]
                                      : bs[r] * Vs[r * ldv + (c - dk)];
        }
        __syncthreads();
        // Forward substitution: row r of (I + A) Y = RHS, rows in order.
        for (int r = 1; r < L; ++r) {
            for (int c = tid; c < ny; c += nt) {
                float acc = Y[r * ldy + c];
                for (int s = 0; s < r; ++s) acc = fmaf(-KK[r * ldc + s], Y[s * ldy + c], acc);
                Y[r * ldy + c] = acc;
            }
            __syncthreads();
        }
        // X = U~ - W S^T
        for (int idx = tid; idx < L * nv; idx += nt) {
            const int r = idx / nv, i = idx % nv;
            float acc = Y[r * ldy + dk + i];
            for (int j = 0; j < dk; ++j) acc = fmaf(-Y[r * ldy + j], Ss[i * ldk + j], acc);
            Xs[r * ldx + i] = acc;
        }
        __syncthreads();
        // O = diag(e^g) (Q - d K) S^T + P X
        for (int idx = tid; idx < L * nv; idx += nt) {
            const int r = idx / nv, i = idx % nv;
            float acc = 0.f;
            for (int j = 0; j < dk; ++j)
                acc = fmaf(Qs[r * ldk + j] - dh * Ks[r * ldk + j], Ss[i * ldk + j], acc);
            acc *= expf(gs[r]);
            for (int s = 0; s <= r; ++s) acc = fmaf(PP[r * ldc + s], Xs[s * ldx + i], acc);
            out[((row0 + c0 + r) * H + h) * dv + i0 + i] = from_f32<Tin>(acc);
        }
        __syncthreads();
        // S <- e^{g_L} S + X^T diag(e^{g_L - g_s}) K
        const float eL = expf(gs[L - 1]);
        for (int idx = tid; idx < nv * dk; idx += nt) {
            const int i = idx / dk, j = idx % dk;
            float acc = eL * Ss[i * ldk + j];
            for (int s = 0; s < L; ++s) acc = fmaf(Xs[s * ldx + i] * es[s], Ks[s * ldk + j], acc);
            Ss[i * ldk + j] = acc;
        }
    }
    __syncthreads();
    if (S_final) {
        for (int idx = tid; idx < nv * dk; idx += nt) {
            const int i = idx / dk, j = idx % dk;
            S_final[state_off + (size_t)(i0 + i) * dk + j] = Ss[i * ldk + j];
        }
    }
}

}  // namespace comba
