/*
 * comba.h -- C ABI of the B200 (sm_100a) Comba chunk-wise forward, its backward
 * and the decode step.
 *
 * The method: Comba, "Improving Bilinear RNNs with Closed-loop Control"
 * (PaperWeekly write-up and arXiv abstract 2506.02475).  Comba's recurrent
 * state S (dv x dk per batch element and head) follows a scalar-plus-low-rank
 * (SPLR) transition with the key as state feedback, and its output is read
 * through a second, output-side feedback on the same key (write-up, section
 * "Comba架构：基于闭环控制理论"):
 *
 *     S_t = alpha_t S_{t-1} - beta_t (S_{t-1} k_t) k_t^T + beta_t v_t k_t^T
 *     o_t = S_t (q_t - d_h k_t),           alpha_t = exp(log_alpha_t)
 *
 * The training/prefill form is chunk-wise: recurrent across chunks of `chunk`
 * tokens and parallel inside a chunk, with one unit-lower-triangular inverse
 * per chunk (write-up, section "硬件高效的分块并行计算").  The single-token
 * form is the constant-memory recurrent step used for decoding (write-up,
 * section "背景知识和相关工作").
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device,
 *    owned by the caller; the library allocates nothing per call and keeps no
 *    reference after the call is enqueued.
 *  - Layouts are dense row-major:
 *        q, k      [B, T, H, dk]      v, out [B, T, H, dv]
 *        log_alpha, beta  [B, T, H]   fp32 (log_alpha <= 0 expected, not required)
 *        d         [H]                fp32, the per-head output-correction factor
 *        S0, S_final [B, H, dv, dk]   fp32 (row i = value index, column j = key index)
 *  - q, k, v, out, S0 and S_final must be 16-byte aligned; log_alpha, beta and d
 *    4-byte aligned.
 *  - S0 == NULL means a zero initial state; S_final == NULL skips the final
 *    state.  S_final may alias S0 exactly (in-place state carry); no other
 *    output may overlap any input.
 *  - Work is enqueued asynchronously on `stream` (NULL = legacy default
 *    stream).  The return value reports argument and launch errors only;
 *    errors found on the device (a bounded wait that gave up) are latched in
 *    a per-device status word read by comba_get_last_error().
 *  - No C++ exception crosses this boundary.
 */
#ifndef COMBA_H_
#define COMBA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st* comba_stream_t;

enum comba_status {
    COMBA_OK = 0,
    COMBA_EINVAL = -1,        /* bad pointer, size, alignment or aliasing; nothing launched */
    COMBA_EUNSUPPORTED = -2,  /* valid but unsupported shape (see each entry point) */
    COMBA_ECUDA = -3,         /* a CUDA runtime call failed (launch, attribute, device query) */
    COMBA_ETIMEOUT = -4,      /* device side: a bounded wait gave up (comba_get_last_error) */
    COMBA_EDEVICE = -5        /* device side: inconsistent internal state detected */
};

/* Element type of q, k, v and the output cotangent in comba_chunk_bwd. */
enum comba_dtype {
    COMBA_BF16 = 0,           /* __nv_bfloat16 */
    COMBA_F32 = 1             /* float */
};

/*
 * Chunk-wise forward, bf16 inputs and output, fp32 gates/state/accumulation.
 *
 * Computes, for every (b, h) chain independently, out[b, t, h, :] = o_t for
 * t = 0..T-1 and S_final[b, h] = S_T, starting from S0[b, h] (write-up,
 * sections "Comba架构：基于闭环控制理论" and "硬件高效的分块并行计算").
 *
 * q, k, v, out: __nv_bfloat16.  Sizes: B, H >= 0; T >= 0 (T == 0 copies S0, or
 * zeros, to S_final); dk, dv multiples of 16 in [16, 128]; chunk in {16, 32,
 * 64}.  Any T is accepted: a last chunk shorter than `chunk` uses the same
 * math.  dk == dv == 128 with chunk == 64 runs the tensor-core kernel; other
 * shapes run the general kernel.
 */
int comba_chunk_fwd(const void* q, const void* k, const void* v,
                    const float* log_alpha, const float* beta, const float* d,
                    const float* S0, void* out, float* S_final,
                    int B, int T, int H, int dk, int dv, int chunk,
                    comba_stream_t stream);

/*
 * Chunk-wise forward over packed variable-length sequences whose value heads
 * share q / k heads in groups (the write-up's "mamba form" of the Comba family,
 * which works like multi-value attention with one shared 128-dim query and key:
 * end of section "硬件高效的分块并行计算").  Each (sequence, value head) is an
 * independent chain with the recurrence of comba_chunk_fwd; packing sequences
 * along one token axis is a layout of that computation (no counterpart in the
 * write-up).
 *
 * Layouts (total_T packed tokens, N sequences):
 *     q, k [total_T, Hqk, dk]   v, out [total_T, H, dv]   bf16
 *     log_alpha, beta [total_T, H] fp32     d [H] fp32
 *     S0, S_final [N, H, dv, dk] fp32 (per sequence and value head)
 *     cu_seqlens  DEVICE int32 [N + 1]: sequence n covers tokens
 *                 cu_seqlens[n] .. cu_seqlens[n+1]-1 (nondecreasing, from 0 to total_T)
 * Value head h reads q / k head h / (H / Hqk); Hqk must divide H (Hqk == H is
 * the plain per-head layout).  Each sequence is chunked from its own first token;
 * a zero-length sequence gets S_final = S0 (or zeros).  Shapes as comba_chunk_fwd
 * (dk == dv == 128 with chunk == 64 runs the tensor-core kernel).  A sequence
 * whose bounds are malformed (negative, decreasing, or past total_T) is skipped
 * and COMBA_EINVAL is latched in the device status word (comba_get_last_error);
 * the host cannot check device-resident bounds.
 */
int comba_chunk_fwd_varlen(const void* q, const void* k, const void* v,
                           const float* log_alpha, const float* beta, const float* d,
                           const float* S0, void* out, float* S_final,
                           const int* cu_seqlens, int N, int total_T, int H, int Hqk,
                           int dk, int dv, int chunk, comba_stream_t stream);

/*
 * comba_chunk_fwd from raw projections ("gate-in-kernel"): the kernel forms the
 * recurrence's inputs itself, per token and head,
 *     q_t = q_raw_t / sqrt(|q_raw_t|^2 + norm_eps)      (likewise k_t)
 *     log_alpha_t = -exp(A_log_h) * softplus(a_raw_t + dt_bias_h)
 *     beta_t = 1 / (1 + exp(-b_raw_t))
 * (the pages fix neither step: the decay follows the diagonal-SSM discretisation
 * described on the MaRK page, the rest are readings).  Layouts as comba_chunk_fwd
 * with q_raw, k_raw in place of q, k and a_raw, b_raw [B, T, H] fp32 in place of
 * log_alpha, beta; A_log [H] fp32 (device, required); dt_bias [H] fp32 (device;
 * NULL means zero); norm_eps >= 0.  In the tensor-core kernel the normalised q, k
 * rows are rounded to bf16 before use, as normalised bf16 inputs would be.
 */
int comba_chunk_fwd_gated(const void* q_raw, const void* k_raw, const void* v,
                          const float* a_raw, const float* b_raw, const float* A_log,
                          const float* dt_bias, const float* d, const float* S0, void* out,
                          float* S_final, int B, int T, int H, int dk, int dv, int chunk,
                          float norm_eps, comba_stream_t stream);

/*
 * Workspace the segmented form of comba_chunk_fwd_ws needs for this shape on the
 * current device, in bytes; 0 when the shape runs unsegmented (enough (b, h)
 * chains to fill the GPU, a T that is not a multiple of 64, or a shape outside the
 * tensor-core kernel).  The answer depends on the device's SM count.
 */
size_t comba_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk);

/*
 * comba_chunk_fwd with a caller-owned device workspace (16-byte aligned, not
 * overlapping any argument).  With at least comba_chunk_fwd_workspace_size()
 * bytes, a shape with too few (b, h) chains for the GPU is run segmented: each
 * chain's sequence is cut into P pieces that run as independent chains, joined by
 * their affine state transitions (the end state from S is S M + R, with R the
 * piece's end state from S = 0 and M its end state from S = I with V = 0), then
 * rerun from the composed start states for the outputs.  The result is the same
 * computation regrouped (write-up, section "硬件高效的分块并行计算": recurrent across
 * blocks, parallel inside), equal up to rounding.  With less workspace (or NULL)
 * it behaves exactly as comba_chunk_fwd.  The workspace is in use until the work
 * enqueued on `stream` completes.
 */
int comba_chunk_fwd_ws(const void* q, const void* k, const void* v,
                       const float* log_alpha, const float* beta, const float* d,
                       const float* S0, void* out, float* S_final,
                       int B, int T, int H, int dk, int dv, int chunk,
                       void* workspace, size_t workspace_bytes, comba_stream_t stream);

/*
 * comba_chunk_fwd_ws with the workspace taken from a scratch array in the
 * library's static device memory (48 MiB, room for B * P * H <= 128 segment-chains;
 * larger shapes run unsegmented): neither the library nor the caller allocates
 * anything for the call.  No counterpart in the write-up; an entry point for
 * callers that cannot provide device memory.  The scratch is one per device for the
 * whole process, so calls must not run concurrently (use one stream, or order them).
 */
int comba_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                            const float* log_alpha, const float* beta, const float* d,
                            const float* S0, void* out, float* S_final,
                            int B, int T, int H, int dk, int dv, int chunk,
                            comba_stream_t stream);

/*
 * comba_chunk_fwd from and to HOST memory: the same computation, with the inputs
 * copied to the device and the results back inside the call, pipelined over
 * `slices` groups of batch rows so that the copies in, the kernel and the copies
 * out of different groups overlap (no counterpart in the write-up).
 *
 * q, k, v, log_alpha, beta, d, S0, out, S_final: HOST pointers with the layouts,
 * alignment and aliasing rules of comba_chunk_fwd (pinned memory lets the copies
 * run asynchronously and overlap; pageable memory works but serialises).  They
 * stay owned by the caller, who keeps them valid, the inputs unchanged and the
 * outputs unread until `stream` has passed this call.
 * workspace: DEVICE memory, 256-byte aligned, at least
 * comba_chunk_fwd_host_workspace_size(B, T, H, dk, dv) bytes, owned by the caller
 * and not to be used by anything else until `stream` has passed this call.  The
 * copies run on two library-owned streams per device (created on first use and
 * kept for the process) ordered after the work already on `stream`; `stream`
 * itself completes only once out and S_final are in host memory.  slices >= 1
 * (more slices than batch rows act as one per row; at most 64).  T == 0 with
 * S0 == NULL zeroes S_final after synchronising `stream`.
 */
size_t comba_chunk_fwd_host_workspace_size(int B, int T, int H, int dk, int dv);
int comba_chunk_fwd_host(const void* q, const void* k, const void* v,
                         const float* log_alpha, const float* beta, const float* d,
                         const float* S0, void* out, float* S_final,
                         int B, int T, int H, int dk, int dv, int chunk,
                         void* workspace, size_t workspace_bytes, int slices,
                         comba_stream_t stream);

/*
 * comba_chunk_fwd on the tensor-core kernel (dk = dv = 128, chunk 64; other shapes
 * return COMBA_EUNSUPPORTED) with its per-wait limit set to `timeout_ns` instead of
 * the default 2 s, and, when `stall` is nonzero, with one extra wait (the MMA-issue
 * warp's, before the first chunk's state pass) on a barrier phase that nothing
 * completes.  It exists to exercise the kernel's failure path without faulting the
 * GPU: the wait runs out, COMBA_ETIMEOUT is latched in the device status word
 * (comba_get_last_error), every thread leaves the chunk loop (the other waits run
 * out too), the kernel waits (for at least 100 ms more) for the copies and MMAs it
 * has already issued, releases its tensor memory and returns; the outputs are then
 * undefined.  With stall == 0 it is comba_chunk_fwd with another wait limit.
 */
int comba_chunk_fwd_stall_test(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta, const float* d,
                               const float* S0, void* out, float* S_final,
                               int B, int T, int H, int dk, int dv, int chunk,
                               unsigned long long timeout_ns, int stall, comba_stream_t stream);

/*
 * The affine state transition of a piece of sequence: over tokens 0 .. T-1 the
 * state pass maps a start state S to S M + R (the write-up's "recurrent across
 * blocks, parallel inside" form, section "硬件高效的分块并行计算", one level up:
 * R is the end state from S = 0, M the end state from S = I with V = 0).  Both
 * come from one launch of the tensor-core kernel over the chains twice stacked,
 * with no outputs written; a caller that holds pieces of a longer sequence (one
 * per GPU, say) composes the pieces' start states from them (comba_state_compose)
 * and reruns each piece with comba_chunk_fwd.
 *
 * q, k, v, log_alpha, beta, d: as comba_chunk_fwd (bf16, dk = dv = 128, chunk 64;
 * other shapes return COMBA_EUNSUPPORTED).  RM: fp32 [2, B, H, 128, 128] device
 * memory, 16-byte aligned, not overlapping an input: R of every chain, then M of
 * every chain (the layout comba_state_compose reads, with P = 1).  T == 0 gives
 * R = 0, M = I.
 */
int comba_chunk_fwd_transition(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta, const float* d,
                               float* RM, int B, int T, int H, int dk, int dv, int chunk,
                               comba_stream_t stream);

/*
 * Chunk-wise forward with fp32 q, k, v and out (same math, same layouts, same
 * size rules as comba_chunk_fwd); every product is an fp32 FMA, no reduced-
 * precision tensor-core arithmetic.
 */
int comba_chunk_fwd_f32(const float* q, const float* k, const float* v,
                        const float* log_alpha, const float* beta, const float* d,
                        const float* S0, float* out, float* S_final,
                        int B, int T, int H, int dk, int dv, int chunk,
                        comba_stream_t stream);

/*
 * One recurrent (decode) step for every (b, h): the recurrence above at a
 * single token, updating the resident state in place (write-up, section
 * "背景知识和相关工作": constant memory and O(1) work per token).
 *
 * q, k [B, H, dk] and v [B, H, dv]: __nv_bfloat16; log_alpha, beta [B, H] fp32;
 * d [H] fp32; S [B, H, dv, dk] fp32, read and overwritten with S_t; out
 * [B, H, dv] __nv_bfloat16 receives o_t = S_t (q - d_h k).  dk in {32, 64,
 * 128}; dv a multiple of 16 in [16, 128].  B or H == 0 is a no-op.
 */
int comba_recurrent_step(const void* q, const void* k, const void* v,
                         const float* log_alpha, const float* beta, const float* d,
                         float* S, void* out, int B, int H, int dk, int dv,
                         comba_stream_t stream);

/*
 * The decode step of the mamba form (value heads sharing q / k heads in groups,
 * as in comba_chunk_fwd_varlen): comba_recurrent_step with q, k [B, Hqk, dk];
 * value head h reads q / k head h / (H / Hqk).  Hqk must divide H; Hqk == H is
 * comba_recurrent_step itself.
 */
int comba_recurrent_step_grouped(const void* q, const void* k, const void* v,
                                 const float* log_alpha, const float* beta, const float* d,
                                 float* S, void* out, int B, int H, int Hqk, int dk, int dv,
                                 comba_stream_t stream);

/*
 * Backward of the chunk-wise forward: the gradients of
 *     L = <dout, out> + <dS_final, S_final>
 * with respect to q, k, v, log_alpha, beta, d and S0, for the recurrence and
 * output above.  The write-up (section "硬件高效的分块并行计算") states only that
 * the backward pass reuses the chunk-level states and the per-chunk inverse; this
 * entry point computes the adjoint of the chunk form in four stages.
 *  1. Per chunk in parallel: W, U~, the inverse and dO^T (Gamma Q~ - P W).
 *  2. The chunk-start states, chunks in order.
 *  3. The end-state gradients, chunks in reverse.
 *  4. Per chunk in parallel: the input gradients.
 * It recomputes the states rather than reading saved ones.  Chunks are 32 tokens
 * (a tiling choice: the result is the same function of the inputs for any chunk
 * length).  Precision: fp32 inputs, and bf16 inputs with dk or dv below 128, are
 * computed to about fp32 accuracy (warp MMAs on split tf32 operands; every gradient
 * within rel-L2 1e-4 of the exact one).  bf16 inputs with dk = dv = 128 take the
 * tensor-core form: stages 2 and 3 run as one launch on tcgen05 MMAs with the
 * states in bf16, as do the state products of stage 4; every gradient, dS0
 * included, is within rel-L2 5e-3 of the exact one (the bf16 workloads' bound).
 *
 * q, k [B, T, H, dk], v and dout [B, T, H, dv]: element type `dtype` (COMBA_BF16 or
 * COMBA_F32), the same values the forward read.  log_alpha, beta [B, T, H], d [H],
 * S0 [B, H, dv, dk]: fp32 (S0 NULL = zero initial state).  dS_final [B, H, dv,
 * dk] fp32 or NULL (= 0).
 * Outputs, fp32:
 *  - dq, dk [B, T, H, dk] and dv [B, T, H, dv];
 *  - dlog_alpha, dbeta [B, T, H];
 *  - dd [H] (NULL skips it; a sum over batch and time in a fixed order);
 *  - dS0 [B, H, dv, dk] (NULL skips it).
 * dk, dv in {32, 64, 128}; any T >= 0 (T == 0: dS0 = dS_final, dd = 0); B * H <= 65535.
 * workspace: DEVICE memory, 16-byte aligned, at least
 * comba_chunk_bwd_workspace_size(B, T, H, dk, dv) bytes (per chunk: room for W, U~
 * and three dv x dk fp32 matrices), owned by the caller and in use until `stream`
 * has passed the call; its contents between calls are unspecified.  q, k, v, dout, S0 and dS_final 16-byte aligned; everything else
 * 4-byte aligned.  No output may overlap an input,
 * another output or the workspace.  Returns COMBA_EINVAL for a bad size, pointer,
 * alignment, overlap or workspace; COMBA_EUNSUPPORTED for B * H > 65535.
 */
size_t comba_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv);
int comba_chunk_bwd(const void* q, const void* k, const void* v,
                    const float* log_alpha, const float* beta, const float* d,
                    const float* S0, const void* dout, const float* dS_final,
                    float* dq, float* dk, float* dv, float* dlog_alpha, float* dbeta,
                    float* dd, float* dS0,
                    int B, int T, int H, int dk_dim, int dv_dim, int dtype,
                    void* workspace, size_t workspace_bytes, comba_stream_t stream);

/*
 * comba_chunk_bwd in its tensor-core form (dtype COMBA_BF16, dk = dv = 128; other
 * inputs return COMBA_EUNSUPPORTED) with the state passes' per-wait limit set to
 * `timeout_ns` instead of the default 2 s, and, when `stall` is nonzero, with one
 * extra wait in each state-pass CTA (its copy and MMA-issue warp's, before the first
 * chunk) on a barrier phase that nothing completes.  It exists to exercise that
 * kernel's failure path without faulting the GPU: the wait runs out, COMBA_ETIMEOUT
 * is latched in the device status word (comba_get_last_error), every thread leaves
 * the chunk walk (the other waits run out too), the kernel waits (for at least 100
 * ms more) for the copies and MMAs it has already issued, releases its tensor memory
 * and returns; the gradients are then undefined.  With stall == 0 it is
 * comba_chunk_bwd with another wait limit.
 */
int comba_chunk_bwd_stall_test(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta, const float* d,
                               const float* S0, const void* dout, const float* dS_final,
                               float* dq, float* dk, float* dv, float* dlog_alpha, float* dbeta,
                               float* dd, float* dS0,
                               int B, int T, int H, int dk_dim, int dv_dim, int dtype,
                               void* workspace, size_t workspace_bytes,
                               unsigned long long timeout_ns, int stall, comba_stream_t stream);

/*
 * Start states of P consecutive sequence pieces from their affine state
 * transitions: over a piece, the state pass maps a start state S to S M + R (R: the
 * end state from S = 0; M: the end state from S = I with V = 0).  This is the
 * write-up's "recurrent across blocks" form applied to pieces, as in
 * comba_chunk_fwd_ws; here the transitions come from the caller, e.g. gathered
 * from the ranks of a context-parallel group.
 *
 *     S_start[b, 0, h] = S0[b, h]  (0 when S0 == NULL)
 *     S_start[b, p, h] = S_start[b, p-1, h] M[b, p-1, h] + R[b, p-1, h]
 *
 * RM: fp32, the R of all pieces [B, P, H, 128, 128] followed by the M of all
 * pieces [B, P, H, 128, 128] (the last piece's R and M are not read).  S0 [B, H,
 * 128, 128] or NULL; S_start [B, P, H, 128, 128].  dk = dv = 128.  All 16-byte
 * aligned; S_start must not overlap RM or S0.  fp32 FMA arithmetic.
 */
int comba_state_compose(const float* RM, const float* S0, float* S_start, int B, int H, int P,
                        comba_stream_t stream);

/*
 * Reads and clears the current device's status word (synchronises the
 * device first).  Returns COMBA_OK, COMBA_ETIMEOUT, COMBA_EDEVICE, COMBA_EINVAL
 * (a malformed packed-sequence bound, see comba_chunk_fwd_varlen), or
 * COMBA_ECUDA if the synchronisation or the read itself failed.
 */
int comba_get_last_error(void);

/*
 * The same status word, read after synchronising `stream` only (work on other
 * streams keeps running).  The word is shared by every stream of the device: it
 * holds the first error latched by any of this library's kernels since the last
 * read, so a kernel still running on another stream may latch an error after this
 * call returns.  The read and the clear are ordered on `stream`.
 */
int comba_get_last_error_stream(comba_stream_t stream);

/* Static, NUL-terminated description of a status code. */
const char* comba_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int comba_version(void);

#ifdef __cplusplus
}
#endif

#endif /* COMBA_H_ */
