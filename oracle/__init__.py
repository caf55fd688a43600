"""Float64 CPU oracle for the Comba chunk-wise forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
package never imports it and shares no code with it; nothing here is a
fallback for the GPU path.

Contents (each pinned by the ``-m "not gpu"`` tests against closed forms, a
hand-worked example, brute-force transition products and invariants):

* ``recurrence``      -- the token-by-token definition in plain C (float64,
                         OpenMP over the independent (b, h) chains);
* ``recurrence_np``   -- the same definition in NumPy, for small cases;
* ``chunked_np``      -- the chunk-wise (inter-chunk recurrent, intra-chunk
                         parallel) formulation with one unit-lower-triangular
                         inverse per chunk, in float64.  It is not the oracle
                         for the GPU; it pins the chunk algebra the kernels use
                         to the recurrence.
* ``decode_steps``    -- repeated single-token steps (the recurrence at T=1).
* ``recurrence_bwd_np`` -- gradients of the recurrence (reverse mode through the
                         token loop, float64), pinned by finite differences of
                         ``recurrence``, torch.autograd and a closed form;
* ``chunked_bwd_np``  -- the same gradients through the chunk form (the adjoint
                         the backward kernels use), pinned to ``recurrence_bwd_np``;
* ``gate_inputs``     -- the inputs of the recurrence from raw projections: q, k
                         L2-normalised per token and head, log_alpha and beta from
                         raw gate projections (a reading: the pages fix neither the
                         normalisation constant nor the gate parameterisation).

The recurrence (Comba, "Improving Bilinear RNNs with Closed-loop Control";
PaperWeekly write-up, sections "Comba架构：基于闭环控制理论" and
"硬件高效的分块并行计算"; arXiv abstract) whose formulas were lost in the
page extraction, read as:

    S_t = alpha_t S_{t-1} - beta_t S_{t-1} k_t k_t^T + beta_t v_t k_t^T
    o_t = S_t (q_t - d_h k_t),          alpha_t = exp(log_alpha_t).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "comba_recurrence.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libcomba_oracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (float64, no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math",
                               "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            lib.comba_oracle_recurrence_f64.argtypes = [dp] * 10 + [ctypes.c_long] * 5 + [ctypes.c_int]
            lib.comba_oracle_recurrence_f64.restype = ctypes.c_int
            lib.comba_oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().comba_oracle_num_threads())


def _f64(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: widen the stored (possibly bf16) values exactly
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def recurrence(q, k, v, log_alpha, beta, d, S0=None, beta_write=None,
               threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Token-by-token float64 recurrence (C).  Shapes: q,k [B,T,H,dk], v [B,T,H,dv],
    log_alpha, beta [B,T,H], d [H], S0 [B,H,dv,dk] or None.
    ``beta_write`` (self-tests only) replaces beta in the write term.
    Returns (out [B,T,H,dv], S_final [B,H,dv,dk]) in float64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be, d = _f64(log_alpha), _f64(beta), _f64(d)
    bw = be if beta_write is None else _f64(beta_write)
    S0 = _f64(S0)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and v.shape == (B, T, H, dv)
    assert la.shape == (B, T, H) and be.shape == (B, T, H) and bw.shape == (B, T, H)
    assert d.shape == (H,)
    assert S0 is None or S0.shape == (B, H, dv, dk)
    out = np.empty((B, T, H, dv), dtype=np.float64)
    S_final = np.empty((B, H, dv, dk), dtype=np.float64)
    rc = _load().comba_oracle_recurrence_f64(
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be), _ptr(bw), _ptr(d), _ptr(S0),
        _ptr(out), _ptr(S_final), B, T, H, dk, dv, int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle recurrence failed with status {rc}")
    return out, S_final


def recurrence_np(q, k, v, log_alpha, beta, d, S0=None, beta_write=None):
    """The same token-by-token definition in NumPy (vectorised over b, h only)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be, d = _f64(log_alpha), _f64(beta), _f64(d)
    bw = be if beta_write is None else _f64(beta_write)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dv, dk)) if S0 is None else _f64(S0).copy()
    out = np.empty((B, T, H, dv))
    for t in range(T):
        kt, qv, vt = k[:, t], q[:, t], v[:, t]                      # [B,H,d]
        a = np.exp(la[:, t])[..., None, None]                       # [B,H,1,1]
        Sk = np.einsum("bhij,bhj->bhi", S, kt)                      # S_{t-1} k_t
        S = (a * S
             - be[:, t][..., None, None] * np.einsum("bhi,bhj->bhij", Sk, kt)
             + bw[:, t][..., None, None] * np.einsum("bhi,bhj->bhij", vt, kt))
        qt = qv - d[None, :, None] * kt
        out[:, t] = np.einsum("bhij,bhj->bhi", S, qt)
    return out, S


def chunked_np(q, k, v, log_alpha, beta, d, S0=None, chunk: int = 64):
    """Chunk-wise formulation in float64: sequential over chunks of length C,
    parallel inside a chunk, with one unit-lower-triangular inverse per chunk
    (the write-up's "block-recurrent, intra-block parallel" form with the single
    inverse that the scalar-plus-low-rank transition allows).

    Per chunk with chunk-start state S, local positions r, s = 1..L, and
    g_r = sum_{i<=r} log_alpha_i (g_0 = 0):
        A_rs  = beta_r exp(g_{r-1} - g_s) (k_r . k_s)      for s < r, else 0
        Tinv  = (I + A)^{-1}
        W     = Tinv diag(beta_r exp(g_{r-1})) K,   U~ = Tinv diag(beta_r) V
        X     = U~ - W S^T                          (rows: beta_r (v_r - S_{r-1} k_r))
        P_rs  = exp(g_r - g_s) ((q_r - d k_r) . k_s)  for s <= r, else 0
        O     = diag(exp(g_r)) (Q - d K) S^T + P X
        S_new = exp(g_L) S + X^T diag(exp(g_L - g_s)) K
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be, d = _f64(log_alpha), _f64(beta), _f64(d)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dv, dk)) if S0 is None else _f64(S0).copy()
    out = np.empty((B, T, H, dv))
    # chain-major views: [B,H,T,*]
    qh, kh, vh = q.transpose(0, 2, 1, 3), k.transpose(0, 2, 1, 3), v.transpose(0, 2, 1, 3)
    lah, beh = la.transpose(0, 2, 1), be.transpose(0, 2, 1)
    dd = d[None, :, None, None]
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        L = c1 - c0
        K, Q, V = kh[:, :, c0:c1], qh[:, :, c0:c1], vh[:, :, c0:c1]
        bt = beh[:, :, c0:c1]
        g = np.cumsum(lah[:, :, c0:c1], axis=-1)                       # g_1..g_L
        g_prev = np.concatenate([np.zeros_like(g[..., :1]), g[..., :-1]], axis=-1)
        KK = np.einsum("bhrd,bhsd->bhrs", K, K)
        QK = np.einsum("bhrd,bhsd->bhrs", Q, K)
        strict = np.tril(np.ones((L, L), dtype=bool), k=-1)
        incl = np.tril(np.ones((L, L), dtype=bool))
        # exponent differences are only formed where they are <= 0 (s <= r)
        dg_prev = np.where(strict, g_prev[..., :, None] - g[..., None, :], 0.0)
        A = np.where(strict, bt[..., :, None] * np.exp(dg_prev) * KK, 0.0)
        Tinv = np.linalg.solve(np.eye(L) + A, np.broadcast_to(np.eye(L), A.shape))
        W = Tinv @ ((bt * np.exp(g_prev))[..., None] * K)
        Ut = Tinv @ (bt[..., None] * V)
        X = Ut - W @ np.swapaxes(S, -1, -2)
        dg = np.where(incl, g[..., :, None] - g[..., None, :], 0.0)
        P = np.where(incl, np.exp(dg) * (QK - dd * KK), 0.0)
        Qt = Q - dd * K
        O = np.exp(g)[..., None] * (Qt @ np.swapaxes(S, -1, -2)) + P @ X
        out[:, c0:c1] = O.transpose(0, 2, 1, 3)
        gL = g[..., -1:]
        S = np.exp(gL)[..., None] * S + np.swapaxes(X, -1, -2) @ (np.exp(gL - g)[..., None] * K)
    return out, S


def decode_steps(steps, d, S, threads: int = 0):
    """Apply single-token steps in order.  ``steps`` yields dicts with q, k [B,H,dk],
    v [B,H,dv], log_alpha, beta [B,H]; S [B,H,dv,dk] is the state before the first
    step.  Returns (list of outputs [B,H,dv], final state), float64."""
    S = _f64(S)
    outs = []
    for st in steps:
        q = _f64(st["q"])[:, None]
        k = _f64(st["k"])[:, None]
        v = _f64(st["v"])[:, None]
        la = _f64(st["log_alpha"])[:, None]
        be = _f64(st["beta"])[:, None]
        o, S = recurrence(q, k, v, la, be, d, S, threads=threads)
        outs.append(o[:, 0])
    return outs, S


def gate_inputs(q_raw, k_raw, a_raw, b_raw, A_log, dt_bias, eps: float = 1e-6):
    """The recurrence's q, k, log_alpha and beta from raw projections, float64:

        q_t = q_raw_t / sqrt(|q_raw_t|^2 + eps)   (likewise k; per token and head)
        log_alpha_t = -exp(A_log_h) * softplus(a_raw_t + dt_bias_h)
        beta_t = sigmoid(b_raw_t)

    q_raw, k_raw [B,T,H,dk]; a_raw, b_raw [B,T,H]; A_log, dt_bias [H].  The Comba
    write-up fixes neither step.  The decay follows the diagonal-SSM discretisation
    the pages describe on the MaRK page (Hydra: A = -exp(A_log), step softplus(input
    + bias), log of the discrete eigenvalue = A * step), which is also how the
    synthetic gates are drawn; beta is a sigmoid gate and q, k are L2-normalised
    with a small eps (readings).  Returns (q, k, log_alpha, beta) as float64 arrays."""
    q, k = _f64(q_raw), _f64(k_raw)
    a, b = _f64(a_raw), _f64(b_raw)
    A, dtb = _f64(A_log), _f64(dt_bias)
    q = q / np.sqrt((q * q).sum(-1, keepdims=True) + eps)
    k = k / np.sqrt((k * k).sum(-1, keepdims=True) + eps)
    x = a + dtb
    softplus = np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))   # log(1 + e^x), stable
    log_alpha = -np.exp(A) * softplus
    beta = 1.0 / (1.0 + np.exp(-b))
    return q, k, log_alpha, beta


def recurrence_bwd_np(q, k, v, log_alpha, beta, d, S0=None, dout=None, dS_final=None,
                      checkpoint: int = 64):
    """Gradients of the token-by-token recurrence, float64 (reverse-mode through the
    definition, one token at a time).  The loss is <dout, out> + <dS_final, S_final>
    (either cotangent may be None = 0).  The pages give no backward formulas (the
    write-up's section "硬件高效的分块并行计算" says only that the backward pass
    reuses the cached inverse and chunk states); these are the adjoint of

        S_t = alpha_t S_{t-1} - beta_t (S_{t-1} k_t) k_t^T + beta_t v_t k_t^T
        o_t = S_t qt_t,   qt_t = q_t - d_h k_t,   alpha_t = exp(log_alpha_t).

    Going backwards with G = dL/dS_t (the future's gradient plus dout_t qt_t^T),
    p = S_{t-1} k_t and u = G k_t:

        dqt_t = S_t^T dout_t            dq_t = dqt_t,  dd_h -= dqt_t . k_t
        dlog_alpha_t = alpha_t <G, S_{t-1}>
        dbeta_t = u . (v_t - p)         dv_t = beta_t u
        dk_t = beta_t (G^T (v_t - p) - S_{t-1}^T u) - d_h dqt_t
        dL/dS_{t-1} = alpha_t G - beta_t u k_t^T

    States S_{t-1} are recomputed forward from checkpoints every ``checkpoint``
    tokens.  Returns a dict of float64 arrays: dq, dk [B,T,H,dk], dv [B,T,H,dv],
    dlog_alpha, dbeta [B,T,H], dd [H], dS0 [B,H,dv,dk]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be, d = _f64(log_alpha), _f64(beta), _f64(d)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dv, dk)) if S0 is None else _f64(S0).copy()
    dO = np.zeros((B, T, H, dv)) if dout is None else _f64(dout)
    G = np.zeros((B, H, dv, dk)) if dS_final is None else _f64(dS_final).copy()
    qt = q - d[None, None, :, None] * k
    al = np.exp(la)

    def step(S, t):
        kt = k[:, t]
        Sk = np.einsum("bhij,bhj->bhi", S, kt)
        return (al[:, t][..., None, None] * S
                - be[:, t][..., None, None] * np.einsum("bhi,bhj->bhij", Sk, kt)
                + be[:, t][..., None, None] * np.einsum("bhi,bhj->bhij", v[:, t], kt))

    # forward: the state before each checkpoint block
    starts = []
    for t in range(T):
        if t % checkpoint == 0:
            starts.append(S.copy())
        S = step(S, t)
    gq = np.zeros_like(q)
    gk = np.zeros_like(k)
    gv = np.zeros_like(v)
    gla = np.zeros_like(la)
    gbe = np.zeros_like(be)
    gd = np.zeros(H)
    for blk in range(len(starts) - 1, -1, -1):
        t0, t1 = blk * checkpoint, min(T, (blk + 1) * checkpoint)
        states = [starts[blk]]                    # states[i] = S_{t0 + i - 1}
        for t in range(t0, t1):
            states.append(step(states[-1], t))
        for t in range(t1 - 1, t0 - 1, -1):
            Sp, St = states[t - t0], states[t - t0 + 1]
            kt, vt = k[:, t], v[:, t]
            G = G + np.einsum("bhi,bhj->bhij", dO[:, t], qt[:, t])
            dqt = np.einsum("bhij,bhi->bhj", St, dO[:, t])
            gq[:, t] = dqt
            gd -= np.einsum("bhj,bhj->h", dqt, kt)
            p = np.einsum("bhij,bhj->bhi", Sp, kt)
            u = np.einsum("bhij,bhj->bhi", G, kt)
            r = vt - p
            bt = be[:, t][..., None]
            gla[:, t] = al[:, t] * np.einsum("bhij,bhij->bh", G, Sp)
            gbe[:, t] = np.einsum("bhi,bhi->bh", u, r)
            gv[:, t] = bt * u
            gk[:, t] = (bt * (np.einsum("bhij,bhi->bhj", G, r) - np.einsum("bhij,bhi->bhj", Sp, u))
                        - d[None, :, None] * dqt)
            G = al[:, t][..., None, None] * G - be[:, t][..., None, None] * np.einsum("bhi,bhj->bhij", u, kt)
    return {"dq": gq, "dk": gk, "dv": gv, "dlog_alpha": gla, "dbeta": gbe, "dd": gd, "dS0": G}


def chunked_bwd_np(q, k, v, log_alpha, beta, d, S0=None, dout=None, dS_final=None, chunk: int = 32):
    """The gradients of ``recurrence_bwd_np`` through the chunk form of ``chunked_np``
    (float64, one (b, h) chain at a time; small cases).  It is not the oracle for
    the GPU; it pins the chunk adjoint the backward kernels use to the token-level
    gradients.  Per chunk (notation of ``chunked_np``; A = diag(beta) AF,
    Gamma = diag(exp g), E_rs = exp(g_r - g_s), Dc = diag(exp(g_L - g))), with dS'
    the gradient at the chunk's end state:

        dS   = exp(g_L) dS' - (dS' K^T Dc) W + dO^T (Gamma Q~ - P W)   (reverse pass)
        dX   = P^T dO + Dc K dS'^T,   dR = Tinv^T dX
        dA   = -(dR X^T) (s < r),     dP = (dO X^T) (s <= r)
        dQ~  = Gamma dO S + (dP o E) K
        dK   = (dP o E)^T Q~ - diag(beta exp g') dR S + (dY + dY^T) K + Dc X dS' - d dQ~,
               dY = dA o (beta_r exp(g'_r - g_s))
        dV   = diag(beta) dR,  dbeta_r = dR_r . (v_r - exp(g'_r) S k_r) + sum_s dA_rs AF_rs
        dg   = every exponent's sensitivity, dlog_alpha_i = sum_{r >= i} dg_r (in the chunk)

    Returns the dict of ``recurrence_bwd_np``."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, be, d = _f64(log_alpha), _f64(beta), _f64(d)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S0 = np.zeros((B, H, dv, dk)) if S0 is None else _f64(S0)
    dO = np.zeros((B, T, H, dv)) if dout is None else _f64(dout)
    dSf = np.zeros((B, H, dv, dk)) if dS_final is None else _f64(dS_final)
    g_out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
             "dlog_alpha": np.zeros_like(la), "dbeta": np.zeros_like(be), "dd": np.zeros(H),
             "dS0": np.zeros((B, H, dv, dk))}
    for b in range(B):
        for h in range(H):
            Kc, Qc, Vc, Oc = k[b, :, h], q[b, :, h], v[b, :, h], dO[b, :, h]
            dh = d[h]
            chunks = []
            for t0 in range(0, T, chunk):      # state-independent pieces of every chunk
                t1 = min(T, t0 + chunk)
                L = t1 - t0
                K, Q, V, bt = Kc[t0:t1], Qc[t0:t1], Vc[t0:t1], be[b, t0:t1, h]
                g = np.cumsum(la[b, t0:t1, h])
                gp = np.concatenate([[0.0], g[:-1]])
                strict = np.tril(np.ones((L, L), dtype=bool), k=-1)
                incl = np.tril(np.ones((L, L), dtype=bool))
                F = np.where(strict, np.exp(np.where(strict, gp[:, None] - g[None, :], 0.0)), 0.0)
                E = np.where(incl, np.exp(np.where(incl, g[:, None] - g[None, :], 0.0)), 0.0)
                Qt = Q - dh * K
                AF = F * (K @ K.T)
                A = bt[:, None] * AF
                Tinv = np.linalg.inv(np.eye(L) + A)
                W = Tinv @ ((bt * np.exp(gp))[:, None] * K)
                Ut = Tinv @ (bt[:, None] * V)
                P = E * (Qt @ K.T)
                dec = np.exp(g[-1] - g)
                C = Oc[t0:t1].T @ (np.exp(g)[:, None] * Qt - P @ W)
                chunks.append(dict(t0=t0, t1=t1, K=K, V=V, Qt=Qt, bt=bt, g=g, gp=gp, F=F, E=E, AF=AF, A=A,
                                   Tinv=Tinv, W=W, Ut=Ut, P=P, dec=dec, C=C))
            S = S0[b, h].copy()                    # chunk-start states, in order
            starts = []
            for c in chunks:
                starts.append(S.copy())
                X = c["Ut"] - c["W"] @ S.T
                S = np.exp(c["g"][-1]) * S + X.T @ (c["dec"][:, None] * c["K"])
            dS = dSf[b, h].copy()                  # end-state gradients, in reverse
            ends = [None] * len(chunks)
            for i in range(len(chunks) - 1, -1, -1):
                c = chunks[i]
                ends[i] = dS.copy()
                dS = np.exp(c["g"][-1]) * dS - ((dS @ c["K"].T) * c["dec"][None, :]) @ c["W"] + c["C"]
            g_out["dS0"][b, h] = dS
            for c, S, dSp in zip(chunks, starts, ends):
                t0, t1 = c["t0"], c["t1"]
                K, V, Qt, bt, g, gp = c["K"], c["V"], c["Qt"], c["bt"], c["g"], c["gp"]
                A, AF, F, E, Tinv, P, dec = c["A"], c["AF"], c["F"], c["E"], c["Tinv"], c["P"], c["dec"]
                O = Oc[t0:t1]
                KS = K @ S.T
                Rv = V - np.exp(gp)[:, None] * KS
                X = Tinv @ (bt[:, None] * Rv)
                dX = P.T @ O + dec[:, None] * (K @ dSp.T)
                dR = Tinv.T @ dX
                dA = -np.tril(dR @ X.T, -1)
                dP = np.tril(O @ X.T)
                dZ = dP * E
                dY = dA * bt[:, None] * F
                GdOS = np.exp(g)[:, None] * (O @ S)
                dQt = GdOS + dZ @ K
                Fm = dec[:, None] * (X @ dSp)
                dK = dZ.T @ Qt - (bt * np.exp(gp))[:, None] * (dR @ S) + (dY + dY.T) @ K + Fm - dh * dQt
                g_out["dq"][b, t0:t1, h] = dQt
                g_out["dk"][b, t0:t1, h] = dK
                g_out["dv"][b, t0:t1, h] = bt[:, None] * dR
                g_out["dbeta"][b, t0:t1, h] = (dR * Rv).sum(1) + (dA * AF).sum(1)
                f = (Fm * K).sum(1)
                dg = (dP * P).sum(1) - (dP * P).sum(0) + (Qt * GdOS).sum(1) - (dA * A).sum(0) - f
                dgp = -bt * (dR * (np.exp(gp)[:, None] * KS)).sum(1) + (dA * A).sum(1)
                dg[:-1] += dgp[1:]                 # the sensitivity to g_{r-1} moves onto g_{r-1}
                dg[-1] += f.sum() + np.exp(g[-1]) * (dSp * S).sum()
                g_out["dlog_alpha"][b, t0:t1, h] = np.cumsum(dg[::-1])[::-1]
                g_out["dd"][h] -= (dQt * K).sum()
    return g_out
