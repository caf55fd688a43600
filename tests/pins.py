"""Pins for the float64 oracle: results the recurrence must reproduce that do not
come from the oracle itself.

Each ``check_*`` takes a function with the oracle's signature
``fn(q, k, v, log_alpha, beta, d, S0=None, beta_write=None) -> (out, S_final)``
and returns the largest deviation from the independently known result, so the
same battery runs against the real oracle and against deliberately broken
copies of it (the mutation test shows every planted mistake is caught).

Sources of the pinned values:
* the hand-worked three-token example in ``tests/golden``;
* closed forms: beta = 0 leaves only the scalar decay of S0; an erase
  coefficient of 0 turns the recurrence into causal gated linear attention
  (a masked matrix product); alpha = beta = 1 with orthonormal keys makes every
  write an exact projection overwrite;
* brute force: the state as explicit products of the dense per-token
  transition matrices (alpha_t I - beta_t k_t k_t^T).
"""
from __future__ import annotations

import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "comba_handworked_dk2_T3.txt")


def load_handworked():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *nums = line.split()
            vals[key] = np.array([float(x) for x in nums])
    T, dk, dv = 3, 2, 2
    ex = {
        "q": vals["q"].reshape(1, T, 1, dk),
        "k": vals["k"].reshape(1, T, 1, dk),
        "v": vals["v"].reshape(1, T, 1, dv),
        "log_alpha": np.log(vals["alpha"]).reshape(1, T, 1),
        "beta": vals["beta"].reshape(1, T, 1),
        "d": vals["d"].reshape(1),
        "S0": vals["S0"].reshape(1, 1, dv, dk),
    }
    want = {"out": vals["out"].reshape(1, T, 1, dv), "S_final": vals["S_final"].reshape(1, 1, dv, dk)}
    return ex, want


def rand_inputs(rng, B=2, T=9, H=3, dk=5, dv=4, s0=0.5, la=(-0.3, -0.01)):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    return {
        "q": q, "k": k, "v": rng.standard_normal((B, T, H, dv)),
        "log_alpha": rng.uniform(la[0], la[1], (B, T, H)),
        "beta": 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H)))),
        "d": rng.uniform(0, 1, (H,)),
        "S0": s0 * rng.standard_normal((B, H, dv, dk)) if s0 else None,
    }


def _err(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) if np.size(a) else 0.0


def check_handworked(fn):
    ex, want = load_handworked()
    out, S = fn(**ex)
    return max(_err(out, want["out"]), _err(S, want["S_final"]))


def check_handworked_embedded(fn, seed=0):
    """The hand example placed at (b=1, h=1) of a B=2, H=2 batch: pins the
    [B,T,H,*] input layout, the [B,H,dv,dk] state layout and per-head d."""
    rng = np.random.default_rng(seed)
    ex, want = load_handworked()
    x = rand_inputs(rng, B=2, T=3, H=2, dk=2, dv=2)
    for key in ("q", "k", "v"):
        x[key][1, :, 1] = ex[key][0, :, 0]
    x["log_alpha"][1, :, 1] = ex["log_alpha"][0, :, 0]
    x["beta"][1, :, 1] = ex["beta"][0, :, 0]
    x["d"][1] = ex["d"][0]
    x["S0"][1, 1] = ex["S0"][0, 0]
    out, S = fn(**x)
    return max(_err(out[1, :, 1], want["out"][0, :, 0]), _err(S[1, 1], want["S_final"][0, 0]))


def check_beta_zero(fn, seed=1):
    """beta = 0: S_t = exp(G_t) S0 and o_t = exp(G_t) S0 (q_t - d k_t), G_t = sum_{i<=t} log a_i."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng)
    x["beta"] = np.zeros_like(x["beta"])
    out, S = fn(**x)
    G = np.cumsum(x["log_alpha"], axis=1)                           # [B,T,H]
    qt = x["q"] - x["d"][None, None, :, None] * x["k"]
    want = np.exp(G)[..., None] * np.einsum("bhij,bthj->bthi", x["S0"], qt)
    Sw = np.exp(G[:, -1])[..., None, None] * x["S0"]
    return max(_err(out, want), _err(S, Sw))


def gated_linear_attention(x, bw):
    """Causal gated linear attention with output correction, as a masked matrix
    product: o_t = sum_{s<=t} e^{G_t-G_s} bw_s v_s (k_s . qt_t) + e^{G_t} S0 qt_t."""
    G = np.cumsum(x["log_alpha"], axis=1)                           # [B,T,H]
    T = G.shape[1]
    qt = x["q"] - x["d"][None, None, :, None] * x["k"]
    scores = np.einsum("bthj,bshj->bhts", qt, x["k"])               # qt_t . k_s
    decay = np.exp(G.transpose(0, 2, 1)[..., :, None] - G.transpose(0, 2, 1)[..., None, :])
    mask = np.tril(np.ones((T, T), dtype=bool))
    Wm = np.where(mask, decay * scores, 0.0) * bw.transpose(0, 2, 1)[..., None, :]
    o = np.einsum("bhts,bshi->bthi", Wm, x["v"])
    if x.get("S0") is not None:
        o = o + np.exp(G)[..., None] * np.einsum("bhij,bthj->bthi", x["S0"], qt)
    Gl = G[:, -1]                                                    # [B,H]
    wS = np.exp(Gl[:, None, :] - G) * bw                             # [B,T,H]
    S = np.einsum("bth,bthi,bthj->bhij", wS, x["v"], x["k"])
    if x.get("S0") is not None:
        S = S + np.exp(Gl)[..., None, None] * x["S0"]
    return o, S


def check_linear_attention_exact(fn, seed=2):
    """Erase coefficient 0, write coefficient beta: exactly gated linear attention."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, T=11)
    bw = x["beta"].copy()
    x_call = dict(x)
    x_call["beta"] = np.zeros_like(bw)
    out, S = fn(**x_call, beta_write=bw)
    o_want, S_want = gated_linear_attention(x, bw)
    return max(_err(out, o_want), _err(S, S_want))


def check_linear_attention_limit(fn, seed=3, eps=1e-7):
    """Tied beta = eps, alpha = 1, S0 = 0: out/eps -> causal linear attention,
    with an O(eps * t) remainder."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, T=12, s0=0)
    x["log_alpha"] = np.zeros_like(x["log_alpha"])
    x["beta"] = np.full_like(x["beta"], eps)
    out, S = fn(**x)
    o_want, S_want = gated_linear_attention(x, np.ones_like(x["beta"]))
    return max(_err(out / eps, o_want), _err(S / eps, S_want))


def check_projection_overwrite(fn, seed=4):
    """alpha = beta = 1 with orthonormal keys: each write replaces the state's
    read-out at its key, S_t k_s = v_s for all s <= t, and
    S_T = S0 (I - sum k k^T) + sum v k^T."""
    rng = np.random.default_rng(seed)
    B, H, T, dk, dv = 1, 2, 5, 6, 3
    x = rand_inputs(rng, B=B, T=T, H=H, dk=dk, dv=dv)
    for h in range(H):
        Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
        x["k"][0, :, h] = Qm[:, :T].T
    x["log_alpha"] = np.zeros_like(x["log_alpha"])
    x["beta"] = np.ones_like(x["beta"])
    worst = 0.0
    for t in range(1, T + 1):
        xt = {kk: (vv[:, :t] if kk in ("q", "k", "v", "log_alpha", "beta") else vv) for kk, vv in x.items()}
        _, S = fn(**xt)
        for h in range(H):
            for s in range(t):
                worst = max(worst, _err(S[0, h] @ x["k"][0, s, h], x["v"][0, s, h]))
    for h in range(H):
        Kh, Vh = x["k"][0, :, h], x["v"][0, :, h]
        Sw = x["S0"][0, h] @ (np.eye(dk) - Kh.T @ Kh) + Vh.T @ Kh
        worst = max(worst, _err(S[0, h], Sw))
    return worst


def check_bruteforce_products(fn, seed=5, T=7):
    """Dense transition products: with M_t = a_t I - beta_t k_t k_t^T,
    S_t = S0 M_1..M_t + sum_{s<=t} beta_s v_s k_s^T M_{s+1}..M_t and o_t = S_t (q_t - d k_t)."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, B=1, T=T, H=2, dk=4, dv=3)
    out, S = fn(**x)
    worst = 0.0
    for h in range(2):
        dk = x["k"].shape[-1]
        M = [np.exp(x["log_alpha"][0, t, h]) * np.eye(dk)
             - x["beta"][0, t, h] * np.outer(x["k"][0, t, h], x["k"][0, t, h]) for t in range(T)]
        for t in range(T):
            P = np.eye(dk)
            for r in range(t + 1):
                P = P @ M[r]
            St = x["S0"][0, h] @ P
            for s in range(t + 1):
                R = np.eye(dk)
                for r in range(s + 1, t + 1):
                    R = R @ M[r]
                St = St + x["beta"][0, s, h] * np.outer(x["v"][0, s, h], x["k"][0, s, h]) @ R
            qt = x["q"][0, t, h] - x["d"][h] * x["k"][0, t, h]
            worst = max(worst, _err(out[0, t, h], St @ qt))
        worst = max(worst, _err(S[0, h], St))
    return worst


def check_single_token(fn, seed=6):
    """T = 1 from S0 = 0: o = beta v (k . (q - d k))."""
    rng = np.random.default_rng(seed)
    x = rand_inputs(rng, T=1, s0=0)
    out, S = fn(**x)
    qt = x["q"] - x["d"][None, None, :, None] * x["k"]
    kq = np.sum(x["k"] * qt, axis=-1)                                # [B,1,H]
    want = (x["beta"] * kq)[..., None] * x["v"]
    Sw = np.einsum("bh,bhi,bhj->bhij", x["beta"][:, 0], x["v"][:, 0], x["k"][:, 0])
    return max(_err(out, want), _err(S, Sw))


BATTERY = {
    "handworked": (check_handworked, 1e-13),
    "handworked_embedded": (check_handworked_embedded, 1e-13),
    "beta_zero": (check_beta_zero, 1e-13),
    "linear_attention_exact": (check_linear_attention_exact, 1e-12),
    "linear_attention_limit": (check_linear_attention_limit, 1e-4),
    "projection_overwrite": (check_projection_overwrite, 1e-12),
    "bruteforce_products": (check_bruteforce_products, 1e-12),
    "single_token": (check_single_token, 1e-14),
}
