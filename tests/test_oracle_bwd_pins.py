"""The oracle's gradients (``oracle.recurrence_bwd_np``) against what fixes them
independently of its own formulas (CPU only):

* central finite differences of the forward recurrence (the C oracle, itself
  pinned by the forward battery), every input element of small cases;
* reverse-mode differentiation by torch.autograd of the recurrence written as a
  plain float64 token loop;
* a closed form: with beta = 0 the state only decays, S_T = (prod alpha) S0;
* plausible mistakes planted in copies of the backward (source edits, CPU) are
  each caught by one of the above."""
import inspect

import numpy as np
import pytest
import torch

import oracle

NAMES = ("q", "k", "v", "log_alpha", "beta", "d", "S0")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dd", "dS0")


def _case(seed, B=1, T=7, H=2, dk=3, dv=2):
    rng = np.random.default_rng(seed)
    k = rng.normal(size=(B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    x = dict(q=rng.normal(size=(B, T, H, dk)), k=k, v=rng.normal(size=(B, T, H, dv)),
             log_alpha=-rng.uniform(0.0, 0.6, size=(B, T, H)), beta=rng.uniform(0.0, 1.0, size=(B, T, H)),
             d=rng.uniform(0.0, 1.0, size=H), S0=rng.normal(size=(B, H, dv, dk)))
    cot = dict(dout=rng.normal(size=(B, T, H, dv)), dS_final=rng.normal(size=(B, H, dv, dk)))
    return x, cot


def _loss(x, cot):
    o, S = oracle.recurrence(**x)
    return float((o * cot["dout"]).sum() + (S * cot["dS_final"]).sum())


def pin_finite_differences(bwd, seed=0, checkpoint=3, **shape):
    """Largest error of the gradients against central differences (step 1e-6),
    relative to the largest gradient entry."""
    x, cot = _case(seed, **shape)
    g = bwd(**x, **cot, checkpoint=checkpoint)
    worst = 0.0
    for name, gname in zip(NAMES, GRADS):
        a = x[name]
        fd = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            xp, xm = dict(x), dict(x)
            xp[name] = a.copy(); xp[name][idx] += 1e-6
            xm[name] = a.copy(); xm[name][idx] -= 1e-6
            fd[idx] = (_loss(xp, cot) - _loss(xm, cot)) / 2e-6
        worst = max(worst, np.abs(fd - g[gname]).max() / max(np.abs(fd).max(), 1e-30))
    return worst


def pin_autograd(bwd, seed=1, B=2, T=20, H=2, dk=4, dv=3):
    x, cot = _case(seed, B=B, T=T, H=H, dk=dk, dv=dv)
    t = {n: torch.tensor(x[n], dtype=torch.float64, requires_grad=True) for n in NAMES}
    S = t["S0"]
    outs = []
    for i in range(T):
        kt, vt = t["k"][:, i], t["v"][:, i]
        a = torch.exp(t["log_alpha"][:, i])[..., None, None]
        b = t["beta"][:, i][..., None, None]
        Sk = (S @ kt[..., None])                       # [B,H,dv,1]
        S = a * S - b * Sk @ kt[..., None, :] + b * vt[..., :, None] @ kt[..., None, :]
        qt = t["q"][:, i] - t["d"][None, :, None] * kt
        outs.append((S @ qt[..., None])[..., 0])
    out = torch.stack(outs, 1)
    L = (out * torch.tensor(cot["dout"])).sum() + (S * torch.tensor(cot["dS_final"])).sum()
    L.backward()
    g = bwd(**x, **cot, checkpoint=8)
    return max(np.abs(t[n].grad.numpy() - g[gn]).max() / np.abs(t[n].grad.numpy()).max()
               for n, gn in zip(NAMES, GRADS))


def pin_beta_zero(bwd, seed=2, B=1, T=5, H=2, dk=3, dv=2):
    """beta = 0, dout = 0: S_t = A_t S0 with A_t = prod_{i<=t} alpha_i, so
    dS0 = A_T dS_final, dlog_alpha_t = A_T <dS_final, S0> for every t,
    dbeta_t = (A_T / A_t) (dS_final k_t) . (v_t - A_{t-1} S0 k_t), and dq = dk = dv = 0."""
    x, cot = _case(seed, B=B, T=T, H=H, dk=dk, dv=dv)
    x["beta"] = np.zeros_like(x["beta"])
    cot["dout"] = np.zeros_like(cot["dout"])
    g = bwd(**x, **cot, checkpoint=2)
    A = np.exp(np.cumsum(x["log_alpha"], axis=1))                       # [B,T,H]
    AT = A[:, -1]
    Aprev = np.concatenate([np.ones_like(A[:, :1]), A[:, :-1]], axis=1)
    dSf, S0 = cot["dS_final"], x["S0"]
    e = [np.abs(g["dS0"] - AT[..., None, None] * dSf).max(),
         np.abs(g["dlog_alpha"] - (AT * np.einsum("bhij,bhij->bh", dSf, S0))[:, None]).max(),
         np.abs(g["dq"]).max(), np.abs(g["dk"]).max(), np.abs(g["dv"]).max(), np.abs(g["dd"]).max()]
    for t in range(T):
        kt, vt = x["k"][:, t], x["v"][:, t]
        u = (AT / A[:, t])[..., None] * np.einsum("bhij,bhj->bhi", dSf, kt)
        p = Aprev[:, t][..., None] * np.einsum("bhij,bhj->bhi", S0, kt)
        e.append(np.abs(g["dbeta"][:, t] - np.einsum("bhi,bhi->bh", u, vt - p)).max())
    return max(e)


BATTERY = {
    "finite_differences": (pin_finite_differences, 1e-6),
    "finite_differences_B2_ragged": (lambda f: pin_finite_differences(f, seed=3, checkpoint=4, B=2, T=6), 1e-6),
    "autograd": (pin_autograd, 1e-11),
    "beta_zero": (pin_beta_zero, 1e-12),
}


@pytest.mark.parametrize("pin", sorted(BATTERY))
def test_backward_pin(pin):
    check, tol = BATTERY[pin]
    assert check(oracle.recurrence_bwd_np) <= tol


def test_checkpoint_spacing_does_not_change_the_result():
    x, cot = _case(5, B=2, T=13, H=3, dk=4, dv=5)
    ref = oracle.recurrence_bwd_np(**x, **cot, checkpoint=64)
    for c in (1, 4, 13):
        g = oracle.recurrence_bwd_np(**x, **cot, checkpoint=c)
        for n in GRADS:
            assert np.array_equal(g[n], ref[n]), (c, n)


def test_missing_cotangents_are_zero():
    x, cot = _case(6)
    g = oracle.recurrence_bwd_np(**x, dout=cot["dout"], dS_final=None)
    h = oracle.recurrence_bwd_np(**x, dout=cot["dout"], dS_final=np.zeros_like(cot["dS_final"]))
    assert all(np.array_equal(g[n], h[n]) for n in GRADS)


# plausible mistakes, planted in copies of the backward's source
MUTANTS = {
    "dk_erase_sign": ('- np.einsum("bhij,bhi->bhj", Sp, u))', '+ np.einsum("bhij,bhi->bhj", Sp, u))'),
    "no_d_term_in_dk": ("- d[None, :, None] * dqt)", ")"),
    "dlog_alpha_new_state": ('np.einsum("bhij,bhij->bh", G, Sp)', 'np.einsum("bhij,bhij->bh", G, St)'),
    "dbeta_without_erase": ("r = vt - p", "r = vt"),
    "adjoint_without_erase": ('- be[:, t][..., None, None] * np.einsum("bhi,bhj->bhij", u, kt)', ""),
    "dq_from_previous_state": ('dqt = np.einsum("bhij,bhi->bhj", St, dO[:, t])',
                               'dqt = np.einsum("bhij,bhi->bhj", Sp, dO[:, t])'),
    "dd_sign": ("gd -= ", "gd += "),
}


def _mutant(kind):
    src = inspect.getsource(oracle.recurrence_bwd_np)
    old, new = MUTANTS[kind]
    assert src.count(old) == 1, kind
    ns = dict(oracle.__dict__)
    exec(compile(src.replace(old, new), f"<mutant {kind}>", "exec"), ns)
    return ns["recurrence_bwd_np"]


@pytest.mark.parametrize("kind", sorted(MUTANTS))
def test_planted_backward_mistake_is_caught(kind):
    fn = _mutant(kind)
    caught = [n for n, (check, tol) in BATTERY.items() if not check(fn) <= tol]
    assert caught, f"no pin catches the '{kind}' mistake"


@pytest.mark.parametrize("T,chunk,dk,dv", [(37, 8, 5, 4), (64, 16, 8, 6), (50, 64, 4, 4), (1, 4, 3, 3),
                                           (17, 1, 3, 2), (70, 32, 6, 5)])
def test_chunked_backward_matches_token_backward(T, chunk, dk, dv):
    """The chunk adjoint (the form the backward kernels compute) against the token
    gradients, ragged last chunks and chunk length 1 included."""
    x, cot = _case(40 + T, B=2, T=T, H=2, dk=dk, dv=dv)
    ref = oracle.recurrence_bwd_np(**x, **cot)
    g = oracle.chunked_bwd_np(**x, **cot, chunk=chunk)
    for n in GRADS:
        err = np.abs(g[n] - ref[n]).max() / max(np.abs(ref[n]).max(), 1e-30)
        assert err <= 1e-12, (n, err)


def test_chunked_backward_without_state_inputs():
    x, cot = _case(77, B=1, T=40, H=1, dk=4, dv=3)
    x["S0"] = None
    ref = oracle.recurrence_bwd_np(**x, dout=cot["dout"], dS_final=None)
    g = oracle.chunked_bwd_np(**x, dout=cot["dout"], dS_final=None, chunk=32)
    for n in GRADS:
        assert np.allclose(g[n], ref[n], rtol=1e-12, atol=1e-12), n
