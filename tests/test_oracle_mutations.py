"""Plants plausible mistakes in copies of the oracle's token step (on the CPU) and
checks that the pin battery catches every one of them."""
import numpy as np
import pytest

from tests import pins


def _mutant(kind):
    def fn(q, k, v, log_alpha, beta, d, S0=None, beta_write=None):
        q, k, v = map(np.asarray, (q, k, v))
        bw = beta if beta_write is None else beta_write
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        S = np.zeros((B, H, dv, dk)) if S0 is None else np.array(S0, dtype=float)
        out = np.empty((B, T, H, dv))
        for t in range(T):
            kt, qv, vt = k[:, t], q[:, t], v[:, t]
            a = np.exp(log_alpha[:, t])[..., None, None]
            be = beta[:, max(t - 1, 0)] if kind == "beta_shift" else beta[:, t]
            be = be[..., None, None]
            w = bw[:, t][..., None, None]
            Sk = np.einsum("bhij,bhj->bhi", S, kt)
            if kind == "transposed_readout" and dk == dv:
                Sk = np.einsum("bhji,bhj->bhi", S, kt)
            erase = be * np.einsum("bhi,bhj->bhij", Sk, kt)
            write = w * np.einsum("bhi,bhj->bhij", vt, kt)
            S_prev = S
            if kind == "iplr":            # decay also on the erase term
                S = a * (S - erase) + write
            elif kind == "no_erase":
                S = a * S + write
            elif kind == "decayed_write":
                S = a * S - erase + a * write
            elif kind == "erase_sign":
                S = a * S + erase + write
            else:
                S = a * S - erase + write
            sign = -1.0
            if kind == "d_sign":
                sign = 1.0
            dd = d[None, :, None]
            if kind == "no_correction":
                dd = 0.0 * dd
            qt = qv + sign * dd * kt
            Sout = S_prev if kind == "pre_update_output" else S
            out[:, t] = np.einsum("bhij,bhj->bhi", Sout, qt)
        return out, S
    return fn


MUTANTS = ["iplr", "no_erase", "decayed_write", "erase_sign", "d_sign", "no_correction",
           "pre_update_output", "beta_shift", "transposed_readout"]


def test_unmutated_copy_passes():
    fn = _mutant("none")
    for name, (check, tol) in pins.BATTERY.items():
        assert check(fn) <= tol, name


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_mistake_is_caught(kind):
    fn = _mutant(kind)
    caught = [name for name, (check, tol) in pins.BATTERY.items() if not check(fn) <= tol]
    assert caught, f"no pin catches the '{kind}' mistake"
