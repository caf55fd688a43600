"""The float64 oracle against what the recurrence's definition and mathematics fix
(CPU only).  See ``tests/pins.py`` for where each pinned value comes from."""
import numpy as np
import pytest

import oracle
from comba_workloads import CONFIGS, make_chunk_inputs
from tests import pins


def _np_chunked(chunk):
    def fn(q, k, v, log_alpha, beta, d, S0=None, beta_write=None):
        assert beta_write is None
        return oracle.chunked_np(q, k, v, log_alpha, beta, d, S0, chunk=chunk)
    return fn


ORACLES = {
    "c": oracle.recurrence,
    "numpy": oracle.recurrence_np,
}


@pytest.mark.parametrize("impl", sorted(ORACLES))
@pytest.mark.parametrize("pin", sorted(pins.BATTERY))
def test_oracle_pin(impl, pin):
    check, tol = pins.BATTERY[pin]
    assert check(ORACLES[impl]) <= tol


@pytest.mark.parametrize("chunk", [1, 2, 3, 16])
@pytest.mark.parametrize("pin", ["handworked", "handworked_embedded", "beta_zero",
                                 "bruteforce_products", "single_token", "projection_overwrite"])
def test_chunked_formulation_pins(pin, chunk):
    check, tol = pins.BATTERY[pin]
    assert check(_np_chunked(chunk)) <= 1e-12


@pytest.mark.parametrize("chunk", [1, 5, 16, 32, 64, 200])
def test_chunked_matches_recurrence(chunk):
    """The chunk algebra (one triangular inverse per chunk) reproduces the
    recurrence for every chunk size, including a ragged last chunk and C >= T."""
    rng = np.random.default_rng(10 + chunk)
    x = pins.rand_inputs(rng, B=2, T=77, H=2, dk=16, dv=12, la=(-1.5, -0.001))
    o1, S1 = oracle.recurrence(**x)
    o2, S2 = oracle.chunked_np(**x, chunk=chunk)
    assert np.max(np.abs(o1 - o2)) < 1e-12
    assert np.max(np.abs(S1 - S2)) < 1e-12


def test_c_matches_numpy_on_workload_shapes():
    cfg = CONFIGS["layer340m_bf16"].replace(B=1, H=2, T=96, dk=32, dv=16)
    x = make_chunk_inputs(cfg)
    o1, S1 = oracle.recurrence(**x)
    o2, S2 = oracle.recurrence_np(**x)
    assert np.max(np.abs(o1 - o2)) < 1e-13
    assert np.max(np.abs(S1 - S2)) < 1e-13


def test_state_split_equals_one_call():
    """Running [0, t) then [t, T) with S_final -> S0 equals one call over [0, T)."""
    rng = np.random.default_rng(20)
    x = pins.rand_inputs(rng, B=2, T=40, H=2, dk=8, dv=8)
    o, S = oracle.recurrence(**x)
    for cut in (1, 17, 39):
        a = {kk: (vv[:, :cut] if kk in ("q", "k", "v", "log_alpha", "beta") else vv) for kk, vv in x.items()}
        b = {kk: (vv[:, cut:] if kk in ("q", "k", "v", "log_alpha", "beta") else vv) for kk, vv in x.items()}
        oa, Sa = oracle.recurrence(**a)
        b["S0"] = Sa
        ob, Sb = oracle.recurrence(**b)
        assert np.max(np.abs(np.concatenate([oa, ob], axis=1) - o)) < 1e-13
        assert np.max(np.abs(Sb - S)) < 1e-13


def test_linear_in_v_and_S0_affine_in_d():
    rng = np.random.default_rng(21)
    x = pins.rand_inputs(rng, B=1, T=30, H=2, dk=8, dv=6)
    o, S = oracle.recurrence(**x)
    lam = -2.5
    y = dict(x, v=lam * x["v"], S0=lam * x["S0"])
    o2, S2 = oracle.recurrence(**y)
    assert np.max(np.abs(o2 - lam * o)) < 1e-12 and np.max(np.abs(S2 - lam * S)) < 1e-12
    # o(d) = o(0) - d * S_t k_t, and the state does not depend on d.
    z = dict(x, d=np.zeros_like(x["d"]))
    o0, Sz = oracle.recurrence(**z)
    assert np.max(np.abs(Sz - S)) < 1e-14
    # S_t k_t from the d = 0 run with q := k
    w = dict(z, q=x["k"])
    okk, _ = oracle.recurrence(**w)
    want = o0 - x["d"][None, None, :, None] * okk
    assert np.max(np.abs(o - want)) < 1e-12


def test_decode_steps_equal_chunk_recurrence():
    """Single-token steps applied in order equal one recurrence over the sequence."""
    rng = np.random.default_rng(22)
    x = pins.rand_inputs(rng, B=2, T=6, H=3, dk=8, dv=4)
    o, S = oracle.recurrence(**x)
    steps = [{"q": x["q"][:, t], "k": x["k"][:, t], "v": x["v"][:, t],
              "log_alpha": x["log_alpha"][:, t], "beta": x["beta"][:, t]} for t in range(6)]
    outs, S2 = oracle.decode_steps(steps, x["d"], x["S0"])
    assert np.max(np.abs(np.stack(outs, axis=1) - o)) < 1e-13
    assert np.max(np.abs(S2 - S)) < 1e-13


def test_state_stays_bounded_under_slow_decay():
    """With unit keys and 0 < beta < 1, |alpha - beta| < 1 along the key, so the
    state norm stays bounded over a long slow-decay run (long-context gates)."""
    cfg = CONFIGS["long64k_bf16"].replace(B=1, H=2, T=4096, dk=16, dv=16)
    x = make_chunk_inputs(cfg)
    o, S = oracle.recurrence(**x)
    assert np.isfinite(o).all() and np.isfinite(S).all()
    # bound: |S_T|_F <= |S0|_F + sum_t beta_t |v_t| (each step is a contraction plus a write)
    bound = np.linalg.norm(x["S0"].double().numpy()) + float(
        (x["beta"].double() * x["v"].double().norm(dim=-1)).sum())
    assert np.linalg.norm(S) <= bound
    assert np.linalg.norm(S) < 200.0


def test_gate_inputs_closed_forms():
    # hand values: softplus(0) = ln 2, sigmoid(0) = 1/2, exp(A_log = ln 3) = 3;
    # a 3-4-0 row normalises to 0.6, 0.8 (eps negligible)
    q = np.zeros((1, 2, 1, 3)); q[0, 0, 0] = [3.0, 4.0, 0.0]; q[0, 1, 0] = [0.0, 0.0, -2.0]
    k = 2.0 * q
    a = np.array([[[0.0], [25.0]]]); b = np.array([[[0.0], [np.log(3.0)]]])
    qn, kn, la, be = oracle.gate_inputs(q, k, a, b, np.array([np.log(3.0)]), np.array([0.0]), eps=0.0)
    np.testing.assert_allclose(qn[0, 0, 0], [0.6, 0.8, 0.0], rtol=1e-15)
    np.testing.assert_allclose(kn[0, 1, 0], [0.0, 0.0, -1.0], rtol=1e-15)
    np.testing.assert_allclose(la[0, 0, 0], -3.0 * np.log(2.0), rtol=1e-15)
    np.testing.assert_allclose(la[0, 1, 0], -3.0 * 25.0, rtol=1e-10)     # softplus(25) = 25 + O(e^-25)
    np.testing.assert_allclose(be[0, :, 0], [0.5, 0.75], rtol=1e-15)


def test_gate_inputs_norms_and_softplus_tails():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 5, 3, 16)); k = rng.standard_normal((2, 5, 3, 16))
    qn, kn, _, _ = oracle.gate_inputs(q, k, np.zeros((2, 5, 3)), np.zeros((2, 5, 3)),
                                      np.zeros(3), np.zeros(3), eps=0.0)
    np.testing.assert_allclose(np.linalg.norm(qn, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(kn, axis=-1), 1.0, rtol=1e-14)
    # softplus stays log(1 + e^x) for large and very negative arguments
    x = np.array([[[25.0], [-30.0]]])
    _, _, la, _ = oracle.gate_inputs(np.ones((1, 2, 1, 2)), np.ones((1, 2, 1, 2)), x, np.zeros((1, 2, 1)),
                                     np.zeros(1), np.zeros(1))
    # log(1 + e^x) = x + e^-x - e^-2x / 2 + ... for x = 25, and e^x - e^2x / 2 + ... for x = -30
    want = [25.0 + np.exp(-25.0) - np.exp(-50.0) / 2, np.exp(-30.0) - np.exp(-60.0) / 2]
    np.testing.assert_allclose(-la[0, :, 0], want, rtol=1e-15)


def test_gate_inputs_match_the_input_modules_decay_draws():
    # the chunk workloads draw log a = -softplus(N(0,1)) * exp(U(-4,-1)) per head: the same
    # form with A_log = that per-head log scale and dt_bias = 0
    rng = np.random.default_rng(4)
    z = rng.standard_normal((1, 7, 2)); A_log = np.array([-4.0, -1.5])
    _, _, la, _ = oracle.gate_inputs(np.ones((1, 7, 2, 4)), np.ones((1, 7, 2, 4)), z, z, A_log, np.zeros(2))
    np.testing.assert_allclose(la, -np.log1p(np.exp(z)) * np.exp(A_log), rtol=1e-14)
