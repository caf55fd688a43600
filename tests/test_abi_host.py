"""The C ABI library on the host: it loads without a GPU, exports every function
the public header declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import chunk_delta_rule_b200 as cdr
from chunk_delta_rule_b200 import build as cbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "comba.h")


@pytest.fixture(scope="module")
def lib():
    cbuild.build()
    return cdr.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(comba_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("comba_chunk_fwd", "comba_chunk_fwd_f32", "comba_recurrent_step",
              "comba_get_last_error", "comba_status_string", "comba_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(cdr.EXPORTS)


def test_version_and_status_strings(lib):
    assert lib.comba_version() == 100
    assert cdr.status_string(0) == "ok"
    for code in (-1, -2, -3, -4, -5):
        assert cdr.status_string(code) not in ("ok", "unknown status")
    assert cdr.status_string(12345) == "unknown status"


# Fake, well-aligned, non-overlapping "device" addresses: validation rejects
# before any CUDA call, so they are never dereferenced.
BASE = 1 << 40
GB = 1 << 30


def _chunk_args(**kw):
    a = dict(q=BASE, k=BASE + GB, v=BASE + 2 * GB, log_alpha=BASE + 3 * GB, beta=BASE + 4 * GB,
             d=BASE + 5 * GB, S0=BASE + 6 * GB, out=BASE + 7 * GB, S_final=BASE + 8 * GB,
             B=2, T=128, H=4, dk=64, dv=64, chunk=64)
    a.update(kw)
    return a


def _call_chunk(lib, a, f32=False):
    fn = lib.comba_chunk_fwd_f32 if f32 else lib.comba_chunk_fwd
    p = lambda x: ctypes.c_void_p(x)
    return fn(p(a["q"]), p(a["k"]), p(a["v"]), p(a["log_alpha"]), p(a["beta"]), p(a["d"]),
              p(a["S0"]), p(a["out"]), p(a["S_final"]), a["B"], a["T"], a["H"], a["dk"],
              a["dv"], a["chunk"], ctypes.c_void_p(None))


@pytest.mark.parametrize("bad", [
    dict(dk=7), dict(dk=0), dict(dk=144), dict(dv=24), dict(dv=256), dict(chunk=48),
    dict(chunk=128), dict(chunk=0), dict(B=-1), dict(T=-3), dict(H=-2),
    dict(q=None), dict(k=None), dict(v=None), dict(log_alpha=None), dict(beta=None),
    dict(d=None), dict(out=None),
    dict(q=BASE + 8), dict(out=BASE + 7 * GB + 2), dict(S0=BASE + 6 * GB + 4),
    dict(log_alpha=BASE + 3 * GB + 2),
    dict(out=BASE + 16),                  # out overlaps q
    dict(S_final=BASE + 2 * GB + 64),     # S_final overlaps v
    dict(S_final=BASE + 6 * GB + 16),     # partial overlap with S0
    dict(S_final=BASE + 7 * GB + 256),    # S_final overlaps out
])
@pytest.mark.parametrize("f32", [False, True])
def test_chunk_rejects_bad_arguments(lib, bad, f32):
    assert _call_chunk(lib, _chunk_args(**bad), f32) == -1


@pytest.mark.parametrize("empty", [dict(B=0), dict(H=0)])
def test_chunk_empty_batch_is_noop(lib, empty):
    # Nothing to compute and nothing enqueued: succeeds without a device.
    assert _call_chunk(lib, _chunk_args(**empty, q=None, k=None, v=None)) == 0


def _step_args(**kw):
    a = dict(q=BASE, k=BASE + GB, v=BASE + 2 * GB, log_alpha=BASE + 3 * GB, beta=BASE + 4 * GB,
             d=BASE + 5 * GB, S=BASE + 6 * GB, out=BASE + 7 * GB, B=4, H=2, dk=128, dv=128)
    a.update(kw)
    return a


def _call_step(lib, a):
    p = lambda x: ctypes.c_void_p(x)
    return lib.comba_recurrent_step(p(a["q"]), p(a["k"]), p(a["v"]), p(a["log_alpha"]),
                                    p(a["beta"]), p(a["d"]), p(a["S"]), p(a["out"]), a["B"],
                                    a["H"], a["dk"], a["dv"], ctypes.c_void_p(None))


@pytest.mark.parametrize("bad", [
    dict(dk=16), dict(dk=96), dict(dv=8), dict(dv=200), dict(B=-1), dict(H=-1),
    dict(S=None), dict(out=None), dict(q=None), dict(S=BASE + 6 * GB + 8),
    dict(out=BASE + 6 * GB + 64),         # out inside S
    dict(S=BASE + 512),                   # S overlaps q
])
def test_step_rejects_bad_arguments(lib, bad):
    assert _call_step(lib, _step_args(**bad)) == -1


def test_step_empty_is_noop(lib):
    assert _call_step(lib, _step_args(B=0)) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 16)
    g = torch.zeros(1, 4, 1)
    with pytest.raises(ValueError):
        cdr.chunk_fwd(x, x, x, g, g, torch.zeros(1))
    with pytest.raises(ValueError):
        cdr.chunk_bwd(x, x, x, g, g, torch.zeros(1), x)
    with pytest.raises(ValueError):   # q, k, v, dout must be bf16 or fp32
        cdr.chunk_bwd(x.double(), x, x, g, g, torch.zeros(1), x)


def _varlen_args(**kw):
    a = dict(q=BASE, k=BASE + GB, v=BASE + 2 * GB, log_alpha=BASE + 3 * GB, beta=BASE + 4 * GB,
             d=BASE + 5 * GB, S0=BASE + 6 * GB, out=BASE + 7 * GB, S_final=BASE + 8 * GB,
             cu=BASE + 9 * GB, N=3, total_T=200, H=4, Hqk=2, dk=128, dv=128, chunk=64)
    a.update(kw)
    return a


def _call_varlen(lib, a):
    p = lambda x: ctypes.c_void_p(x)
    return lib.comba_chunk_fwd_varlen(p(a["q"]), p(a["k"]), p(a["v"]), p(a["log_alpha"]),
                                      p(a["beta"]), p(a["d"]), p(a["S0"]), p(a["out"]),
                                      p(a["S_final"]), p(a["cu"]), a["N"], a["total_T"], a["H"],
                                      a["Hqk"], a["dk"], a["dv"], a["chunk"], ctypes.c_void_p(None))


@pytest.mark.parametrize("bad", [
    dict(N=-1), dict(total_T=-1), dict(H=-1), dict(Hqk=0), dict(Hqk=3), dict(Hqk=8),
    dict(dk=24), dict(chunk=48), dict(cu=None), dict(d=None), dict(q=None), dict(out=None),
    dict(cu=BASE + 9 * GB + 2),            # misaligned cu_seqlens
    dict(q=BASE + 8),                      # misaligned q
    dict(out=BASE + 9 * GB),               # out overlaps cu_seqlens
    dict(S_final=BASE + 2 * GB + 64),      # S_final overlaps v
    dict(S_final=BASE + 6 * GB + 16),      # partial overlap with S0
])
def test_varlen_rejects_bad_arguments(lib, bad):
    assert _call_varlen(lib, _varlen_args(**bad)) == -1


@pytest.mark.parametrize("empty", [dict(N=0), dict(H=0)])
def test_varlen_empty_is_noop(lib, empty):
    assert _call_varlen(lib, _varlen_args(**empty, q=None, k=None, v=None, cu=None)) == 0


def _call_step_grouped(lib, a, Hqk):
    p = lambda x: ctypes.c_void_p(x)
    return lib.comba_recurrent_step_grouped(p(a["q"]), p(a["k"]), p(a["v"]), p(a["log_alpha"]),
                                            p(a["beta"]), p(a["d"]), p(a["S"]), p(a["out"]), a["B"],
                                            a["H"], Hqk, a["dk"], a["dv"], ctypes.c_void_p(None))


@pytest.mark.parametrize("Hqk", [0, -1, 3, 4])
def test_grouped_step_rejects_bad_head_counts(lib, Hqk):
    # H = 2: Hqk must be 1 or 2
    assert _call_step_grouped(lib, _step_args(), Hqk) == -1


def test_grouped_step_empty_is_noop(lib):
    assert _call_step_grouped(lib, _step_args(B=0), 1) == 0


def _call_host(lib, a, ws, ws_bytes, slices):
    p = lambda x: ctypes.c_void_p(x)
    return lib.comba_chunk_fwd_host(p(a["q"]), p(a["k"]), p(a["v"]), p(a["log_alpha"]), p(a["beta"]),
                                    p(a["d"]), p(a["S0"]), p(a["out"]), p(a["S_final"]), a["B"], a["T"],
                                    a["H"], a["dk"], a["dv"], a["chunk"], p(ws), ws_bytes, slices,
                                    ctypes.c_void_p(None))


def test_host_entry_workspace_size_and_rejections(lib):
    a = _chunk_args()
    need = lib.comba_chunk_fwd_host_workspace_size(a["B"], a["T"], a["H"], a["dk"], a["dv"])
    bth = a["B"] * a["T"] * a["H"]
    assert need >= bth * (2 * a["dk"] + 2 * a["dv"]) * 2 + 2 * bth * 4 + 2 * a["B"] * a["H"] * a["dk"] * a["dv"] * 4
    assert lib.comba_chunk_fwd_host_workspace_size(0, 8, 2, 64, 64) == 0
    ws = BASE + 20 * GB
    assert _call_host(lib, a, ws, need - 1, 4) == -1          # workspace too small
    assert _call_host(lib, a, ws + 128, need, 4) == -1        # workspace misaligned
    assert _call_host(lib, a, None, need, 4) == -1            # no workspace
    assert _call_host(lib, a, ws, need, 0) == -1              # no slices
    assert _call_host(lib, _chunk_args(dk=24), ws, need, 4) == -1
    assert _call_host(lib, _chunk_args(out=BASE + 16), ws, need, 4) == -1   # out overlaps q


def _call_gated(lib, a, A_log, dt_bias, eps):
    p = lambda x: ctypes.c_void_p(x)
    return lib.comba_chunk_fwd_gated(p(a["q"]), p(a["k"]), p(a["v"]), p(a["log_alpha"]), p(a["beta"]),
                                     p(A_log), p(dt_bias), p(a["d"]), p(a["S0"]), p(a["out"]),
                                     p(a["S_final"]), a["B"], a["T"], a["H"], a["dk"], a["dv"],
                                     a["chunk"], ctypes.c_float(eps), ctypes.c_void_p(None))


@pytest.mark.parametrize("A_log,dt_bias,eps", [
    (None, BASE + 11 * GB, 1e-6),                     # A_log required
    (BASE + 10 * GB + 2, BASE + 11 * GB, 1e-6),       # misaligned A_log
    (BASE + 10 * GB, BASE + 11 * GB + 1, 1e-6),       # misaligned dt_bias
    (BASE + 10 * GB, BASE + 11 * GB, -1.0),           # negative eps
    (BASE + 10 * GB, BASE + 11 * GB, float("nan")),
    (BASE + 7 * GB + 64, BASE + 11 * GB, 1e-6),       # A_log inside out
])
def test_gated_rejects_bad_arguments(lib, A_log, dt_bias, eps):
    assert _call_gated(lib, _chunk_args(), A_log, dt_bias, eps) == -1


def test_gated_rejects_the_chunk_entrys_bad_arguments(lib):
    assert _call_gated(lib, _chunk_args(dk=24), BASE + 10 * GB, None, 1e-6) == -1
    assert _call_gated(lib, _chunk_args(out=BASE + 16), BASE + 10 * GB, None, 1e-6) == -1


def test_gated_empty_is_noop(lib):
    assert _call_gated(lib, _chunk_args(B=0, q=None, k=None, v=None), BASE + 10 * GB, None, 1e-6) == 0


def _bwd_args(**kw):
    a = dict(q=BASE, k=BASE + GB, v=BASE + 2 * GB, log_alpha=BASE + 3 * GB, beta=BASE + 4 * GB,
             d=BASE + 5 * GB, S0=BASE + 6 * GB, dout=BASE + 7 * GB, dS_final=BASE + 8 * GB,
             dq=BASE + 9 * GB, dk=BASE + 10 * GB, dv=BASE + 11 * GB, dlog_alpha=BASE + 12 * GB,
             dbeta=BASE + 13 * GB, dd=BASE + 14 * GB, dS0=BASE + 15 * GB,
             B=2, T=100, H=4, dk_dim=64, dv_dim=64, dtype=0, ws=BASE + 20 * GB, ws_bytes=None)
    a.update(kw)
    return a


def _call_bwd(lib, a):
    p = lambda x: ctypes.c_void_p(x)
    need = lib.comba_chunk_bwd_workspace_size(a["B"], a["T"], a["H"], a["dk_dim"], a["dv_dim"])
    nb = need if a["ws_bytes"] is None else a["ws_bytes"]
    return lib.comba_chunk_bwd(*(p(a[n]) for n in ("q", "k", "v", "log_alpha", "beta", "d", "S0", "dout",
                                                    "dS_final", "dq", "dk", "dv", "dlog_alpha", "dbeta",
                                                    "dd", "dS0")),
                               a["B"], a["T"], a["H"], a["dk_dim"], a["dv_dim"], a["dtype"], p(a["ws"]), nb,
                               ctypes.c_void_p(None))


def test_bwd_workspace_size(lib):
    # per chunk of 32 tokens: W [32, dk], U~ [32, dv], three dv x dk matrices, one dd partial
    n = 2 * 4 * 4          # B * H chains x ceil(100 / 32) chunks
    assert lib.comba_chunk_bwd_workspace_size(2, 100, 4, 64, 64) == n * (32 * 128 + 3 * 64 * 64 + 1) * 4
    assert lib.comba_chunk_bwd_workspace_size(2, 100, 4, 48, 64) == 0     # unsupported dk
    assert lib.comba_chunk_bwd_workspace_size(0, 100, 4, 64, 64) == 0


@pytest.mark.parametrize("bad", [
    dict(dk_dim=48), dict(dv_dim=16), dict(dtype=2), dict(B=-1), dict(T=-3),
    dict(q=None), dict(dout=None), dict(dq=None), dict(dbeta=None), dict(d=None),
    dict(ws=None), dict(ws_bytes=1024), dict(ws=BASE + 20 * GB + 8),
    dict(dq=BASE + 16),                    # dq overlaps q
    dict(dk=BASE + 9 * GB + 64),           # dk overlaps dq
    dict(dS0=BASE + 20 * GB + 4096),       # dS0 inside the workspace
    dict(log_alpha=BASE + 3 * GB + 2),     # fp32 array misaligned
    dict(q=BASE + 1),                      # bf16 array misaligned
    dict(dout=BASE + 7 * GB + 8),          # rows need 16-byte alignment
    dict(S0=BASE + 6 * GB + 4),
])
def test_bwd_rejects_bad_arguments(lib, bad):
    assert _call_bwd(lib, _bwd_args(**bad)) == -1


def test_bwd_too_many_chains_and_empty_batch(lib):
    assert _call_bwd(lib, _bwd_args(B=65536, H=1, T=1)) == -2
    assert _call_bwd(lib, _bwd_args(B=0, dd=None, q=None, k=None, v=None, ws=None)) == 0


def test_state_compose_rejects_bad_arguments(lib):
    p = lambda x: ctypes.c_void_p(x)
    call = lambda RM, S0, Sst, B=2, H=4, P=3: lib.comba_state_compose(p(RM), p(S0), p(Sst), B, H, P,
                                                                       ctypes.c_void_p(None))
    RM, S0, Sst = BASE, BASE + GB, BASE + 2 * GB
    assert call(RM, S0, Sst, P=0) == -1
    assert call(RM, S0, Sst, B=-1) == -1
    assert call(None, S0, Sst) == -1
    assert call(RM, S0, None) == -1
    assert call(RM + 8, S0, Sst) == -1                  # misaligned
    assert call(RM, S0, RM + 4096) == -1                # S_start inside RM
    assert call(RM, S0, S0 + 64) == -1                  # S_start overlaps S0
    assert call(None, None, None, B=0) == 0             # empty


def test_chunk_transition_rejects_bad_arguments(lib):
    p = lambda x: ctypes.c_void_p(x)

    def call(q=BASE, k=BASE + GB, v=BASE + 2 * GB, la=BASE + 3 * GB, be=BASE + 4 * GB, d=BASE + 5 * GB,
             RM=BASE + 6 * GB, B=2, T=128, H=4, dk=128, dv=128, chunk=64):
        return lib.comba_chunk_fwd_transition(p(q), p(k), p(v), p(la), p(be), p(d), p(RM), B, T, H, dk, dv,
                                              chunk, ctypes.c_void_p(None))

    assert call(B=-1) == -1
    assert call(RM=None) == -1
    assert call(RM=BASE + 6 * GB + 8) == -1          # misaligned
    assert call(q=BASE + 2) == -1                     # misaligned input
    assert call(v=None) == -1
    assert call(RM=BASE + 2 * GB + 4096) == -1       # RM inside v
    assert call(dk=64, dv=64) == -2                   # only the tensor-core shape
    assert call(chunk=32) == -2
    assert call(B=0) == 0                             # empty: nothing launched


def test_chunk_bwd_stall_test_takes_only_the_tensor_core_form(lib):
    p = lambda x: ctypes.c_void_p(x)
    args = [p(BASE + i * GB) for i in range(16)]

    def call(dk=128, dv=128, dtype=0):
        return lib.comba_chunk_bwd_stall_test(*args, 2, 64, 2, dk, dv, dtype, p(BASE + 20 * GB),
                                              ctypes.c_size_t(1 << 30), ctypes.c_ulonglong(1000), 1,
                                              ctypes.c_void_p(None))

    assert call(dtype=1) == -2          # fp32 inputs: not the tensor-core form
    assert call(dk=64) == -2
    assert call(dv=32) == -2


def test_stream_status_read_is_exported(lib):
    assert hasattr(lib, "comba_get_last_error_stream")
    assert "comba_get_last_error_stream" in cdr.EXPORTS
