"""Comba chunk-wise forward, its backward and the decode step on B200 (sm_100a).

Thin ctypes binding over the C ABI in ``include/comba.h``: it checks tensor
placement, dtypes and contiguity, allocates outputs with PyTorch when the
caller does not pass them, and hands raw device pointers and sizes to the
library.  Every step of the computation runs in the library's CUDA kernels;
there is no other implementation behind these functions, and they raise if
the library is missing or a tensor is not on a CUDA device.

Recurrence (Comba, "Improving Bilinear RNNs with Closed-loop Control"):
    S_t = alpha_t S_{t-1} - beta_t (S_{t-1} k_t) k_t^T + beta_t v_t k_t^T
    o_t = S_t (q_t - d_h k_t),        alpha_t = exp(log_alpha_t)
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

__all__ = ["chunk_fwd", "chunk_bwd", "state_compose", "chunk_fwd_transition", "chunk_fwd_gated", "chunk_fwd_host", "chunk_fwd_varlen", "chunk_fwd_noalloc",
           "recurrent_step",
           "get_last_error", "CombaError", "library", "library_path", "EXPORTS", "status_string"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libcomba.so")
_lib = None
_lock = threading.Lock()

EXPORTS = ("comba_chunk_fwd", "comba_chunk_fwd_f32", "comba_chunk_fwd_varlen",
           "comba_chunk_fwd_workspace_size", "comba_chunk_fwd_ws", "comba_chunk_fwd_noalloc",
           "comba_chunk_fwd_host", "comba_chunk_fwd_host_workspace_size", "comba_chunk_fwd_gated",
           "comba_chunk_bwd", "comba_chunk_bwd_workspace_size", "comba_state_compose",
           "comba_chunk_fwd_transition", "comba_chunk_fwd_stall_test", "comba_chunk_bwd_stall_test",
           "comba_recurrent_step", "comba_recurrent_step_grouped", "comba_get_last_error",
           "comba_get_last_error_stream", "comba_status_string", "comba_version")


class CombaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({status_string(status)})")


def library_path() -> str:
    return _LIB_PATH


def library():
    """The loaded ``libcomba.so`` (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                                   "`python -m chunk_delta_rule_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            vp, i = ctypes.c_void_p, ctypes.c_int
            chunk_sig = [vp] * 9 + [i] * 6 + [vp]
            lib.comba_chunk_fwd.argtypes = chunk_sig
            lib.comba_chunk_fwd_f32.argtypes = chunk_sig
            lib.comba_chunk_fwd_ws.argtypes = [vp] * 9 + [i] * 6 + [vp, ctypes.c_size_t, vp]
            lib.comba_chunk_fwd_noalloc.argtypes = chunk_sig
            lib.comba_chunk_fwd_workspace_size.argtypes = [i] * 6
            lib.comba_chunk_fwd_workspace_size.restype = ctypes.c_size_t
            lib.comba_chunk_fwd_varlen.argtypes = [vp] * 10 + [i] * 7 + [vp]
            lib.comba_chunk_fwd_gated.argtypes = [vp] * 11 + [i] * 6 + [ctypes.c_float, vp]
            lib.comba_chunk_fwd_host.argtypes = [vp] * 9 + [i] * 6 + [vp, ctypes.c_size_t, i, vp]
            lib.comba_chunk_fwd_host_workspace_size.argtypes = [i] * 5
            lib.comba_chunk_fwd_host_workspace_size.restype = ctypes.c_size_t
            lib.comba_recurrent_step.argtypes = [vp] * 8 + [i] * 4 + [vp]
            lib.comba_chunk_bwd.argtypes = [vp] * 16 + [i] * 6 + [vp, ctypes.c_size_t, vp]
            lib.comba_chunk_bwd_workspace_size.argtypes = [i] * 5
            lib.comba_state_compose.argtypes = [vp] * 3 + [i] * 3 + [vp]
            lib.comba_chunk_fwd_transition.argtypes = [vp] * 7 + [i] * 6 + [vp]
            lib.comba_chunk_fwd_stall_test.argtypes = [vp] * 9 + [i] * 6 + [ctypes.c_ulonglong, i, vp]
            lib.comba_chunk_bwd_stall_test.argtypes = ([vp] * 16 + [i] * 6 + [vp, ctypes.c_size_t, ctypes.c_ulonglong, i,
                                                        vp])
            lib.comba_chunk_bwd_workspace_size.restype = ctypes.c_size_t
            lib.comba_recurrent_step_grouped.argtypes = [vp] * 8 + [i] * 5 + [vp]
            for fn in (lib.comba_chunk_fwd, lib.comba_chunk_fwd_f32, lib.comba_chunk_fwd_ws,
                       lib.comba_chunk_fwd_noalloc, lib.comba_chunk_fwd_varlen,
                       lib.comba_recurrent_step_grouped, lib.comba_chunk_fwd_host,
                       lib.comba_chunk_fwd_gated, lib.comba_chunk_bwd, lib.comba_state_compose,
                       lib.comba_chunk_fwd_transition, lib.comba_chunk_fwd_stall_test, lib.comba_chunk_bwd_stall_test,
                       lib.comba_recurrent_step, lib.comba_get_last_error,
                       lib.comba_get_last_error_stream, lib.comba_version):
                fn.restype = ctypes.c_int
            lib.comba_get_last_error.argtypes = []
            lib.comba_get_last_error_stream.argtypes = [vp]
            lib.comba_version.argtypes = []
            lib.comba_status_string.argtypes = [ctypes.c_int]
            lib.comba_status_string.restype = ctypes.c_char_p
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().comba_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(None) if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t: torch.Tensor, name: str, dtype, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream_handle(device: torch.device, stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _keep_for_stream(t: Optional[torch.Tensor], device: torch.device, stream) -> None:
    """A device buffer from PyTorch's caching allocator that a call enqueues work on
    ``stream`` with: when that is not the device's current stream, the allocator is
    told, so the memory is not handed out again before the stream has passed the
    work (the allocator otherwise tracks only the stream it was allocated on)."""
    if t is None or stream is None:
        return
    cur = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        if stream.cuda_stream == cur.cuda_stream:
            return
        t.record_stream(stream)
    else:
        handle = int(stream)
        if handle == cur.cuda_stream:
            return
        t.record_stream(torch.cuda.ExternalStream(handle, device=device))


def chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
              beta: torch.Tensor, d: torch.Tensor, S0: Optional[torch.Tensor] = None,
              chunk: int = 64, out: Optional[torch.Tensor] = None,
              S_final: Optional[torch.Tensor] = None, return_state: bool = True,
              stream=None, segment: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunk-wise forward.  q, k [B,T,H,dk], v [B,T,H,dv] (bf16 or fp32, same
    dtype); log_alpha, beta [B,T,H] fp32; d [H] fp32; S0 [B,H,dv,dk] fp32 or None.
    Returns (out [B,T,H,dv] in q's dtype, S_final [B,H,dv,dk] fp32 or None).
    ``S_final`` may be passed as ``S0`` itself for an in-place state carry.
    ``segment=False`` keeps every chain in one CTA even when the library would cut
    long sequences of few chains into segments (comba_chunk_fwd_ws)."""
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in (torch.bfloat16, torch.float32):
        raise TypeError("q, k, v must be bf16 or fp32")
    _check(q, "q", dt, (B, T, H, dk))
    _check(k, "k", dt, (B, T, H, dk))
    _check(v, "v", dt, (B, T, H, dv))
    _check(log_alpha, "log_alpha", torch.float32, (B, T, H))
    _check(beta, "beta", torch.float32, (B, T, H))
    _check(d, "d", torch.float32, (H,))
    dev = q.device
    if S0 is not None:
        _check(S0, "S0", torch.float32, (B, H, dv, dk))
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _check(out, "out", dt, (B, T, H, dv))
    if S_final is None and return_state:
        S_final = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    if S_final is not None:
        _check(S_final, "S_final", torch.float32, (B, H, dv, dk))
    lib = library()
    with torch.cuda.device(dev):
        args = (_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(d), _ptr(S0),
                _ptr(out), _ptr(S_final), B, T, H, dk, dv, int(chunk))
        if dt == torch.bfloat16:
            # too few (b, h) chains for the GPU: the library runs them segmented in a
            # workspace from PyTorch's allocator (empty otherwise)
            nbytes = lib.comba_chunk_fwd_workspace_size(B, T, H, dk, dv, int(chunk)) if segment else 0
            ws = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None
            st = lib.comba_chunk_fwd_ws(*args, _ptr(ws), nbytes, _stream_handle(dev, stream))
            _keep_for_stream(ws, dev, stream)
            name = "comba_chunk_fwd_ws"
        else:
            st = lib.comba_chunk_fwd_f32(*args, _stream_handle(dev, stream))
            name = "comba_chunk_fwd_f32"
    if st != 0:
        raise CombaError(st, name)
    return out, S_final


def chunk_fwd_gated(q_raw: torch.Tensor, k_raw: torch.Tensor, v: torch.Tensor, a_raw: torch.Tensor,
                    b_raw: torch.Tensor, A_log: torch.Tensor, dt_bias: Optional[torch.Tensor],
                    d: torch.Tensor, S0: Optional[torch.Tensor] = None, chunk: int = 64,
                    norm_eps: float = 1e-6, out: Optional[torch.Tensor] = None,
                    S_final: Optional[torch.Tensor] = None, return_state: bool = True,
                    stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """comba_chunk_fwd_gated: the chunk-wise forward from raw projections.  q_raw,
    k_raw [B,T,H,dk] and v [B,T,H,dv] bf16; a_raw, b_raw [B,T,H] fp32 (raw gate
    projections); A_log [H], dt_bias [H] or None, d [H] fp32; S0 [B,H,dv,dk] or None.
    The kernel L2-normalises q, k (eps ``norm_eps``) and forms log_alpha =
    -exp(A_log) softplus(a_raw + dt_bias), beta = sigmoid(b_raw)."""
    if q_raw.dim() != 4:
        raise ValueError("q_raw must be [B, T, H, dk]")
    B, T, H, dk = q_raw.shape
    dv = v.shape[-1]
    _check(q_raw, "q_raw", torch.bfloat16, (B, T, H, dk))
    _check(k_raw, "k_raw", torch.bfloat16, (B, T, H, dk))
    _check(v, "v", torch.bfloat16, (B, T, H, dv))
    _check(a_raw, "a_raw", torch.float32, (B, T, H))
    _check(b_raw, "b_raw", torch.float32, (B, T, H))
    _check(A_log, "A_log", torch.float32, (H,))
    if dt_bias is not None:
        _check(dt_bias, "dt_bias", torch.float32, (H,))
    _check(d, "d", torch.float32, (H,))
    dev = q_raw.device
    if S0 is not None:
        _check(S0, "S0", torch.float32, (B, H, dv, dk))
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    _check(out, "out", torch.bfloat16, (B, T, H, dv))
    if S_final is None and return_state:
        S_final = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    if S_final is not None:
        _check(S_final, "S_final", torch.float32, (B, H, dv, dk))
    with torch.cuda.device(dev):
        st = library().comba_chunk_fwd_gated(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(a_raw), _ptr(b_raw),
                                             _ptr(A_log), _ptr(dt_bias), _ptr(d), _ptr(S0), _ptr(out),
                                             _ptr(S_final), B, T, H, dk, dv, int(chunk), float(norm_eps),
                                             _stream_handle(dev, stream))
    if st != 0:
        raise CombaError(st, "comba_chunk_fwd_gated")
    return out, S_final


def state_compose(R: torch.Tensor, M: torch.Tensor, S0: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """comba_state_compose: start states of P consecutive sequence pieces from their
    affine state transitions (a piece maps S to S M + R).  R, M [B, P, H, 128, 128]
    fp32; S0 [B, H, 128, 128] or None.  Returns S_start [B, P, H, 128, 128] with
    S_start[:, 0] = S0 and S_start[:, p] = S_start[:, p-1] M[:, p-1] + R[:, p-1]."""
    if R.dim() != 5:
        raise ValueError("R must be [B, P, H, 128, 128]")
    B, P, H = R.shape[:3]
    _check(R, "R", torch.float32, (B, P, H, 128, 128))
    _check(M, "M", torch.float32, (B, P, H, 128, 128))
    if S0 is not None:
        _check(S0, "S0", torch.float32, (B, H, 128, 128))
    dev = R.device
    RM = torch.stack([R, M])   # the entry point's layout: all R, then all M
    S_start = torch.empty((B, P, H, 128, 128), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        st = library().comba_state_compose(_ptr(RM), _ptr(S0), _ptr(S_start), B, H, P,
                                           _stream_handle(dev, stream))
        _keep_for_stream(RM, dev, stream)
    if st != 0:
        raise CombaError(st, "comba_state_compose")
    return S_start


def chunk_fwd_transition(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                         beta: torch.Tensor, d: torch.Tensor, chunk: int = 64,
                         RM: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """comba_chunk_fwd_transition: the affine state transition of these tokens, (R, M)
    with the state pass mapping S to S M + R.  q, k, v [B,T,H,128] bf16; log_alpha,
    beta [B,T,H] fp32; d [H] fp32.  Returns R, M [B, H, 128, 128] fp32 (views of one
    [2, B, H, 128, 128] buffer, ``RM`` if given)."""
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", torch.bfloat16, (B, T, H, dk))
    _check(k, "k", torch.bfloat16, (B, T, H, dk))
    _check(v, "v", torch.bfloat16, (B, T, H, dv))
    _check(log_alpha, "log_alpha", torch.float32, (B, T, H))
    _check(beta, "beta", torch.float32, (B, T, H))
    _check(d, "d", torch.float32, (H,))
    dev = q.device
    if RM is None:
        RM = torch.empty((2, B, H, dv, dk), dtype=torch.float32, device=dev)
    _check(RM, "RM", torch.float32, (2, B, H, dv, dk))
    with torch.cuda.device(dev):
        st = library().comba_chunk_fwd_transition(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                                  _ptr(d), _ptr(RM), B, T, H, dk, dv, int(chunk),
                                                  _stream_handle(dev, stream))
    if st != 0:
        raise CombaError(st, "comba_chunk_fwd_transition")
    return RM[0], RM[1]


_bwd_ws = {}


def chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
              beta: torch.Tensor, d: torch.Tensor, dout: torch.Tensor, S0: Optional[torch.Tensor] = None,
              dS_final: Optional[torch.Tensor] = None, need_dd: bool = True, need_dS0: bool = True,
              workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """comba_chunk_bwd: gradients of <dout, out> + <dS_final, S_final> of the chunk
    forward with respect to q, k, v, log_alpha, beta, d and S0.  q, k [B,T,H,dk], v,
    dout [B,T,H,dv]: all bf16 or all fp32; log_alpha, beta [B,T,H], d [H], S0 and
    dS_final [B,H,dv,dk] (or None): fp32.  Returns a dict of fp32 tensors dq, dk, dv,
    dlog_alpha, dbeta, dd (or None) and dS0 (or None).  ``workspace``: a uint8 device
    tensor of at least comba_chunk_bwd_workspace_size bytes; by default one is kept per
    device and grown as needed (it must not be shared by calls in flight on different
    streams)."""
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q, k, v, dout must be bf16 or fp32")
    dt = q.dtype
    _check(q, "q", dt, (B, T, H, dk))
    _check(k, "k", dt, (B, T, H, dk))
    _check(v, "v", dt, (B, T, H, dv))
    _check(dout, "dout", dt, (B, T, H, dv))
    _check(log_alpha, "log_alpha", torch.float32, (B, T, H))
    _check(beta, "beta", torch.float32, (B, T, H))
    _check(d, "d", torch.float32, (H,))
    if S0 is not None:
        _check(S0, "S0", torch.float32, (B, H, dv, dk))
    if dS_final is not None:
        _check(dS_final, "dS_final", torch.float32, (B, H, dv, dk))
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"dq": torch.empty((B, T, H, dk), **f32), "dk": torch.empty((B, T, H, dk), **f32),
         "dv": torch.empty((B, T, H, dv), **f32), "dlog_alpha": torch.empty((B, T, H), **f32),
         "dbeta": torch.empty((B, T, H), **f32),
         "dd": torch.empty((H,), **f32) if need_dd else None,
         "dS0": torch.empty((B, H, dv, dk), **f32) if need_dS0 else None}
    lib = library()
    need = int(lib.comba_chunk_bwd_workspace_size(B, T, H, dk, dv))
    if workspace is None:
        key = dev.index if dev.index is not None else torch.cuda.current_device()
        workspace = _bwd_ws.get(key)
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
            _bwd_ws[key] = workspace
    with torch.cuda.device(dev):
        st = lib.comba_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(d), _ptr(S0),
                                 _ptr(dout), _ptr(dS_final), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                                 _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]), _ptr(g["dd"]), _ptr(g["dS0"]),
                                 B, T, H, dk, dv, 0 if dt == torch.bfloat16 else 1, _ptr(workspace),
                                 workspace.numel(), _stream_handle(dev, stream))
        _keep_for_stream(workspace, dev, stream)   # also covers a cached buffer replaced later
    if st != 0:
        raise CombaError(st, "comba_chunk_bwd")
    return g


_host_ws = {}


def chunk_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                   beta: torch.Tensor, d: torch.Tensor, S0: Optional[torch.Tensor] = None,
                   chunk: int = 64, out: Optional[torch.Tensor] = None,
                   S_final: Optional[torch.Tensor] = None, return_state: bool = True,
                   slices: int = 8, device=None, stream=None,
                   workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """comba_chunk_fwd_host: bf16 HOST tensors in (pin them for overlap), host
    results out, the device work and both copy directions pipelined over `slices`
    groups of batch rows.  Layouts as chunk_fwd.  The device workspace comes from
    PyTorch's allocator (kept per device for later calls) unless given.  The call
    returns once the work is enqueued: keep every host tensor alive, and do not
    write the inputs or read the results, until ``stream`` (default: the current
    stream of ``device``) has passed the call."""
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]

    def host(t, name, dtype, shape):
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
            raise ValueError(f"{name} must be a CPU tensor")
        if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")

    for t, name in ((q, "q"), (k, "k")):
        host(t, name, torch.bfloat16, (B, T, H, dk))
    host(v, "v", torch.bfloat16, (B, T, H, dv))
    host(log_alpha, "log_alpha", torch.float32, (B, T, H))
    host(beta, "beta", torch.float32, (B, T, H))
    host(d, "d", torch.float32, (H,))
    if S0 is not None:
        host(S0, "S0", torch.float32, (B, H, dv, dk))
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=torch.bfloat16, pin_memory=True)
    host(out, "out", torch.bfloat16, (B, T, H, dv))
    if S_final is None and return_state:
        S_final = torch.empty((B, H, dv, dk), dtype=torch.float32, pin_memory=True)
    if S_final is not None:
        host(S_final, "S_final", torch.float32, (B, H, dv, dk))
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    lib = library()
    nbytes = lib.comba_chunk_fwd_host_workspace_size(B, T, H, dk, dv)
    if workspace is None and nbytes:
        ws = _host_ws.get(dev)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
            _host_ws[dev] = ws
        workspace = ws
    with torch.cuda.device(dev):
        st = lib.comba_chunk_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(d),
                                      _ptr(S0), _ptr(out), _ptr(S_final), B, T, H, dk, dv, int(chunk),
                                      _ptr(workspace), nbytes, int(slices), _stream_handle(dev, stream))
        _keep_for_stream(workspace, dev, stream)
    if st != 0:
        raise CombaError(st, "comba_chunk_fwd_host")
    return out, S_final


def chunk_fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                     beta: torch.Tensor, d: torch.Tensor, cu_seqlens: torch.Tensor,
                     S0: Optional[torch.Tensor] = None, chunk: int = 64,
                     out: Optional[torch.Tensor] = None, S_final: Optional[torch.Tensor] = None,
                     return_state: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunk-wise forward over packed variable-length sequences (comba_chunk_fwd_varlen).
    q, k [total_T, Hqk, dk] bf16; v [total_T, H, dv] bf16 with Hqk dividing H (value
    head h reads q / k head h // (H // Hqk)); log_alpha, beta [total_T, H] fp32; d [H]
    fp32; cu_seqlens [N+1] int32 on the device (sequence n = tokens cu_seqlens[n] ..
    cu_seqlens[n+1]-1); S0 [N, H, dv, dk] fp32 or None.  Returns (out [total_T, H, dv]
    bf16, S_final [N, H, dv, dk] fp32 or None)."""
    if q.dim() != 3:
        raise ValueError("q must be [total_T, Hqk, dk]")
    total_T, Hqk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be [N + 1]")
    N = cu_seqlens.numel() - 1
    _check(q, "q", torch.bfloat16, (total_T, Hqk, dk))
    _check(k, "k", torch.bfloat16, (total_T, Hqk, dk))
    _check(v, "v", torch.bfloat16, (total_T, H, dv))
    _check(log_alpha, "log_alpha", torch.float32, (total_T, H))
    _check(beta, "beta", torch.float32, (total_T, H))
    _check(d, "d", torch.float32, (H,))
    _check(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,))
    dev = q.device
    if S0 is not None:
        _check(S0, "S0", torch.float32, (N, H, dv, dk))
    if out is None:
        out = torch.empty((total_T, H, dv), dtype=torch.bfloat16, device=dev)
    _check(out, "out", torch.bfloat16, (total_T, H, dv))
    if S_final is None and return_state:
        S_final = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    if S_final is not None:
        _check(S_final, "S_final", torch.float32, (N, H, dv, dk))
    with torch.cuda.device(dev):
        st = library().comba_chunk_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                              _ptr(d), _ptr(S0), _ptr(out), _ptr(S_final),
                                              _ptr(cu_seqlens), N, total_T, H, Hqk, dk, dv, int(chunk),
                                              _stream_handle(dev, stream))
    if st != 0:
        raise CombaError(st, "comba_chunk_fwd_varlen")
    return out, S_final


def chunk_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                      beta: torch.Tensor, d: torch.Tensor, S0: Optional[torch.Tensor],
                      out: torch.Tensor, S_final: Optional[torch.Tensor], chunk: int = 64,
                      stream=None) -> None:
    """comba_chunk_fwd_noalloc on caller-allocated bf16 tensors (same layouts as
    chunk_fwd): the segmented form's scratch is the library's static device array."""
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check(t, name, torch.bfloat16, (B, T, H, dk if name in ("q", "k") else dv))
    _check(log_alpha, "log_alpha", torch.float32, (B, T, H))
    _check(beta, "beta", torch.float32, (B, T, H))
    _check(d, "d", torch.float32, (H,))
    for t, name in ((S0, "S0"), (S_final, "S_final")):
        if t is not None:
            _check(t, name, torch.float32, (B, H, dv, dk))
    dev = q.device
    with torch.cuda.device(dev):
        st = library().comba_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                               _ptr(d), _ptr(S0), _ptr(out), _ptr(S_final), B, T, H, dk,
                                               dv, int(chunk), _stream_handle(dev, stream))
    if st != 0:
        raise CombaError(st, "comba_chunk_fwd_noalloc")


def recurrent_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, log_alpha: torch.Tensor,
                   beta: torch.Tensor, d: torch.Tensor, S: torch.Tensor,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decode token: q, k [B,Hqk,dk] bf16, v [B,H,dv] bf16 with Hqk dividing H
    (Hqk == H: one q / k head per value head; otherwise value head h reads q / k head
    h // (H // Hqk)), log_alpha, beta [B,H] fp32, d [H] fp32, S [B,H,dv,dk] fp32
    updated in place.  Returns out [B,H,dv] bf16."""
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q must be [B, Hqk, dk] and v [B, H, dv]")
    B, Hqk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    _check(q, "q", torch.bfloat16, (B, Hqk, dk))
    _check(k, "k", torch.bfloat16, (B, Hqk, dk))
    _check(v, "v", torch.bfloat16, (B, H, dv))
    _check(log_alpha, "log_alpha", torch.float32, (B, H))
    _check(beta, "beta", torch.float32, (B, H))
    _check(d, "d", torch.float32, (H,))
    _check(S, "S", torch.float32, (B, H, dv, dk))
    dev = q.device
    if out is None:
        out = torch.empty((B, H, dv), dtype=torch.bfloat16, device=dev)
    _check(out, "out", torch.bfloat16, (B, H, dv))
    with torch.cuda.device(dev):
        st = library().comba_recurrent_step_grouped(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                                    _ptr(beta), _ptr(d), _ptr(S), _ptr(out), B, H, Hqk,
                                                    dk, dv, _stream_handle(dev, stream))
    if st != 0:
        raise CombaError(st, "comba_recurrent_step_grouped")
    return out


def get_last_error(device=None, stream=None) -> int:
    """Reads and clears the device-side status word.  Without ``stream`` the whole
    device is synchronised first (comba_get_last_error); with one, only that stream
    (comba_get_last_error_stream: the word is shared by all streams of the device)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        if stream is None:
            return int(library().comba_get_last_error())
        return int(library().comba_get_last_error_stream(_stream_handle(dev, stream)))
