"""Python binding of the C ABI in include/lightning_attn.h (argument marshalling only).

Every function here checks tensor dtypes/shapes/devices, then calls the
matching ``extern "C"`` entry point of ``liblightning_attn.so`` through ctypes
on the current CUDA stream.  There is no other implementation behind these
functions: if the library is missing or a call fails, they raise.
"""
from __future__ import annotations

import ctypes
import functools
import os
import threading
from typing import Optional

import torch

_SO = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblightning_attn.so")
_lock = threading.Lock()
_lib = None

LA_OK = 0
STATUS_NAMES = {0: "LA_OK", 1: "LA_ERR_NULL", 2: "LA_ERR_SHAPE", 3: "LA_ERR_ALIGN",
                4: "LA_ERR_UNSUPPORTED", 5: "LA_ERR_CUDA", 6: "LA_ERR_TIMEOUT",
                7: "LA_ERR_WORKSPACE"}

# Exported entry points and their ctypes signatures (all return int).
_P, _I = ctypes.c_void_p, ctypes.c_int
SIGNATURES = {
    "lightning_attn_fwd": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P],
    "lightning_attn_fwd_ex": [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P],
    "lightning_attn_fwd_noalloc": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P],
    "lightning_attn_fwd_f32": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P],
    "lightning_attn_fault_test_scan_stall": [_P, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_uint, _P],
    "lightning_attn_decode": [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P],
    "lightning_attn_status_string": [_I],
    "lightning_attn_last_cuda_error": [],
    "lightning_attn_device_status": [_P, _I],
    "lightning_attn_fwd_plan": [_I, _I, _I, _I, _I, _P, _P, _I, _P],
    "lightning_attn_fwd_anticausal": [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P],
    "lightning_attn_fwd_fused": [_P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _I, _I, _I, _I, _I,
                                 _P],
    "lightning_attn_bwd": [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P],
    "lightning_attn_fwd_strided": [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P,
                                   _I, _P],
    "lightning_attn_set_cta_limit": [_I, _P],
    "lightning_attn_fwd_fused_ex": [_P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P, _I, _I,
                                    _I, _I, _I, _P, _P, _P, _P, _P, _I, _P],
    "lightning_attn_decode_fused": [_P, _P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _I, _I, _I,
                                    _I, _P, _P, _P, _P, _P, _P],
    "lightning_attn_state": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P],
    "lightning_attn_state_combine": [_P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _P],
}


class LightningAttnError(RuntimeError):
    """A C-ABI call returned a non-zero status."""

    def __init__(self, fn: str, code: int):
        detail = ""
        if code == 5:
            detail = f" [{lib().lightning_attn_last_cuda_error().decode()}]"
        super().__init__(f"{fn} failed: {status_string(code)} (code {code}){detail}")
        self.code = code


def library_path() -> str:
    return _SO


def lib():
    """Loads liblightning_attn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_SO):
                raise RuntimeError(
                    f"{_SO} is missing: build it with `python -m long_context_fwd_b200.build` "
                    "(or __graft_entry__.build()); there is no fallback implementation")
            L = ctypes.CDLL(_SO)
            for name, argtypes in SIGNATURES.items():
                fn = getattr(L, name)
                fn.argtypes = argtypes
                fn.restype = (ctypes.c_char_p if name in ("lightning_attn_status_string",
                                                          "lightning_attn_last_cuda_error") else _I)
            _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().lightning_attn_status_string(int(code)).decode()


def _check(fn: str, rc: int):
    if rc != LA_OK:
        raise LightningAttnError(fn, rc)


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _on_tensor_device(fn):
    """Runs an entry point on the CUDA device its tensors live on (the library
    launches on the calling thread's current device, with that device's
    current stream by default); tensors on different devices are refused, so
    no kernel is ever handed another device's pointers."""
    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        tensors = [a for a in (*args, *kwargs.values()) if isinstance(a, torch.Tensor)]
        devices = {t.device for t in tensors if t.is_cuda}
        if len(devices) > 1:
            raise ValueError(f"{fn.__name__}: all tensors must be on one CUDA device, got "
                             f"{sorted(str(d) for d in devices)}")
        if not devices:
            return fn(*args, **kwargs)  # the argument checks reject non-CUDA tensors
        (dev,) = devices
        stream = kwargs.get("stream")
        if stream is not None and stream.device != dev:
            raise ValueError(f"{fn.__name__}: stream is on {stream.device}, tensors on {dev}")
        with torch.cuda.device(dev):
            return fn(*args, **kwargs)
    return wrapper


def _need(t: torch.Tensor, name: str, dtype, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@_on_tensor_device
def fwd(q, k, v, slopes, out=None, *, init_state=None, final_state=None, chunk: int = 0,
        stream=None) -> torch.Tensor:
    """Prefill: bf16 q, k [B,H,N,D], v [B,H,N,E], fp32 slopes [H] -> fp32 out [B,H,N,E]."""
    B, H, N, D = q.shape
    E = v.shape[-1]
    _need(q, "q", torch.bfloat16, (B, H, N, D))
    _need(k, "k", torch.bfloat16, (B, H, N, D))
    _need(v, "v", torch.bfloat16, (B, H, N, E))
    _need(slopes, "slopes", torch.float32, (H,))
    if out is None:
        out = torch.empty((B, H, N, E), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, H, N, E))
    for name, st in (("init_state", init_state), ("final_state", final_state)):
        if st is not None:
            _need(st, name, torch.float32, (B, H, D, E))
    L = lib()
    if init_state is None and final_state is None and chunk == 0:
        rc = L.lightning_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), slopes.data_ptr(),
                                  out.data_ptr(), B, H, N, D, E, _stream_handle(stream))
        _check("lightning_attn_fwd", rc)
    else:
        rc = L.lightning_attn_fwd_ex(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), slopes.data_ptr(),
            None if init_state is None else init_state.data_ptr(),
            None if final_state is None else final_state.data_ptr(),
            out.data_ptr(), B, H, N, D, E, int(chunk), _stream_handle(stream))
        _check("lightning_attn_fwd_ex", rc)
    return out


def _need_view(t: torch.Tensor, name: str, dtype, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.stride(-1) != 1:
        raise ValueError(f"{name}: the last dimension must be contiguous")


@_on_tensor_device
def fwd_strided(q, k, v, slopes, out, *, init_state=None, final_state=None, chunk: int = 0,
                stream=None) -> torch.Tensor:
    """Prefill on strided views: q, k [B,H,N,D] and v [B,H,N,E] bf16, out [B,H,N,E] fp32,
    each with any (b, h, t) strides and a contiguous last dimension -- e.g.
    ``qt.permute(0, 2, 1, 3)`` of a token-major ``qt`` [B,N,H,D], or slices of a
    fused [B,N,3,H,D] projection output."""
    B, H, N, D = q.shape
    E = v.shape[-1]
    _need_view(q, "q", torch.bfloat16, (B, H, N, D))
    _need_view(k, "k", torch.bfloat16, (B, H, N, D))
    _need_view(v, "v", torch.bfloat16, (B, H, N, E))
    _need_view(out, "out", torch.float32, (B, H, N, E))
    _need(slopes, "slopes", torch.float32, (H,))
    for name, st in (("init_state", init_state), ("final_state", final_state)):
        if st is not None:
            _need(st, name, torch.float32, (B, H, D, E))
    arr = [(ctypes.c_longlong * 3)(*t.stride()[:3]) for t in (q, k, v, out)]
    rc = lib().lightning_attn_fwd_strided(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), slopes.data_ptr(),
        None if init_state is None else init_state.data_ptr(),
        None if final_state is None else final_state.data_ptr(),
        out.data_ptr(), B, H, N, D, E, *[ctypes.cast(a, ctypes.c_void_p) for a in arr],
        int(chunk), _stream_handle(stream))
    _check("lightning_attn_fwd_strided", rc)
    return out


@_on_tensor_device
def fwd_anticausal(q, k, v, slopes, out=None, *, init_state=None, final_state=None,
                   chunk: int = 0, stream=None) -> torch.Tensor:
    """Anti-causal prefill, o_t = sum_{s >= t} g^(s-t) (q_t . k_s) v_s (shapes as fwd)."""
    B, H, N, D = q.shape
    E = v.shape[-1]
    _need(q, "q", torch.bfloat16, (B, H, N, D))
    _need(k, "k", torch.bfloat16, (B, H, N, D))
    _need(v, "v", torch.bfloat16, (B, H, N, E))
    _need(slopes, "slopes", torch.float32, (H,))
    if out is None:
        out = torch.empty((B, H, N, E), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, H, N, E))
    for name, st in (("init_state", init_state), ("final_state", final_state)):
        if st is not None:
            _need(st, name, torch.float32, (B, H, D, E))
    rc = lib().lightning_attn_fwd_anticausal(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), slopes.data_ptr(),
        None if init_state is None else init_state.data_ptr(),
        None if final_state is None else final_state.data_ptr(),
        out.data_ptr(), B, H, N, D, E, int(chunk), _stream_handle(stream))
    _check("lightning_attn_fwd_anticausal", rc)
    return out


@_on_tensor_device
def fwd_fused(q, k, v, gate, slopes, norm_weight, eps: float = 1e-6, out=None, *,
              stream=None) -> torch.Tensor:
    """The fused layer: raw bf16 q, k [B,H,N,D], v, gate [B,H,N,E], fp32 norm_weight
    [H,E] -> bf16 w * RMSNorm_E(attention(silu(q), silu(k), silu(v))) * sigmoid(gate)."""
    B, H, N, D = q.shape
    E = v.shape[-1]
    _need(q, "q", torch.bfloat16, (B, H, N, D))
    _need(k, "k", torch.bfloat16, (B, H, N, D))
    _need(v, "v", torch.bfloat16, (B, H, N, E))
    _need(gate, "gate", torch.bfloat16, (B, H, N, E))
    _need(slopes, "slopes", torch.float32, (H,))
    _need(norm_weight, "norm_weight", torch.float32, (H, E))
    if out is None:
        out = torch.empty((B, H, N, E), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, (B, H, N, E))
    rc = lib().lightning_attn_fwd_fused(q.data_ptr(), k.data_ptr(), v.data_ptr(), gate.data_ptr(),
                                        slopes.data_ptr(), norm_weight.data_ptr(), float(eps),
                                        out.data_ptr(), B, H, N, D, E, _stream_handle(stream))
    _check("lightning_attn_fwd_fused", rc)
    return out


@_on_tensor_device
def fwd_fused_ex(q, k, v, gate, slopes, norm_weight, eps: float = 1e-6, out=None, *,
                 init_state=None, final_state=None, chunk: int = 0, stream=None) -> torch.Tensor:
    """The fused layer on [B,H,N,*] views with any (b, h, t) strides and a
    contiguous last dimension (e.g. ``x.permute(0, 2, 1, 3)`` of token-major
    [B,N,H,*] buffers, or slices of a fused [B,N,3,H,D] projection), with the
    recurrent state (over the activated k, v) optionally handed in and out:
    fp32 init_state / final_state [B,H,D,E].  out defaults to a head-major
    contiguous bf16 tensor."""
    B, H, N, D = q.shape
    E = v.shape[-1]
    _need_view(q, "q", torch.bfloat16, (B, H, N, D))
    _need_view(k, "k", torch.bfloat16, (B, H, N, D))
    _need_view(v, "v", torch.bfloat16, (B, H, N, E))
    _need_view(gate, "gate", torch.bfloat16, (B, H, N, E))
    _need(slopes, "slopes", torch.float32, (H,))
    _need(norm_weight, "norm_weight", torch.float32, (H, E))
    if out is None:
        out = torch.empty((B, H, N, E), dtype=torch.bfloat16, device=q.device)
    _need_view(out, "out", torch.bfloat16, (B, H, N, E))
    for name, st in (("init_state", init_state), ("final_state", final_state)):
        if st is not None:
            _need(st, name, torch.float32, (B, H, D, E))
    arr = [(ctypes.c_longlong * 3)(*t.stride()[:3]) for t in (q, k, v, gate, out)]
    rc = lib().lightning_attn_fwd_fused_ex(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), gate.data_ptr(), slopes.data_ptr(),
        norm_weight.data_ptr(), float(eps),
        None if init_state is None else init_state.data_ptr(),
        None if final_state is None else final_state.data_ptr(), out.data_ptr(), B, H, N, D, E,
        *[ctypes.cast(a, ctypes.c_void_p) for a in arr], int(chunk), _stream_handle(stream))
    _check("lightning_attn_fwd_fused_ex", rc)
    return out


@_on_tensor_device
def decode_fused(q, k, v, gate, state, slopes, norm_weight, eps: float = 1e-6, out=None, *,
                 stream=None) -> torch.Tensor:
    """One decode step of the fused layer: raw bf16 q, k [B,H,D], v, gate [B,H,E]
    views (any (b, h) strides, contiguous last dimension); fp32 state
    [B,H,D,E] (contiguous) advanced in place; bf16 out [B,H,E]."""
    B, H, D = q.shape
    E = v.shape[-1]
    _need_view(q, "q", torch.bfloat16, (B, H, D))
    _need_view(k, "k", torch.bfloat16, (B, H, D))
    _need_view(v, "v", torch.bfloat16, (B, H, E))
    _need_view(gate, "gate", torch.bfloat16, (B, H, E))
    _need(state, "state", torch.float32, (B, H, D, E))
    _need(slopes, "slopes", torch.float32, (H,))
    _need(norm_weight, "norm_weight", torch.float32, (H, E))
    if out is None:
        out = torch.empty((B, H, E), dtype=torch.bfloat16, device=q.device)
    _need_view(out, "out", torch.bfloat16, (B, H, E))
    arr = [(ctypes.c_longlong * 2)(*t.stride()[:2]) for t in (q, k, v, gate, out)]
    rc = lib().lightning_attn_decode_fused(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), gate.data_ptr(), state.data_ptr(),
        slopes.data_ptr(), norm_weight.data_ptr(), float(eps), out.data_ptr(), B, H, D, E,
        *[ctypes.cast(a, ctypes.c_void_p) for a in arr], _stream_handle(stream))
    _check("lightning_attn_decode_fused", rc)
    return out


@_on_tensor_device
def state(k, v, slopes, final_state=None, *, init_state=None, chunk: int = 0,
          stream=None) -> torch.Tensor:
    """The state after N tokens without the outputs: bf16 k [B,H,N,D], v [B,H,N,E]
    -> fp32 [B,H,D,E] (from init_state, zero if None)."""
    B, H, N, D = k.shape
    E = v.shape[-1]
    _need(k, "k", torch.bfloat16, (B, H, N, D))
    _need(v, "v", torch.bfloat16, (B, H, N, E))
    _need(slopes, "slopes", torch.float32, (H,))
    if final_state is None:
        final_state = torch.empty((B, H, D, E), dtype=torch.float32, device=k.device)
    _need(final_state, "final_state", torch.float32, (B, H, D, E))
    if init_state is not None:
        _need(init_state, "init_state", torch.float32, (B, H, D, E))
    rc = lib().lightning_attn_state(
        k.data_ptr(), v.data_ptr(), slopes.data_ptr(),
        None if init_state is None else init_state.data_ptr(), final_state.data_ptr(),
        B, H, N, D, E, int(chunk), _stream_handle(stream))
    _check("lightning_attn_state", rc)
    return final_state


@_on_tensor_device
def state_combine(states, chunk_tokens, slopes, out=None, *, init_state=None,
                  stream=None) -> torch.Tensor:
    """The state after R consecutive chunks: fp32 states [R,B,H,D,E] (each chunk's
    state from a zero initial state), chunk_tokens a sequence of R token counts
    -> fp32 [B,H,D,E] (from init_state, zero if None)."""
    R, B, H, D, E = states.shape
    _need(states, "states", torch.float32, (R, B, H, D, E))
    _need(slopes, "slopes", torch.float32, (H,))
    counts = [int(x) for x in chunk_tokens]
    if len(counts) != R:
        raise ValueError(f"chunk_tokens must have {R} entries, got {len(counts)}")
    if out is None:
        out = torch.empty((B, H, D, E), dtype=torch.float32, device=states.device)
    _need(out, "out", torch.float32, (B, H, D, E))
    if init_state is not None:
        _need(init_state, "init_state", torch.float32, (B, H, D, E))
    arr = (ctypes.c_int * max(1, R))(*counts)
    rc = lib().lightning_attn_state_combine(
        states.data_ptr() if R else None, R, ctypes.cast(arr, ctypes.c_void_p),
        slopes.data_ptr(), None if init_state is None else init_state.data_ptr(),
        out.data_ptr(), B, H, D, E, _stream_handle(stream))
    _check("lightning_attn_state_combine", rc)
    return out


@_on_tensor_device
def bwd(q, k, v, dout, slopes, dq=None, dk=None, dv=None, *, stream=None):
    """Backward pass: bf16 q, k [B,H,N,D], v, dout [B,H,N,E] -> fp32 (dq, dk, dv)."""
    B, H, N, D = q.shape
    E = v.shape[-1]
    _need(q, "q", torch.bfloat16, (B, H, N, D))
    _need(k, "k", torch.bfloat16, (B, H, N, D))
    _need(v, "v", torch.bfloat16, (B, H, N, E))
    _need(dout, "dout", torch.bfloat16, (B, H, N, E))
    _need(slopes, "slopes", torch.float32, (H,))
    dq = torch.empty((B, H, N, D), dtype=torch.float32, device=q.device) if dq is None else dq
    dk = torch.empty((B, H, N, D), dtype=torch.float32, device=q.device) if dk is None else dk
    dv = torch.empty((B, H, N, E), dtype=torch.float32, device=q.device) if dv is None else dv
    _need(dq, "dq", torch.float32, (B, H, N, D))
    _need(dk, "dk", torch.float32, (B, H, N, D))
    _need(dv, "dv", torch.float32, (B, H, N, E))
    rc = lib().lightning_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(),
                                  slopes.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                  B, H, N, D, E, _stream_handle(stream))
    _check("lightning_attn_bwd", rc)
    return dq, dk, dv


@_on_tensor_device
def fwd_noalloc(q, k, v, slopes, out=None, *, chunk: int = 0, stream=None) -> torch.Tensor:
    """Prefill through the allocation-free entry point (scratch in a fixed device array).

    For callers that must not allocate device memory on the call path; see
    lightning_attn_fwd_noalloc in include/lightning_attn.h for the limit and
    the rule that overlapping calls on one device race on the shared scratch.
    `out` should be passed preallocated by such callers.
    """
    B, H, N, D = q.shape
    E = v.shape[-1]
    _need(q, "q", torch.bfloat16, (B, H, N, D))
    _need(k, "k", torch.bfloat16, (B, H, N, D))
    _need(v, "v", torch.bfloat16, (B, H, N, E))
    _need(slopes, "slopes", torch.float32, (H,))
    if out is None:
        out = torch.empty((B, H, N, E), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, H, N, E))
    rc = lib().lightning_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                          slopes.data_ptr(), out.data_ptr(), B, H, N, D, E,
                                          int(chunk), _stream_handle(stream))
    _check("lightning_attn_fwd_noalloc", rc)
    return out


@_on_tensor_device
def fwd_f32(q, k, v, slopes, out=None, *, stream=None) -> torch.Tensor:
    """Prefill with fp32 q, k, v -> fp32 out."""
    B, H, N, D = q.shape
    E = v.shape[-1]
    _need(q, "q", torch.float32, (B, H, N, D))
    _need(k, "k", torch.float32, (B, H, N, D))
    _need(v, "v", torch.float32, (B, H, N, E))
    _need(slopes, "slopes", torch.float32, (H,))
    if out is None:
        out = torch.empty((B, H, N, E), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, H, N, E))
    rc = lib().lightning_attn_fwd_f32(q.data_ptr(), k.data_ptr(), v.data_ptr(), slopes.data_ptr(),
                                      out.data_ptr(), B, H, N, D, E, _stream_handle(stream))
    _check("lightning_attn_fwd_f32", rc)
    return out


@_on_tensor_device
def decode(q, k, v, state, slopes, out=None, *, stream=None) -> torch.Tensor:
    """One decode step: bf16 q, k [B,H,D], v [B,H,E]; fp32 state [B,H,D,E] in place."""
    B, H, D = q.shape
    E = v.shape[-1]
    _need(q, "q", torch.bfloat16, (B, H, D))
    _need(k, "k", torch.bfloat16, (B, H, D))
    _need(v, "v", torch.bfloat16, (B, H, E))
    _need(state, "state", torch.float32, (B, H, D, E))
    _need(slopes, "slopes", torch.float32, (H,))
    if out is None:
        out = torch.empty((B, H, E), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, H, E))
    rc = lib().lightning_attn_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), state.data_ptr(),
                                     slopes.data_ptr(), out.data_ptr(), B, H, D, E,
                                     _stream_handle(stream))
    _check("lightning_attn_decode", rc)
    return out


@_on_tensor_device
def fault_test_scan_stall(q, k, v, slopes, out, *, chunk: int, wait_limit_ms: int,
                          stream=None) -> None:
    """Runs the prefill with chunk 0 never processed (see the C header): every
    chunk-1 item waits on a flag nothing sets until its bounded wait gives up."""
    B, H, N, D = q.shape
    _need(q, "q", torch.bfloat16, (B, H, N, 128))
    _need(k, "k", torch.bfloat16, (B, H, N, 128))
    _need(v, "v", torch.bfloat16, (B, H, N, 128))
    _need(slopes, "slopes", torch.float32, (H,))
    _need(out, "out", torch.float32, (B, H, N, 128))
    rc = lib().lightning_attn_fault_test_scan_stall(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), slopes.data_ptr(), out.data_ptr(), B, H, N,
        int(chunk), int(wait_limit_ms), _stream_handle(stream))
    _check("lightning_attn_fault_test_scan_stall", rc)


def set_cta_limit(max_ctas: int) -> int:
    """Caps the prefill kernel's persistent grid for later calls (0 = one CTA
    per SM); returns the previous cap.  Process-wide."""
    prev = ctypes.c_int(0)
    _check("lightning_attn_set_cta_limit",
           lib().lightning_attn_set_cta_limit(int(max_ctas), ctypes.byref(prev)))
    return prev.value


def device_status(reset: bool = True) -> int:
    """Sticky device-side status of the current device (synchronises)."""
    v = ctypes.c_int(0)
    _check("lightning_attn_device_status",
           lib().lightning_attn_device_status(ctypes.byref(v), 1 if reset else 0))
    return v.value


PLAN_FIELDS = ("cta", "kind", "seq", "a", "b", "flags", "enter_slot", "enter_val", "pub_slot",
               "pub_val")
PLAN_INFO = ("mode", "grid", "L", "nchunks", "F", "G2", "slots", "flags")


def fwd_plan(B: int, H: int, N: int, chunk: int = 0, sms: int = 148):
    """Host-side enumeration of the prefill kernel's work items (no GPU needed):
    returns (info dict, int32 array [n, 10] of records; see PLAN_FIELDS)."""
    import numpy as np
    info = (ctypes.c_int * 8)()
    n = ctypes.c_int(0)
    rc = lib().lightning_attn_fwd_plan(B, H, N, chunk, sms, info, None, 0, ctypes.byref(n))
    if rc not in (0, 7):
        _check("lightning_attn_fwd_plan", rc)
    rec = np.zeros((max(n.value, 1), 10), np.int32)
    _check("lightning_attn_fwd_plan",
           lib().lightning_attn_fwd_plan(B, H, N, chunk, sms, info,
                                         rec.ctypes.data_as(ctypes.c_void_p), n.value,
                                         ctypes.byref(n)))
    return dict(zip(PLAN_INFO, list(info))), rec[:n.value]
