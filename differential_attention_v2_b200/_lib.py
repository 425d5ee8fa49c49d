"""ctypes binding of libdiffattn_v2.so: the same entry points as include/diffattn_v2.h.

Argument marshalling only: every step of the operator runs in the CUDA library. The
wrappers take torch CUDA tensors, check dtype/shape/contiguity, pass data pointers and the
current (or given) stream, and raise on a non-OK status. Output tensors and the decode
workspace are allocated with torch when the caller does not pass them.

There is no CPU fallback: if the library is missing, importing fails with an error that
says how to build it.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdiffattn_v2.so")

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE = 0, -1, -2, -3, -4

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

_SIGNATURES = {
    "diffattn_v2_version": (_i, []),
    "diffattn_v2_status_string": (ctypes.c_char_p, [_i]),
    "diffattn_v2_prefill": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "diffattn_v2_prefill_f32": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "diffattn_v2_prefill_window": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "diffattn_v2_prefill_varlen": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "diffattn_v2_prefill_train": (_i, [_vp] * 7 + [_i] * 6 + [_vp]),
    "diffattn_v2_backward_workspace_size": (_sz, [_i, _i, _i]),
    "diffattn_v2_backward": (_i, [_vp] * 11 + [_i] * 6 + [_vp, _sz, _vp]),
    "diffattn_v2_prefill_window_train": (_i, [_vp] * 7 + [_i] * 6 + [_vp]),
    "diffattn_v2_backward_window": (_i, [_vp] * 11 + [_i] * 6 + [_vp, _sz, _vp]),
    "diffattn_v2_prefill_varlen_train": (_i, [_vp] * 8 + [_i] * 7 + [_vp]),
    "diffattn_v2_backward_varlen_workspace_size": (_sz, [_i, _i, _i]),
    "diffattn_v2_backward_varlen": (_i, [_vp] * 12 + [_i] * 7 + [_vp, _sz, _vp]),
    "diffattn_v2_prefill_varlen_window_train": (_i, [_vp] * 8 + [_i] * 7 + [_vp]),
    "diffattn_v2_backward_varlen_window": (_i, [_vp] * 12 + [_i] * 7 + [_vp, _sz, _vp]),
    "diffattn_v2_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "diffattn_v2_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "diffattn_v2_decode_window": (_i, [_vp] * 6 + [_i] * 6 + [_vp, _sz, _vp]),
    "diffattn_v2_decode_f32": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "diffattn_v2_decode_paged": (_i, [_vp] * 7 + [_i] * 7 + [_vp, _sz, _vp]),
    "diffattn_v2_decode_paged_window": (_i, [_vp] * 7 + [_i] * 8 + [_vp, _sz, _vp]),
    "diffattn_v2_decode_multi_workspace_size": (_sz, [_i] * 6),
    "diffattn_v2_decode_multi": (_i, [_vp] * 6 + [_i] * 6 + [_vp, _sz, _vp]),
    "diffattn_v2_lambda_v1": (_i, [_vp, _vp, _vp, _vp, _f, _i, _i, _i, _vp, _vp]),
    "diffattn_v2_lambda_v2": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _vp]),
    "diffattn_v2_prefill_fused_lambda": (_i, [_vp] * 8 + [_i] * 7 + [_vp]),
    "diffattn_v2_prefill_varlen_window": (_i, [_vp] * 6 + [_i] * 7 + [_vp]),
    "diffattn_v2_device_error": (_i, [ctypes.POINTER(_i), _vp]),
    "diffattn_v2_decode_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
}
EXPORTED = tuple(_SIGNATURES)


def load(path=LIB_PATH):
    """Load a build of the library (the default, or e.g. its bounds-checking twin
    libdiffattn_v2_debug.so) with the entry points' argument and result types set. The
    wrappers below call the module's LIB."""
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing; build it with `python -m differential_attention_v2_b200.build` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = load()


class DiffAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {LIB.diffattn_v2_status_string(status).decode()} ({status})")


def _check(status: int, what: str):
    if status != OK:
        raise DiffAttnError(status, what)


def _stream(stream, device):
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, name, dtype, ndim):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dimensions, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def version() -> int:
    return LIB.diffattn_v2_version()


def prefill(q, k, v, lam, out=None, causal=True, stream=None):
    """bf16 prefill: q [B,S,Hq,D], k/v [B,S,Hkv,D], lam fp32 [B,S,Hq/2] -> out bf16 [B,S,Hq/2,D]."""
    for t, n, nd in ((q, "q", 4), (k, "k", 4), (v, "v", 4)):
        _need(t, n, torch.bfloat16, nd)
    _need(lam, "lam", torch.float32, 3)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty((B, S, Hq // 2, D), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    st = LIB.diffattn_v2_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), B, S, Hq, Hkv, D,
                                 1 if causal else 0, _stream(stream, q.device))
    _check(st, "diffattn_v2_prefill")
    return out


def prefill_window(q, k, v, lam, window, out=None, stream=None):
    """bf16 causal prefill where query i sees only keys i-window+1 .. i."""
    for t, n, nd in ((q, "q", 4), (k, "k", 4), (v, "v", 4)):
        _need(t, n, torch.bfloat16, nd)
    _need(lam, "lam", torch.float32, 3)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty((B, S, Hq // 2, D), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    st = LIB.diffattn_v2_prefill_window(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), B, S, Hq, Hkv, D,
                                        int(window), _stream(stream, q.device))
    _check(st, "diffattn_v2_prefill_window")
    return out


def prefill_varlen(q, k, v, lam, cu_seqlens, max_seqlen, out=None, causal=True, stream=None):
    """bf16 prefill of packed sequences: q [T,Hq,D], k/v [T,Hkv,D], lam fp32 [T,Hq/2],
    cu_seqlens int32 [B+1] on the device; max_seqlen >= the longest sequence."""
    for t, n, nd in ((q, "q", 3), (k, "k", 3), (v, "v", 3)):
        _need(t, n, torch.bfloat16, nd)
    _need(lam, "lam", torch.float32, 2)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((T, Hq // 2, D), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 3)
    st = LIB.diffattn_v2_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), _ptr(cu_seqlens), B,
                                        int(max_seqlen), T, Hq, Hkv, D, 1 if causal else 0, _stream(stream, q.device))
    _check(st, "diffattn_v2_prefill_varlen")
    return out


def prefill_varlen_window(q, k, v, lam, cu_seqlens, max_seqlen, window, out=None, stream=None):
    """Causal sliding-window prefill of packed sequences (layouts of prefill_varlen): query i
    of a sequence sees that sequence's keys i-window+1 .. i."""
    for t, n, nd in ((q, "q", 3), (k, "k", 3), (v, "v", 3)):
        _need(t, n, torch.bfloat16, nd)
    _need(lam, "lam", torch.float32, 2)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((T, Hq // 2, D), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 3)
    st = LIB.diffattn_v2_prefill_varlen_window(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), _ptr(cu_seqlens), B,
                                               int(max_seqlen), T, Hq, Hkv, D, int(window), _stream(stream, q.device))
    _check(st, "diffattn_v2_prefill_varlen_window")
    return out


def prefill_f32(q, k, v, lam, out=None, causal=True, stream=None):
    """fp32 prefill on CUDA cores; same layout as prefill with fp32 tensors."""
    for t, n, nd in ((q, "q", 4), (k, "k", 4), (v, "v", 4), (lam, "lam", 3)):
        _need(t, n, torch.float32, nd)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty((B, S, Hq // 2, D), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, 4)
    st = LIB.diffattn_v2_prefill_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), B, S, Hq, Hkv, D,
                                     1 if causal else 0, _stream(stream, q.device))
    _check(st, "diffattn_v2_prefill_f32")
    return out


def prefill_train(q, k, v, lam, out=None, o_branch=None, lse=None, causal=True, window=None, stream=None):
    """Training forward: prefill plus the per-head normalised O_b (bf16 [B,S,Hq,D]) and the
    log2-domain row log-sum-exp (fp32 [B,S,Hq]) that backward reads. Returns (out, o_branch, lse).
    With `window` the causal sliding-window prefill (query i sees keys i-window+1 .. i)."""
    for t, n, nd in ((q, "q", 4), (k, "k", 4), (v, "v", 4)):
        _need(t, n, torch.bfloat16, nd)
    _need(lam, "lam", torch.float32, 3)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty((B, S, Hq // 2, D), dtype=torch.bfloat16, device=q.device)
    if o_branch is None:
        o_branch = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, S, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    _need(o_branch, "o_branch", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    if window is not None:
        st = LIB.diffattn_v2_prefill_window_train(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), _ptr(o_branch),
                                                  _ptr(lse), B, S, Hq, Hkv, D, int(window), _stream(stream, q.device))
        _check(st, "diffattn_v2_prefill_window_train")
        return out, o_branch, lse
    st = LIB.diffattn_v2_prefill_train(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), _ptr(o_branch), _ptr(lse),
                                       B, S, Hq, Hkv, D, 1 if causal else 0, _stream(stream, q.device))
    _check(st, "diffattn_v2_prefill_train")
    return out, o_branch, lse


def backward_workspace_size(B, S, Hq) -> int:
    return int(LIB.diffattn_v2_backward_workspace_size(B, S, Hq))


def backward(q, k, v, lam, o_branch, lse, dout, causal=True, dq=None, dk=None, dv=None, dlam=None,
             workspace=None, window=None, stream=None):
    """Gradients of the bf16 prefill: returns (dq, dk, dv, dlam) with the layouts of q, k, v, lam.
    With `window` the gradients of the causal sliding-window prefill."""
    for t, n, nd in ((q, "q", 4), (k, "k", 4), (v, "v", 4), (o_branch, "o_branch", 4), (dout, "dout", 4)):
        _need(t, n, torch.bfloat16, nd)
    _need(lam, "lam", torch.float32, 3)
    _need(lse, "lse", torch.float32, 3)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    dlam = torch.empty_like(lam) if dlam is None else dlam
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, n, torch.bfloat16, 4)
    _need(dlam, "dlam", torch.float32, 3)
    ws_bytes = backward_workspace_size(B, S, Hq)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    if window is not None:
        st = LIB.diffattn_v2_backward_window(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(o_branch), _ptr(lse),
                                             _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlam), B, S, Hq, Hkv, D,
                                             int(window), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                             _stream(stream, q.device))
        _check(st, "diffattn_v2_backward_window")
        return dq, dk, dv, dlam
    st = LIB.diffattn_v2_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(o_branch), _ptr(lse), _ptr(dout),
                                  _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlam), B, S, Hq, Hkv, D, 1 if causal else 0,
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream, q.device))
    _check(st, "diffattn_v2_backward")
    return dq, dk, dv, dlam


def prefill_varlen_train(q, k, v, lam, cu_seqlens, max_seqlen, out=None, o_branch=None, lse=None, causal=True,
                         stream=None, window=None):
    """Training forward of packed sequences (layouts of prefill_varlen): returns
    (out [T,Hq/2,D], o_branch [T,Hq,D], lse [T,Hq]). With `window` the causal sliding window
    inside every sequence."""
    for t, n, nd in ((q, "q", 3), (k, "k", 3), (v, "v", 3)):
        _need(t, n, torch.bfloat16, nd)
    _need(lam, "lam", torch.float32, 2)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    out = torch.empty((T, Hq // 2, D), dtype=torch.bfloat16, device=q.device) if out is None else out
    o_branch = torch.empty((T, Hq, D), dtype=torch.bfloat16, device=q.device) if o_branch is None else o_branch
    lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    _need(out, "out", torch.bfloat16, 3)
    _need(o_branch, "o_branch", torch.bfloat16, 3)
    _need(lse, "lse", torch.float32, 2)
    if window is not None:
        st = LIB.diffattn_v2_prefill_varlen_window_train(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out),
                                                         _ptr(o_branch), _ptr(lse), _ptr(cu_seqlens), B,
                                                         int(max_seqlen), T, Hq, Hkv, D, int(window),
                                                         _stream(stream, q.device))
        _check(st, "diffattn_v2_prefill_varlen_window_train")
        return out, o_branch, lse
    st = LIB.diffattn_v2_prefill_varlen_train(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), _ptr(o_branch),
                                              _ptr(lse), _ptr(cu_seqlens), B, int(max_seqlen), T, Hq, Hkv, D,
                                              1 if causal else 0, _stream(stream, q.device))
    _check(st, "diffattn_v2_prefill_varlen_train")
    return out, o_branch, lse


def backward_varlen_workspace_size(B, total_tokens, Hq) -> int:
    return int(LIB.diffattn_v2_backward_varlen_workspace_size(B, total_tokens, Hq))


def backward_varlen(q, k, v, lam, o_branch, lse, dout, cu_seqlens, max_seqlen, causal=True, workspace=None,
                    stream=None, window=None):
    """Gradients of the packed-sequence prefill: returns (dq, dk, dv, dlam) in the packed layouts.
    With `window` the gradients of the causal sliding-window packed prefill."""
    for t, n, nd in ((q, "q", 3), (k, "k", 3), (v, "v", 3), (o_branch, "o_branch", 3), (dout, "dout", 3)):
        _need(t, n, torch.bfloat16, nd)
    _need(lam, "lam", torch.float32, 2)
    _need(lse, "lse", torch.float32, 2)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    dq, dk, dv, dlam = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(lam)
    ws_bytes = backward_varlen_workspace_size(B, T, Hq)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    ws_given = workspace.numel() * workspace.element_size()
    if window is not None:
        st = LIB.diffattn_v2_backward_varlen_window(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(o_branch), _ptr(lse),
                                                    _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlam),
                                                    _ptr(cu_seqlens), B, int(max_seqlen), T, Hq, Hkv, D, int(window),
                                                    _ptr(workspace), ws_given, _stream(stream, q.device))
        _check(st, "diffattn_v2_backward_varlen_window")
        return dq, dk, dv, dlam
    st = LIB.diffattn_v2_backward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(o_branch), _ptr(lse),
                                         _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlam), _ptr(cu_seqlens), B,
                                         int(max_seqlen), T, Hq, Hkv, D, 1 if causal else 0, _ptr(workspace),
                                         ws_given, _stream(stream, q.device))
    _check(st, "diffattn_v2_backward_varlen")
    return dq, dk, dv, dlam


def decode_workspace_size(B, Smax, Hq, Hkv, D) -> int:
    return int(LIB.diffattn_v2_decode_workspace_size(B, Smax, Hq, Hkv, D))


def decode(q, kcache, vcache, seqlens, lam, out=None, workspace=None, stream=None, window=None):
    """bf16 decode step: q [B,Hq,D], caches [B,Smax,Hkv,D], seqlens int32 [B], lam fp32 [B,Hq/2].
    With `window` the new token sees only its sequence's last `window` keys."""
    _need(q, "q", torch.bfloat16, 3)
    _need(kcache, "kcache", torch.bfloat16, 4)
    _need(vcache, "vcache", torch.bfloat16, 4)
    _need(seqlens, "seqlens", torch.int32, 1)
    _need(lam, "lam", torch.float32, 2)
    B, Hq, D = q.shape
    Smax, Hkv = kcache.shape[1], kcache.shape[2]
    if out is None:
        out = torch.empty((B, Hq // 2, D), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 3)
    need = decode_workspace_size(B, Smax, Hq, Hkv, D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if window is not None:
        st = LIB.diffattn_v2_decode_window(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(lam), _ptr(out), B,
                                           Smax, Hq, Hkv, D, int(window), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), _stream(stream, q.device))
        _check(st, "diffattn_v2_decode_window")
        return out
    st = LIB.diffattn_v2_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(lam), _ptr(out), B, Smax,
                                Hq, Hkv, D, _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream, q.device))
    _check(st, "diffattn_v2_decode")
    return out


def decode_multi(q, kcache, vcache, seqlens, lam, out=None, workspace=None, stream=None):
    """bf16 decode of T new tokens per sequence: q [B,T,Hq,D], lam fp32 [B,T,Hq/2] ->
    out bf16 [B,T,Hq/2,D]; token t sees keys [0, seqlens[b] - T + t + 1)."""
    _need(q, "q", torch.bfloat16, 4)
    _need(kcache, "kcache", torch.bfloat16, 4)
    _need(vcache, "vcache", torch.bfloat16, 4)
    _need(seqlens, "seqlens", torch.int32, 1)
    _need(lam, "lam", torch.float32, 3)
    B, T, Hq, D = q.shape
    Smax, Hkv = kcache.shape[1], kcache.shape[2]
    if out is None:
        out = torch.empty((B, T, Hq // 2, D), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    need = int(LIB.diffattn_v2_decode_multi_workspace_size(B, T, Smax, Hq, Hkv, D))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = LIB.diffattn_v2_decode_multi(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(lam), _ptr(out), B, T,
                                      Smax, Hq, Hkv, D, _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream(stream, q.device))
    _check(st, "diffattn_v2_decode_multi")
    return out


def decode_paged(q, kpages, vpages, block_table, seqlens, lam, out=None, workspace=None, stream=None, window=None):
    """bf16 decode over a paged cache: kpages/vpages [num_pages, page_size, Hkv, D],
    block_table int32 [B, max_pages], seqlens int32 [B], lam fp32 [B, Hq/2]. With `window`
    the new token sees only its sequence's last `window` keys."""
    _need(q, "q", torch.bfloat16, 3)
    _need(kpages, "kpages", torch.bfloat16, 4)
    _need(vpages, "vpages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seqlens, "seqlens", torch.int32, 1)
    _need(lam, "lam", torch.float32, 2)
    B, Hq, D = q.shape
    num_pages, page_size, Hkv = kpages.shape[0], kpages.shape[1], kpages.shape[2]
    max_pages = block_table.shape[1]
    if out is None:
        out = torch.empty((B, Hq // 2, D), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 3)
    need = decode_workspace_size(B, max_pages * page_size, Hq, Hkv, D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if window is not None:
        st = LIB.diffattn_v2_decode_paged_window(_ptr(q), _ptr(kpages), _ptr(vpages), _ptr(block_table), _ptr(seqlens),
                                                 _ptr(lam), _ptr(out), B, max_pages, page_size, num_pages, Hq, Hkv, D,
                                                 int(window), _ptr(workspace),
                                                 workspace.numel() * workspace.element_size(), _stream(stream, q.device))
        _check(st, "diffattn_v2_decode_paged_window")
        return out
    st = LIB.diffattn_v2_decode_paged(_ptr(q), _ptr(kpages), _ptr(vpages), _ptr(block_table), _ptr(seqlens), _ptr(lam),
                                      _ptr(out), B, max_pages, page_size, num_pages, Hq, Hkv, D, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream, q.device))
    _check(st, "diffattn_v2_decode_paged")
    return out


def decode_f32(q, kcache, vcache, seqlens, lam, out=None, stream=None):
    """fp32 decode step on CUDA cores; same layout as decode with fp32 tensors."""
    _need(q, "q", torch.float32, 3)
    _need(kcache, "kcache", torch.float32, 4)
    _need(vcache, "vcache", torch.float32, 4)
    _need(seqlens, "seqlens", torch.int32, 1)
    _need(lam, "lam", torch.float32, 2)
    B, Hq, D = q.shape
    Smax, Hkv = kcache.shape[1], kcache.shape[2]
    if out is None:
        out = torch.empty((B, Hq // 2, D), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, 3)
    st = LIB.diffattn_v2_decode_f32(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(lam), _ptr(out), B,
                                    Smax, Hq, Hkv, D, _stream(stream, q.device))
    _check(st, "diffattn_v2_decode_f32")
    return out


def lambda_v1(lq1, lk1, lq2, lk2, lambda_init=0.8, rows=1, out=None, stream=None):
    """V1 lambda per pair, broadcast to `rows` rows: out fp32 [rows, n_pairs]."""
    for t, n in ((lq1, "lq1"), (lk1, "lk1"), (lq2, "lq2"), (lk2, "lk2")):
        _need(t, n, torch.float32, 2)
    n_pairs, d = lq1.shape
    if out is None:
        out = torch.empty((rows, n_pairs), dtype=torch.float32, device=lq1.device)
    if out.dtype != torch.float32 or not out.is_contiguous() or out.numel() != rows * n_pairs:
        raise ValueError("out must be a contiguous fp32 tensor with rows*n_pairs elements")
    st = LIB.diffattn_v2_lambda_v1(_ptr(lq1), _ptr(lk1), _ptr(lq2), _ptr(lk2), float(lambda_init), n_pairs, d, rows,
                                   _ptr(out), _stream(stream, lq1.device))
    _check(st, "diffattn_v2_lambda_v1")
    return out


def lambda_v2(x, w_lambda, bias=None, out=None, stream=None):
    """V2 lambda sigmoid(x @ w_lambda + bias): x bf16 [T, d_model], w_lambda bf16
    [d_model, n_pairs], bias fp32 [n_pairs] or None -> fp32 [T, n_pairs]."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w_lambda, "w_lambda", torch.bfloat16, 2)
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    T, d = x.shape
    n_pairs = w_lambda.shape[1]
    if out is None:
        out = torch.empty((T, n_pairs), dtype=torch.float32, device=x.device)
    st = LIB.diffattn_v2_lambda_v2(_ptr(x), _ptr(w_lambda), _ptr(bias), T, d, n_pairs, _ptr(out),
                                   _stream(stream, x.device))
    _check(st, "diffattn_v2_lambda_v2")
    return out


def prefill_fused_lambda(q, k, v, x, w_lambda_t, bias=None, out=None, lambda_out=None, causal=True, stream=None):
    """bf16 prefill with the V2 lambda sigmoid(x . w_lambda_t[p] + bias[p]) computed inside the
    kernel: q [B,S,Hq,D], k/v [B,S,Hkv,D], x bf16 [B,S,d_model], w_lambda_t bf16 [Hq/2, d_model]
    (the projection transposed), bias fp32 [Hq/2] or None; lambda_out fp32 [B,S,Hq/2] receives
    the lambda when given. Returns out bf16 [B,S,Hq/2,D]."""
    for t, n, nd in ((q, "q", 4), (k, "k", 4), (v, "v", 4), (x, "x", 3), (w_lambda_t, "w_lambda_t", 2)):
        _need(t, n, torch.bfloat16, nd)
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if lambda_out is not None:
        _need(lambda_out, "lambda_out", torch.float32, 3)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    d_model = x.shape[2]
    if out is None:
        out = torch.empty((B, S, Hq // 2, D), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    st = LIB.diffattn_v2_prefill_fused_lambda(_ptr(q), _ptr(k), _ptr(v), _ptr(x), _ptr(w_lambda_t), _ptr(bias),
                                              _ptr(out), _ptr(lambda_out), B, S, Hq, Hkv, D, d_model,
                                              1 if causal else 0, _stream(stream, q.device))
    _check(st, "diffattn_v2_prefill_fused_lambda")
    return out


def device_error(stream=None, device=None) -> int:
    """Synchronise the stream and return (and clear) the kernels' device error word."""
    code = ctypes.c_int(0)
    st = LIB.diffattn_v2_device_error(ctypes.byref(code), _stream(stream, device))
    if st == ERR_CUDA:
        raise DiffAttnError(st, "diffattn_v2_device_error")
    return code.value


def decode_noalloc(q, kcache, vcache, seqlens, lam, out=None, stream=None):
    """bf16 decode step whose partials live in the library's fixed 16 MiB device array.

    For callers that cannot allocate device memory (a KV-cache pool or caching allocator
    that owns nearly all HBM, plugin interfaces without a workspace). The library allocates
    nothing; calls that overlap on the GPU share the array and race, so serialise them.
    Sizes needing more than 16 MiB of partials raise (DA2_ERR_UNSUPPORTED)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(kcache, "kcache", torch.bfloat16, 4)
    _need(vcache, "vcache", torch.bfloat16, 4)
    _need(seqlens, "seqlens", torch.int32, 1)
    _need(lam, "lam", torch.float32, 2)
    B, Hq, D = q.shape
    Smax, Hkv = kcache.shape[1], kcache.shape[2]
    if out is None:
        out = torch.empty((B, Hq // 2, D), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 3)
    st = LIB.diffattn_v2_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(lam), _ptr(out),
                                        B, Smax, Hq, Hkv, D, _stream(stream, q.device))
    _check(st, "diffattn_v2_decode_noalloc")
    return out
