"""Thin Python binding of libwkv7.so (argument marshalling only).

Every step of the recurrence runs in the library's CUDA kernels; this module
only checks tensors, allocates outputs with PyTorch and passes raw device
pointers plus the current CUDA stream through the C ABI declared in
``include/wkv7.h``.  There is no CPU or PyTorch fallback: if the library is
missing or the tensors are not on a CUDA device, the call raises.

Names follow the C ABI: ``wkv7_fwd`` (generalized_delta_rule /
generalized_delta_rule_inference, forward only) and ``wkv7_step``
(rwkv7_op_rnn) -- rwkv-ops 0.9.0 README, sections "rwkv7op 使用方法" and
"rwkv7_op_rnn 使用方法"; ``wkv7_gdn_fwd`` / ``wkv7_gdn_step`` (Gated DeltaNet:
gated_delta_net_recurrent / _chunk / _single_step, same README, "gdn_recurrent
使用方法" and "gdn_chunk 使用方法").
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwkv7.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_DEVICE_BAD_SEQLENS = range(6)
BF16, F32 = 0, 1
ALGO = {"auto": 0, "recurrent": 1, "chunked": 2}

_lib = None


class WKV7Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def library() -> ctypes.CDLL:
    """Load libwkv7.so (built in-tree by ``build.py``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libwkv7.so not built ({LIB_PATH}); run "
                              "python -m linear_attention_rnn_wkv7_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        p, i = ctypes.c_void_p, ctypes.c_int
        lib.wkv7_fwd.restype = i
        lib.wkv7_fwd.argtypes = [p, p, p, p, p, p, p, p, p, p, i, i, i, i, i, p, i, i, i, i, p]
        lib.wkv7_step.restype = i
        lib.wkv7_step.argtypes = [p, p, p, p, p, p, p, p, i, i, i, i, i, p]
        lib.wkv7_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.wkv7_bwd_workspace_bytes.argtypes = [i, i, i, i, i, i]
        lib.wkv7_bwd.restype = i
        lib.wkv7_bwd.argtypes = [p] * 17 + [i, i, i, i, i, p, i, i, i, p, ctypes.c_size_t, p]
        lib.wkv7_bwd_workspace_bytes_algo.restype = ctypes.c_size_t
        lib.wkv7_bwd_workspace_bytes_algo.argtypes = [i] * 8
        lib.wkv7_bwd_with_algo.restype = i
        lib.wkv7_bwd_with_algo.argtypes = ([p] * 17 + [i, i, i, i, i, p, i, i, i, i, p,
                                                       ctypes.c_size_t, p])
        lib.wkv7_bwd_noalloc.restype = i
        lib.wkv7_bwd_noalloc.argtypes = [p] * 17 + [i, i, i, i, i, p, i, i, i, p]
        lib.wkv7_gdn_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.wkv7_gdn_bwd_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
        lib.wkv7_gdn_bwd.restype = i
        lib.wkv7_gdn_bwd.argtypes = ([p] * 6 + [i] + [p] * 8 + [i] * 5 + [p, i, i, i, p,
                                                                         ctypes.c_size_t, p])
        lib.wkv7_gdn_fwd.restype = i
        lib.wkv7_gdn_fwd.argtypes = [p, p, p, p, p, p, i, p, p, i, i, i, i, i, p, i, i, i, i, p]
        lib.wkv7_gdn_step.restype = i
        lib.wkv7_gdn_step.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, p]
        lib.wkv7_get_last_error.restype = i
        lib.wkv7_get_last_error.argtypes = [p]
        lib.wkv7_status_string.restype = ctypes.c_char_p
        lib.wkv7_status_string.argtypes = [i]
        lib.wkv7_version.restype = i
        lib.wkv7_version.argtypes = []
        lib.wkv7_test_stall_next_chunked.restype = i
        lib.wkv7_test_stall_next_chunked.argtypes = [i]
        lib.wkv7_test_chunked_schedule.restype = i
        lib.wkv7_test_chunked_schedule.argtypes = [ctypes.c_longlong, i, ctypes.POINTER(i),
                                                   ctypes.POINTER(ctypes.c_longlong),
                                                   ctypes.POINTER(ctypes.c_longlong)]
        lib.wkv7_sane_fwd.restype = i
        lib.wkv7_sane_fwd.argtypes = [p] * 9 + [i, p, p, i, i, i, i, i, i, i, p]
        lib.wkv7_sane_step.restype = i
        lib.wkv7_sane_step.argtypes = [p] * 8 + [i, p, p, i, i, i, i, i, p]
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().wkv7_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype} (bfloat16 or float32)")


def _check(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def wkv7_fwd(r, w, k, v, a, b, s0=None, mask=None, cu_seqlens=None,
             output_final_state: bool = True, algo: str = "auto", o=None, sT=None,
             head_first: bool = False):
    """WKV7 forward.  r,w,k,a,b [B,T,H,K]; v [B,T,H,V] (bf16 or fp32, all alike), or
    [B,H,T,*] with head_first; s0 [N,H,K,V] fp32 or None; mask [B,T] uint8/bool or
    None; cu_seqlens [N+1] int32 (B must be 1) or None.
    Returns (o shaped like v, sT [N,H,K,V] or None)."""
    _check(r, "r")
    dt = r.dtype
    if head_first:
        B, H, T, K = r.shape
    else:
        B, T, H, K = r.shape
    V = v.shape[-1]
    kshape = (B, H, T, K) if head_first else (B, T, H, K)
    vshape = (B, H, T, V) if head_first else (B, T, H, V)
    for name, t in (("w", w), ("k", k), ("a", a), ("b", b)):
        _check(t, name, dt, kshape)
    _check(v, "v", dt, vshape)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if s0 is not None:
        _check(s0, "s0", torch.float32, (N, H, K, V))
    if mask is not None:
        if mask.dtype == torch.bool:
            mask = mask.to(torch.uint8)
        _check(mask, "mask", torch.uint8, (B, T))
    if o is None:
        o = torch.empty(vshape, dtype=dt, device=r.device)
    else:
        _check(o, "o", dt, vshape)
    if output_final_state and sT is None:
        sT = torch.empty((N, H, K, V), dtype=torch.float32, device=r.device)
    elif sT is not None:
        _check(sT, "sT", torch.float32, (N, H, K, V))
    st = library().wkv7_fwd(_ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0),
                            _ptr(mask), _ptr(o), _ptr(sT), B, T, H, K, V, _ptr(cu_seqlens), N,
                            int(bool(head_first)), _dtype_code(r), ALGO[algo], _stream(r.device))
    if st != OK:
        raise WKV7Error(st, "wkv7_fwd")
    return o, sT


def wkv7_step(r, w, k, v, a, b, state, o=None):
    """One decode token.  r,w,k,a,b [B,H,K]; v [B,H,V]; state [B,H,K,V] fp32,
    updated in place.  Returns o [B,H,V] (dtype of the inputs)."""
    _check(r, "r")
    dt = r.dtype
    B, H, K = r.shape
    V = v.shape[-1]
    for name, t in (("w", w), ("k", k), ("a", a), ("b", b)):
        _check(t, name, dt, (B, H, K))
    _check(v, "v", dt, (B, H, V))
    _check(state, "state", torch.float32, (B, H, K, V))
    if o is None:
        o = torch.empty((B, H, V), dtype=dt, device=r.device)
    else:
        _check(o, "o", dt, (B, H, V))
    st = library().wkv7_step(_ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(state),
                             _ptr(o), B, H, K, V, _dtype_code(r), _stream(r.device))
    if st != OK:
        raise WKV7Error(st, "wkv7_step")
    return o


def _flags_u8(x, name, shape):
    """A 0/1 flag tensor (bool, uint8 or float 0/1, as the README's SANE flags) as uint8."""
    if x.dtype != torch.uint8:
        x = (x != 0).to(torch.uint8)
    _check(x.contiguous(), name, torch.uint8, shape)
    return x.contiguous()


def wkv7_sane_fwd(r, w, k, v, a, b, tau, sane_mask=None, s0=None,
                  output_final_state: bool = True, o=None, sT=None, head_first: bool = False):
    """WKV7 forward with State Anomaly Neutralization (generalized_delta_rule_sane): the
    state is soft-clipped, S <- tau * tanh(S / tau), after every full 16-token chunk
    whose flag is set; outputs are read before the clip.  r,w,k,a,b [B,T,H,K], v
    [B,T,H,V] (or [B,H,T,*] with head_first), bf16 or fp32; tau [B,T//16,H] fp32 > 0;
    sane_mask [B,T//16] (bool / uint8 / float 0-1) or None (every chunk); s0 [B,H,K,V]
    or [1,H,K,V] fp32 or None.  Returns (o shaped like v, sT [B,H,K,V] or None).
    Unlike the README's wrapper, the final state is returned whenever asked for, with or
    without sane_mask."""
    _check(r, "r")
    dt = r.dtype
    if head_first:
        B, H, T, K = r.shape
    else:
        B, T, H, K = r.shape
    V = v.shape[-1]
    kshape = (B, H, T, K) if head_first else (B, T, H, K)
    vshape = (B, H, T, V) if head_first else (B, T, H, V)
    for name, t in (("w", w), ("k", k), ("a", a), ("b", b)):
        _check(t, name, dt, kshape)
    _check(v, "v", dt, vshape)
    C = T // 16
    _check(tau, "tau", torch.float32, (B, C, H))
    if sane_mask is not None:
        sane_mask = _flags_u8(sane_mask, "sane_mask", (B, C))
    shared = 0
    if s0 is not None:
        _check(s0, "s0", torch.float32)
        if tuple(s0.shape) == (1, H, K, V) and B != 1:
            shared = 1
        elif tuple(s0.shape) != (B, H, K, V):
            raise ValueError(f"s0 must have shape {(B, H, K, V)} or {(1, H, K, V)}")
    if o is None:
        o = torch.empty(vshape, dtype=dt, device=r.device)
    else:
        _check(o, "o", dt, vshape)
    if output_final_state and sT is None:
        sT = torch.empty((B, H, K, V), dtype=torch.float32, device=r.device)
    elif sT is not None:
        _check(sT, "sT", torch.float32, (B, H, K, V))
    st = library().wkv7_sane_fwd(_ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                 _ptr(tau), _ptr(sane_mask), _ptr(s0), shared, _ptr(o), _ptr(sT),
                                 B, T, H, K, V, int(bool(head_first)), _dtype_code(r),
                                 _stream(r.device))
    if st != OK:
        raise WKV7Error(st, "wkv7_sane_fwd")
    return o, sT


def wkv7_sane_step(r, w, k, v, a, b, tau, do_sane, state, o=None):
    """One decode token with State Anomaly Neutralization (rwkv7_op_sane_rnn).
    r,w,k,a,b [B,H,K]; v [B,H,V]; tau [B,H] fp32 > 0; do_sane a bool (every row) or a
    [B] flag tensor; state [B,H,K,V] fp32, updated in place (clipped where flagged).
    Returns o [B,H,V], read from the state before the clip."""
    _check(r, "r")
    dt = r.dtype
    B, H, K = r.shape
    V = v.shape[-1]
    for name, t in (("w", w), ("k", k), ("a", a), ("b", b)):
        _check(t, name, dt, (B, H, K))
    _check(v, "v", dt, (B, H, V))
    _check(tau, "tau", torch.float32, (B, H))
    _check(state, "state", torch.float32, (B, H, K, V))
    flags, every = None, 0
    if isinstance(do_sane, torch.Tensor):
        flags = _flags_u8(do_sane, "do_sane", (B,))
    else:
        every = int(bool(do_sane))
    if o is None:
        o = torch.empty((B, H, V), dtype=dt, device=r.device)
    else:
        _check(o, "o", dt, (B, H, V))
    st = library().wkv7_sane_step(_ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                  _ptr(tau), _ptr(flags), every, _ptr(state), _ptr(o), B, H, K,
                                  V, _dtype_code(r), _stream(r.device))
    if st != OK:
        raise WKV7Error(st, "wkv7_sane_step")
    return o


def wkv7_bwd_workspace_bytes(B, T, H, K=64, V=64, N=None, dtype=None, algo: str = None) -> int:
    """Workspace bytes of wkv7_bwd: with dtype (torch.bfloat16 / torch.float32) and algo,
    the need of the kernel family that runs; without, the larger of the two."""
    N = B if N is None else N
    if dtype is None and algo is None:
        return int(library().wkv7_bwd_workspace_bytes(B, T, H, K, V, N))
    code = 0 if (dtype is None or dtype == torch.bfloat16) else 1
    return int(library().wkv7_bwd_workspace_bytes_algo(B, T, H, K, V, N, code,
                                                        ALGO[algo or "auto"]))


def wkv7_bwd(r, w, k, v, a, b, dout, s0=None, mask=None, dsT=None, cu_seqlens=None,
             head_first: bool = False, workspace=None, algo: str = "auto"):
    """Backward of wkv7_fwd for L = sum(o * dout) + sum(S_T * dsT).  Inputs as for
    wkv7_fwd (K = V = 64); dout shaped like v; dsT [N,H,K,V] fp32 or None.
    Returns a dict: dr, dw, dk, dv, da, db (input dtype, shaped like the inputs) and
    ds0 (fp32 [N,H,K,V]).  The workspace (uint8 device tensor of at least
    wkv7_bwd_workspace_bytes) is allocated here when not given.  algo: "auto" (the
    tensor-core chunked form for bf16, the fp32 recurrences for fp32), "chunked"
    (bf16 only) or "recurrent"."""
    _check(r, "r")
    dt = r.dtype
    if head_first:
        B, H, T, K = r.shape
    else:
        B, T, H, K = r.shape
    V = v.shape[-1]
    kshape = (B, H, T, K) if head_first else (B, T, H, K)
    vshape = (B, H, T, V) if head_first else (B, T, H, V)
    for name, t in (("w", w), ("k", k), ("a", a), ("b", b)):
        _check(t, name, dt, kshape)
    _check(v, "v", dt, vshape)
    _check(dout, "dout", dt, vshape)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if s0 is not None:
        _check(s0, "s0", torch.float32, (N, H, K, V))
    if dsT is not None:
        _check(dsT, "dsT", torch.float32, (N, H, K, V))
    if mask is not None:
        if mask.dtype == torch.bool:
            mask = mask.to(torch.uint8)
        _check(mask, "mask", torch.uint8, (B, T))
    nbytes = wkv7_bwd_workspace_bytes(B, T, H, K, V, N, dtype=dt, algo=algo)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=r.device)
    else:
        _check(workspace, "workspace", torch.uint8)
    g = {n: torch.empty(kshape, dtype=dt, device=r.device) for n in ("dr", "dw", "dk", "da", "db")}
    g["dv"] = torch.empty(vshape, dtype=dt, device=r.device)
    g["ds0"] = torch.empty((N, H, K, V), dtype=torch.float32, device=r.device)
    st = library().wkv7_bwd_with_algo(
        _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0), _ptr(mask), _ptr(dout),
        _ptr(dsT), _ptr(g["dr"]), _ptr(g["dw"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["da"]),
        _ptr(g["db"]), _ptr(g["ds0"]), B, T, H, K, V, _ptr(cu_seqlens), N,
        int(bool(head_first)), _dtype_code(r), ALGO[algo], _ptr(workspace), workspace.numel(),
        _stream(r.device))
    if st != OK:
        raise WKV7Error(st, "wkv7_bwd")
    return g


def wkv7_bwd_noalloc(r, w, k, v, a, b, dout, s0=None, mask=None, dsT=None, cu_seqlens=None,
                     head_first: bool = False):
    """wkv7_bwd on the library's static scratch (no workspace argument; small problems
    only -- larger ones raise WKV7Error with WKV7_ERR_UNSUPPORTED).  Same results."""
    _check(r, "r")
    dt = r.dtype
    if head_first:
        B, H, T, K = r.shape
    else:
        B, T, H, K = r.shape
    V = v.shape[-1]
    kshape = (B, H, T, K) if head_first else (B, T, H, K)
    vshape = (B, H, T, V) if head_first else (B, T, H, V)
    for name, t in (("w", w), ("k", k), ("a", a), ("b", b)):
        _check(t, name, dt, kshape)
    _check(v, "v", dt, vshape)
    _check(dout, "dout", dt, vshape)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if s0 is not None:
        _check(s0, "s0", torch.float32, (N, H, K, V))
    if dsT is not None:
        _check(dsT, "dsT", torch.float32, (N, H, K, V))
    if mask is not None:
        if mask.dtype == torch.bool:
            mask = mask.to(torch.uint8)
        _check(mask, "mask", torch.uint8, (B, T))
    g = {n: torch.empty(kshape, dtype=dt, device=r.device) for n in ("dr", "dw", "dk", "da", "db")}
    g["dv"] = torch.empty(vshape, dtype=dt, device=r.device)
    g["ds0"] = torch.empty((N, H, K, V), dtype=torch.float32, device=r.device)
    for name, t in (("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("dout", dout),
                    ("s0", s0), ("dsT", dsT), ("mask", mask), ("cu_seqlens", cu_seqlens)):
        if t is not None and t.device != r.device:
            raise ValueError(f"{name} is on {t.device}, r on {r.device}: one device only")
    # The library's static scratch is per device: the call must run with r's device
    # current, which is also the device of the stream passed.
    with torch.cuda.device(r.device):
        st = library().wkv7_bwd_noalloc(_ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                        _ptr(s0), _ptr(mask), _ptr(dout), _ptr(dsT),
                                        _ptr(g["dr"]), _ptr(g["dw"]), _ptr(g["dk"]),
                                        _ptr(g["dv"]), _ptr(g["da"]), _ptr(g["db"]),
                                        _ptr(g["ds0"]), B, T, H, K, V, _ptr(cu_seqlens), N,
                                        int(bool(head_first)), _dtype_code(r),
                                        _stream(r.device))
    if st != OK:
        raise WKV7Error(st, "wkv7_bwd_noalloc")
    return g


class GeneralizedDeltaRule(torch.autograd.Function):
    """generalized_delta_rule as a differentiable op: forward through wkv7_fwd, backward
    through wkv7_bwd (token-major inputs, K = V = 64, no varlen)."""

    @staticmethod
    def forward(ctx, r, w, k, v, a, b, s0, mask, cu_seqlens, head_first):
        o, sT = wkv7_fwd(r, w, k, v, a, b, s0=s0, mask=mask, cu_seqlens=cu_seqlens,
                         head_first=head_first)
        ctx.save_for_backward(r, w, k, v, a, b, s0, mask, cu_seqlens)
        ctx.head_first = head_first
        return o, sT

    @staticmethod
    def backward(ctx, do, dsT):
        r, w, k, v, a, b, s0, mask, cu_seqlens = ctx.saved_tensors
        do = torch.zeros_like(v) if do is None else do.contiguous()
        dsT = None if dsT is None else dsT.contiguous().float()
        g = wkv7_bwd(r, w, k, v, a, b, do.to(r.dtype), s0=s0, mask=mask, dsT=dsT,
                     cu_seqlens=cu_seqlens, head_first=ctx.head_first)
        ds0 = g["ds0"] if s0 is not None else None
        return g["dr"], g["dw"], g["dk"], g["dv"], g["da"], g["db"], ds0, None, None, None


def generalized_delta_rule(r, w, k, v, a, b, initial_state=None, output_final_state=True,
                           mask=None, cu_seqlens=None, head_first: bool = False):
    """Differentiable forward (README: generalized_delta_rule); returns (o, final state or
    None).  Backward through wkv7_bwd."""
    o, sT = GeneralizedDeltaRule.apply(r, w, k, v, a, b, initial_state, mask, cu_seqlens,
                                       head_first)
    return o, (sT if output_final_state else None)


def wkv7_gdn_fwd(q, k, v, g, beta, s0=None, cu_seqlens=None, output_final_state: bool = True,
                 algo: str = "auto", o=None, sT=None, head_first: bool = False):
    """Gated DeltaNet forward.  q, k [B,T,H,K]; v [B,T,H,V]; g, beta [B,T,H] (bf16 or
    fp32, all alike), or [B,H,T,*] / [B,H,T] with head_first; s0 [N,H,K,V] or
    [1,H,K,V] (shared) fp32 or None; cu_seqlens [N+1] int32 (B must be 1) or None.
    Returns (o shaped like v, sT [N,H,K,V] or None)."""
    _check(q, "q")
    dt = q.dtype
    if head_first:
        B, H, T, K = q.shape
    else:
        B, T, H, K = q.shape
    V = v.shape[-1]
    kshape = (B, H, T, K) if head_first else (B, T, H, K)
    vshape = (B, H, T, V) if head_first else (B, T, H, V)
    _check(k, "k", dt, kshape)
    _check(v, "v", dt, vshape)
    _check(g, "g", dt, kshape[:3])
    _check(beta, "beta", dt, kshape[:3])
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    shared = 0
    if s0 is not None:
        _check(s0, "s0", torch.float32)
        if tuple(s0.shape) == (1, H, K, V) and N != 1:
            shared = 1
        elif tuple(s0.shape) != (N, H, K, V):
            raise ValueError(f"s0 must have shape {(N, H, K, V)} or {(1, H, K, V)}")
    if o is None:
        o = torch.empty(vshape, dtype=dt, device=q.device)
    else:
        _check(o, "o", dt, vshape)
    if output_final_state and sT is None:
        sT = torch.empty((N, H, K, V), dtype=torch.float32, device=q.device)
    elif sT is not None:
        _check(sT, "sT", torch.float32, (N, H, K, V))
    st = library().wkv7_gdn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0), shared,
                                _ptr(o), _ptr(sT), B, T, H, K, V, _ptr(cu_seqlens), N,
                                int(bool(head_first)), _dtype_code(q), ALGO[algo],
                                _stream(q.device))
    if st != OK:
        raise WKV7Error(st, "wkv7_gdn_fwd")
    return o, sT


def wkv7_gdn_step(q, k, v, g, beta, state, o=None):
    """One Gated DeltaNet decode token.  q, k [B,H,K]; v [B,H,V]; g, beta [B,H];
    state [B,H,K,V] fp32, updated in place.  Returns o [B,H,V]."""
    _check(q, "q")
    dt = q.dtype
    B, H, K = q.shape
    V = v.shape[-1]
    _check(k, "k", dt, (B, H, K))
    _check(v, "v", dt, (B, H, V))
    _check(g, "g", dt, (B, H))
    _check(beta, "beta", dt, (B, H))
    _check(state, "state", torch.float32, (B, H, K, V))
    if o is None:
        o = torch.empty((B, H, V), dtype=dt, device=q.device)
    else:
        _check(o, "o", dt, (B, H, V))
    st = library().wkv7_gdn_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
                                 _ptr(o), B, H, K, V, _dtype_code(q), _stream(q.device))
    if st != OK:
        raise WKV7Error(st, "wkv7_gdn_step")
    return o


def wkv7_get_last_error(device=None) -> int:
    """Synchronise the current stream; return and clear the device-side flag."""
    return library().wkv7_get_last_error(_stream(device))


def wkv7_gdn_bwd(q, k, v, g, beta, dout, s0=None, dsT=None, cu_seqlens=None,
                 head_first: bool = False, workspace=None):
    """Backward of wkv7_gdn_fwd for L = sum(o * dout) + sum(S_T * dsT).  Returns a dict:
    dq, dk, dv, dg, dbeta (input dtype, shaped like the inputs) and ds0 (fp32, shaped
    like s0; [N,H,K,V] when s0 is None)."""
    _check(q, "q")
    dt = q.dtype
    if head_first:
        B, H, T, K = q.shape
    else:
        B, T, H, K = q.shape
    V = v.shape[-1]
    kshape = (B, H, T, K) if head_first else (B, T, H, K)
    vshape = (B, H, T, V) if head_first else (B, T, H, V)
    _check(k, "k", dt, kshape)
    _check(v, "v", dt, vshape)
    _check(g, "g", dt, kshape[:3])
    _check(beta, "beta", dt, kshape[:3])
    _check(dout, "dout", dt, vshape)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    shared = 0
    if s0 is not None:
        _check(s0, "s0", torch.float32)
        if tuple(s0.shape) == (1, H, K, V) and N != 1:
            shared = 1
        elif tuple(s0.shape) != (N, H, K, V):
            raise ValueError(f"s0 must have shape {(N, H, K, V)} or {(1, H, K, V)}")
    if dsT is not None:
        _check(dsT, "dsT", torch.float32, (N, H, K, V))
    nbytes = int(library().wkv7_gdn_bwd_workspace_bytes(B, T, H, K, V, N, _dtype_code(q), shared))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    else:
        _check(workspace, "workspace", torch.uint8)
    out = {"dq": torch.empty(kshape, dtype=dt, device=q.device),
           "dk": torch.empty(kshape, dtype=dt, device=q.device),
           "dv": torch.empty(vshape, dtype=dt, device=q.device),
           "dg": torch.empty(kshape[:3], dtype=dt, device=q.device),
           "dbeta": torch.empty(kshape[:3], dtype=dt, device=q.device),
           "ds0": torch.empty(tuple(s0.shape) if s0 is not None else (N, H, K, V),
                              dtype=torch.float32, device=q.device)}
    st = library().wkv7_gdn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0), shared,
                                _ptr(dout), _ptr(dsT), _ptr(out["dq"]), _ptr(out["dk"]),
                                _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
                                _ptr(out["ds0"]), B, T, H, K, V, _ptr(cu_seqlens), N,
                                int(bool(head_first)), _dtype_code(q), _ptr(workspace),
                                workspace.numel(), _stream(q.device))
    if st != OK:
        raise WKV7Error(st, "wkv7_gdn_bwd")
    return out


class GatedDeltaNet(torch.autograd.Function):
    """gated_delta_net_chunk / gated_delta_net_recurrent as a differentiable op: forward
    through wkv7_gdn_fwd, backward through wkv7_gdn_bwd (K = V = 64)."""

    @staticmethod
    def forward(ctx, q, k, v, g, beta, s0, cu_seqlens, head_first):
        o, sT = wkv7_gdn_fwd(q, k, v, g, beta, s0=s0, cu_seqlens=cu_seqlens,
                             head_first=head_first)
        ctx.save_for_backward(q, k, v, g, beta, s0, cu_seqlens)
        ctx.head_first = head_first
        return o, sT

    @staticmethod
    def backward(ctx, do, dsT):
        q, k, v, g, beta, s0, cu_seqlens = ctx.saved_tensors
        do = torch.zeros_like(v) if do is None else do.contiguous()
        dsT = None if dsT is None else dsT.contiguous().float()
        gr = wkv7_gdn_bwd(q, k, v, g, beta, do.to(q.dtype), s0=s0, dsT=dsT,
                          cu_seqlens=cu_seqlens, head_first=ctx.head_first)
        ds0 = gr["ds0"] if s0 is not None else None
        return gr["dq"], gr["dk"], gr["dv"], gr["dg"], gr["dbeta"], ds0, None, None


def gated_delta_net(q, k, v, g, beta, initial_state=None, output_final_state=True,
                    cu_seqlens=None, head_first: bool = False):
    """Differentiable Gated DeltaNet (README: gated_delta_net_recurrent / _chunk);
    returns (o, final state or None)."""
    o, sT = GatedDeltaNet.apply(q, k, v, g, beta, initial_state, cu_seqlens, head_first)
    return o, (sT if output_final_state else None)
