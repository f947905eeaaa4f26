"""fp64 CPU oracle for the WKV7 recurrence -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The product path (``linear_attention_rnn_wkv7_b200``)
never does; the two share no code.

``fwd`` runs the plain sequential recurrence of the generalized delta rule
(rwkv-ops 0.9.0 README, "rwkv7op 使用方法", generalized_delta_rule docstring:
shapes [B,T,H,K], log-space decay, mask[B,T] 1 = update / 0 = keep, initial
and final state [N,H,K,V]) in C, fp64, OpenMP over (sequence, head) units;
see ``wkv7_oracle.c`` for the equations.  ``step`` is the length-one case
(rwkv-ops 0.9.0 README, "rwkv7_op_rnn 使用方法": inputs (B,1,H,K), state
(B,H,K,K)).  ``brute`` holds an independent dense-product form used only to
pin this one on tiny inputs.

``bwd`` is the backward of ``fwd`` (plain reverse-mode differentiation of the
same recurrence, every state kept), for dL/do and dL/dS_T given.

``sane_fwd`` is the State Anomaly Neutralization variant (README, "rwkv7op_sane
使用方法"): the same recurrence with a soft clip of the state after every 16th token;
the clip function is not on the pages (reading: tau * tanh(S / tau)), so its parity
is unpinned beyond the structure the tests check.

``gdn_bwd`` is the Gated DeltaNet backward: the generalized-rule backward on the
substituted inputs, then the chain rule through that substitution and through the
L2 normalisation of q and k (numpy, written out below).

``gdn_fwd`` / ``gdn_step`` are the Gated DeltaNet operator of the same README
(sections "gdn_recurrent 使用方法" and "gdn_chunk 使用方法": q, k L2-normalised
inside, g a log-space decay gate per (b, t, h), beta a write strength in (0, 1)
per (b, t, h)), written in its delta-rule form in ``wkv7_oracle.c``.

Every input is converted exactly to float64 (bf16 and fp32 values are exactly
representable), so the oracle sees the very values a kernel sees.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv7_oracle.c")
_LIB = os.path.join(_HERE, "libwkv7_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, OpenMP) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str):
    """Open a compiled oracle library (the default one, or a test's variant)."""
    lib = ctypes.CDLL(path)
    p = ctypes.c_void_p
    i = ctypes.c_int
    lib.wkv7_oracle_fwd.restype = ctypes.c_int
    lib.wkv7_oracle_fwd.argtypes = [p, p, p, p, p, p, p, p, p, p,
                                    i, i, i, i, i, p, i, i, ctypes.POINTER(ctypes.c_int)]
    if hasattr(lib, "wkv7_oracle_bwd"):
        lib.wkv7_oracle_bwd.restype = ctypes.c_int
        lib.wkv7_oracle_bwd.argtypes = [p] * 17 + [i, i, i, i, i, p, i, i,
                                                   ctypes.POINTER(ctypes.c_int)]
    if hasattr(lib, "wkv7_oracle_sane_fwd"):
        lib.wkv7_oracle_sane_fwd.restype = ctypes.c_int
        lib.wkv7_oracle_sane_fwd.argtypes = [p] * 11 + [i, i, i, i, i]
    if hasattr(lib, "gdn_oracle_fwd"):
        lib.gdn_oracle_fwd.restype = ctypes.c_int
        lib.gdn_oracle_fwd.argtypes = [p, p, p, p, p, p, i, p, p,
                                       i, i, i, i, i, p, i, i, ctypes.POINTER(ctypes.c_int)]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (any float dtype, CPU)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def fwd(r, w, k, v, a, b, s0=None, mask=None, cu_seqlens=None,
        output_final_state: bool = True, nthreads: int = 0, library=None):
    """Oracle forward.  Returns (o [B,T,H,V] f64, sT [N,H,K,V] f64 or None, threads).

    r,w,k,a,b: [B,T,H,K]; v: [B,T,H,V]; s0: [N,H,K,V] or None (zeros);
    mask: [B,T] (nonzero = update) or None; cu_seqlens: [N+1] ints or None.
    """
    r, w, k, v, a, b = (_f64(x) for x in (r, w, k, v, a, b))
    B, T, H, K = r.shape
    V = v.shape[-1]
    for x in (w, k, a, b):
        assert x.shape == (B, T, H, K)
    assert v.shape == (B, T, H, V)
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int32))
        N = cu.shape[0] - 1
    else:
        N = B
    s0 = _f64(s0)
    if s0 is not None:
        assert s0.shape == (N, H, K, V)
    m = None
    if mask is not None:
        m = mask.cpu().numpy() if hasattr(mask, "cpu") else np.asarray(mask)
        m = np.ascontiguousarray((m != 0).astype(np.uint8))
        assert m.shape == (B, T)
    o = np.zeros((B, T, H, V), dtype=np.float64)
    sT = np.zeros((N, H, K, V), dtype=np.float64) if output_final_state else None
    used = ctypes.c_int(0)
    lib = _load() if library is None else library
    rc = lib.wkv7_oracle_fwd(_ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                 _ptr(s0), _ptr(m), _ptr(o), _ptr(sT), B, T, H, K, V,
                                 _ptr(cu), N, int(nthreads), ctypes.byref(used))
    if rc != 0:
        raise ValueError("wkv7_oracle_fwd rejected its arguments")
    return o, sT, used.value


def step(r, w, k, v, a, b, state, nthreads: int = 0):
    """One decode step: inputs [B,H,K] / v [B,H,V], state [B,H,K,V] (not modified).

    Returns (o [B,H,V], new_state [B,H,K,V]) in float64.
    """
    r, w, k, v, a, b = (_f64(x)[:, None] for x in (r, w, k, v, a, b))
    o, sT, _ = fwd(r, w, k, v, a, b, s0=_f64(state), nthreads=nthreads)
    return o[:, 0], sT


def _cu(cu_seqlens):
    if cu_seqlens is None:
        return None
    return np.ascontiguousarray(np.asarray(
        cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int32))


def gdn_fwd(q, k, v, g, beta, s0=None, cu_seqlens=None, output_final_state: bool = True,
            nthreads: int = 0, library=None):
    """Gated DeltaNet oracle forward.  Returns (o [B,T,H,V], sT [N,H,K,V] or None, threads).

    q, k: [B,T,H,K]; v: [B,T,H,V]; g, beta: [B,T,H]; s0: [N,H,K,V], [1,H,K,V]
    (one state shared by every sequence) or None (zeros); cu_seqlens: [N+1] or None.
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    B, T, H, K = q.shape
    V = v.shape[-1]
    assert k.shape == (B, T, H, K) and v.shape == (B, T, H, V)
    assert g.shape == (B, T, H) and beta.shape == (B, T, H)
    cu = _cu(cu_seqlens)
    N = B if cu is None else cu.shape[0] - 1
    s0 = _f64(s0)
    shared = 0
    if s0 is not None:
        assert s0.shape in ((N, H, K, V), (1, H, K, V))
        shared = int(s0.shape[0] == 1 and N != 1)
    o = np.zeros((B, T, H, V), dtype=np.float64)
    sT = np.zeros((N, H, K, V), dtype=np.float64) if output_final_state else None
    used = ctypes.c_int(0)
    lib = _load() if library is None else library
    rc = lib.gdn_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0), shared,
                            _ptr(o), _ptr(sT), B, T, H, K, V, _ptr(cu), N, int(nthreads),
                            ctypes.byref(used))
    if rc != 0:
        raise ValueError("gdn_oracle_fwd rejected its arguments")
    return o, sT, used.value


def gdn_step(q, k, v, g, beta, state, nthreads: int = 0):
    """One Gated DeltaNet decode step: q, k [B,H,K], v [B,H,V], g, beta [B,H],
    state [B,H,K,V] (not modified).  Returns (o [B,H,V], new_state) in float64."""
    q, k, v, g, beta = (_f64(x)[:, None] for x in (q, k, v, g, beta))
    o, sT, _ = gdn_fwd(q, k, v, g, beta, s0=_f64(state), nthreads=nthreads)
    return o[:, 0], sT


def bwd(r, w, k, v, a, b, dout, s0=None, mask=None, dsT=None, cu_seqlens=None,
        nthreads: int = 0, library=None):
    """Oracle backward.  Returns a dict of float64 arrays: dr, dw, dk, da, db [B,T,H,K],
    dv [B,T,H,V], ds0 [N,H,K,V]."""
    r, w, k, v, a, b, dout = (_f64(x) for x in (r, w, k, v, a, b, dout))
    B, T, H, K = r.shape
    V = v.shape[-1]
    assert dout.shape == (B, T, H, V)
    cu = _cu(cu_seqlens)
    N = B if cu is None else cu.shape[0] - 1
    s0, dsT = _f64(s0), _f64(dsT)
    m = None
    if mask is not None:
        m = mask.cpu().numpy() if hasattr(mask, "cpu") else np.asarray(mask)
        m = np.ascontiguousarray((m != 0).astype(np.uint8))
    g = {n: np.zeros((B, T, H, K)) for n in ("dr", "dw", "dk", "da", "db")}
    g["dv"] = np.zeros((B, T, H, V))
    g["ds0"] = np.zeros((N, H, K, V))
    used = ctypes.c_int(0)
    lib = _load() if library is None else library
    rc = lib.wkv7_oracle_bwd(_ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0),
                             _ptr(m), _ptr(dout), _ptr(dsT), _ptr(g["dr"]), _ptr(g["dw"]),
                             _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["da"]), _ptr(g["db"]),
                             _ptr(g["ds0"]), B, T, H, K, V, _ptr(cu), N, int(nthreads),
                             ctypes.byref(used))
    if rc != 0:
        raise ValueError("wkv7_oracle_bwd rejected its arguments")
    return g


def gdn_bwd(q, k, v, g, beta, dout, s0=None, dsT=None, cu_seqlens=None, nthreads: int = 0):
    """Gated DeltaNet backward for L = sum(o * dout) + sum(S_T * dsT).  Returns float64
    dq, dk, dv [B,T,H,*], dg, dbeta [B,T,H] and ds0 (shaped like s0, or [N,H,K,V]).

    Gated DeltaNet is the generalized rule with r = qh, w = g on every channel, write
    key beta kh, a = kh and b = -e^g beta kh (qh = q/|q|, kh = k/|k|).  The gradients
    of those inputs come from ``bwd``; then, by the chain rule,
        dkh = beta dk_w + da - e^g beta db,   dg = sum(dw) + db . b,
        dbeta = kh . dk_w - e^g (kh . db),
        dx = (dxh - xh (xh . dxh)) / |x| for x = q (dxh = dr) and x = k (a zero x gets 0).
    """
    q, k, v, g, beta, dout = (_f64(x) for x in (q, k, v, g, beta, dout))
    B, T, H, K = q.shape
    cu = _cu(cu_seqlens)
    N = B if cu is None else cu.shape[0] - 1
    s0 = _f64(s0)
    shared = s0 is not None and s0.shape[0] == 1 and N != 1
    s0_full = np.repeat(s0, N, axis=0) if shared else s0
    nq = np.linalg.norm(q, axis=-1, keepdims=True)
    nk = np.linalg.norm(k, axis=-1, keepdims=True)
    qh = np.where(nq > 0, q / np.where(nq > 0, nq, 1.0), 0.0)
    kh = np.where(nk > 0, k / np.where(nk > 0, nk, 1.0), 0.0)
    eg = np.exp(g)[..., None]
    bt = beta[..., None]
    w = np.repeat(g[..., None], K, axis=-1)
    gr = bwd(qh, w, bt * kh, v, kh, -eg * bt * kh, dout, s0=s0_full, dsT=_f64(dsT),
             cu_seqlens=cu, nthreads=nthreads)
    dkh = bt * gr["dk"] + gr["da"] - eg * bt * gr["db"]
    out = {"dv": gr["dv"]}
    out["dg"] = gr["dw"].sum(-1) + np.sum(gr["db"] * (-eg * bt * kh), axis=-1)
    out["dbeta"] = np.sum(kh * gr["dk"], axis=-1) - eg[..., 0] * np.sum(kh * gr["db"], axis=-1)

    def through_norm(xh, n, dxh):
        proj = dxh - xh * np.sum(xh * dxh, axis=-1, keepdims=True)
        return np.where(n > 0, proj / np.where(n > 0, n, 1.0), 0.0)

    out["dq"] = through_norm(qh, nq, gr["dr"])
    out["dk"] = through_norm(kh, nk, dkh)
    out["ds0"] = gr["ds0"].sum(axis=0, keepdims=True) if shared else gr["ds0"]
    return out


def sane_fwd(r, w, k, v, a, b, tau, sane_mask=None, s0=None, library=None):
    """SANE forward.  r,w,k,a,b [B,T,H,K]; v [B,T,H,V]; tau [B,T//16,H] (> 0);
    sane_mask [B,T//16] (nonzero = clip that chunk) or None (every chunk); s0
    [B,H,K,V] or None.  Returns (o [B,T,H,V], sT [B,H,K,V]) in float64."""
    r, w, k, v, a, b, tau = (_f64(x) for x in (r, w, k, v, a, b, tau))
    B, T, H, K = r.shape
    V = v.shape[-1]
    assert tau.shape == (B, T // 16, H)
    m = None
    if sane_mask is not None:
        m = sane_mask.cpu().numpy() if hasattr(sane_mask, "cpu") else np.asarray(sane_mask)
        m = np.ascontiguousarray((m != 0).astype(np.uint8))
        assert m.shape == (B, T // 16)
    s0 = _f64(s0)
    o = np.zeros((B, T, H, V))
    sT = np.zeros((B, H, K, V))
    lib = _load() if library is None else library
    rc = lib.wkv7_oracle_sane_fwd(_ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                  _ptr(tau), _ptr(m), _ptr(s0), _ptr(o), _ptr(sT), B, T, H, K, V)
    if rc != 0:
        raise ValueError("wkv7_oracle_sane_fwd rejected its arguments")
    return o, sT


def sane_step(r, w, k, v, a, b, tau, do_sane, state, nthreads: int = 0):
    """SANE single step (README, "rwkv7_op_sane_rnn 使用方法"): one step of the recurrence
    (``step``), the output read from the state before the clip, then the soft clip
    S <- tau * tanh(S / tau) of the rows whose flag is set.  r,w,k,a,b [B,H,K], v [B,H,V],
    tau [B,H] (> 0), do_sane a bool or [B] flags, state [B,H,K,V] (not modified).
    Returns (o [B,H,V], new_state [B,H,K,V]) in float64.  The clip function is the
    reading taken for SANE (parity unpinned by the pages)."""
    o, new = step(r, w, k, v, a, b, state, nthreads=nthreads)
    tau = _f64(tau)
    B = new.shape[0]
    flags = np.broadcast_to(np.asarray(
        do_sane.cpu().numpy() if hasattr(do_sane, "cpu") else do_sane) != 0, (B,))
    for bb in range(B):
        if flags[bb]:
            tc = tau[bb][:, None, None]
            new[bb] = tc * np.tanh(new[bb] / tc)
    return o, new
