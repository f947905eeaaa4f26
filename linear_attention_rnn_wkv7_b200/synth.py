"""Seeded synthetic inputs for the WKV7 workloads (no WKV7 arithmetic here).

This module is the one piece shared by the CUDA path's tests/benchmark and the
CPU oracle: it only draws random numbers on the CPU with ``torch.Generator``
(device independent, fixed draw order) and shapes them.  Nothing in it computes
any part of the recurrence.

Value recipe (the RWKV-7 parametrisation the workloads use):
  r, k, v ~ N(0, 1); k is L2-normalised over its K entries per (b, t, h);
  w = -exp(-0.5 - softplus(z)), z ~ N(0, 1)   (log-space decay in (-0.607, 0));
  a = -k, b = k * eta, eta ~ U(0, 1) one scalar per (b, t, h);
  initial states ~ N(0, std) fp32.
Draw order: r, k, v, z, eta, then the initial state, then the mask.  Values are
drawn in fp32 and rounded to the requested dtype once.

Gated DeltaNet inputs (``gdn_inputs``): q, k, v ~ N(0, 1) as drawn (the operator
normalises q and k itself); g = -exp(-0.5 - softplus(z)), z ~ N(0, 1), one log
decay per (b, t, h); beta = sigmoid(y), y ~ N(0, 1), per (b, t, h).  Draw order:
q, k, v, z, y, then the initial state.
"""
from __future__ import annotations

import math

import torch
import torch.nn.functional as F

__all__ = ["fwd_inputs", "padding_mask", "sane_tau", "varlen_lengths", "decode_state",
           "decode_step_inputs", "gdn_inputs", "gdn_varlen_inputs", "gdn_step_inputs",
           "WORKLOADS"]


def _token_vectors(g: torch.Generator, shape_k, shape_v, dtype):
    r = torch.randn(shape_k, generator=g)
    k = torch.randn(shape_k, generator=g)
    k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    v = torch.randn(shape_v, generator=g)
    z = torch.randn(shape_k, generator=g)
    w = -torch.exp(-0.5 - F.softplus(z))
    del z
    eta = torch.rand(shape_k[:-1] + (1,), generator=g)
    a = -k
    b = k * eta
    return {name: t.to(dtype).contiguous() for name, t in
            (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b))}


def fwd_inputs(B: int, T: int, H: int, K: int = 64, V: int = 64,
               dtype: torch.dtype = torch.bfloat16, seed: int = 0,
               s0_std: float | None = 0.1, n_states: int | None = None):
    """Inputs r,w,k,a,b [B,T,H,K], v [B,T,H,V]; s0 [N,H,K,V] fp32 (or None)."""
    g = torch.Generator().manual_seed(seed)
    out = _token_vectors(g, (B, T, H, K), (B, T, H, V), dtype)
    N = B if n_states is None else n_states
    if s0_std is None:
        out["s0"] = None
    elif s0_std == 0.0:
        out["s0"] = torch.zeros(N, H, K, V, dtype=torch.float32)
    else:
        out["s0"] = (torch.randn(N, H, K, V, generator=g) * s0_std).contiguous()
    return out


def _gdn_vectors(g: torch.Generator, shape_k, shape_v, dtype):
    q = torch.randn(shape_k, generator=g)
    k = torch.randn(shape_k, generator=g)
    v = torch.randn(shape_v, generator=g)
    z = torch.randn(shape_k[:-1], generator=g)
    gate = -torch.exp(-0.5 - F.softplus(z))
    beta = torch.sigmoid(torch.randn(shape_k[:-1], generator=g))
    return {name: t.to(dtype).contiguous() for name, t in
            (("q", q), ("k", k), ("v", v), ("g", gate), ("beta", beta))}


def gdn_inputs(B: int, T: int, H: int, K: int = 64, V: int = 64,
               dtype: torch.dtype = torch.bfloat16, seed: int = 0,
               s0_std: float | None = 0.1, n_states: int | None = None):
    """Gated DeltaNet inputs q, k [B,T,H,K], v [B,T,H,V], g, beta [B,T,H];
    s0 [N,H,K,V] fp32 (or None)."""
    g = torch.Generator().manual_seed(seed)
    out = _gdn_vectors(g, (B, T, H, K), (B, T, H, V), dtype)
    N = B if n_states is None else n_states
    if s0_std is None:
        out["s0"] = None
    elif s0_std == 0.0:
        out["s0"] = torch.zeros(N, H, K, V, dtype=torch.float32)
    else:
        out["s0"] = (torch.randn(N, H, K, V, generator=g) * s0_std).contiguous()
    return out


def gdn_varlen_inputs(lengths: torch.Tensor, H: int, K: int = 64, V: int = 64,
                      dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                      s0_std: float | None = 0.1):
    """Packed [1, sum(lengths), H, *] Gated DeltaNet inputs, per-sequence s0, cu_seqlens."""
    out = gdn_inputs(1, int(lengths.sum()), H, K, V, dtype, seed, s0_std,
                     n_states=lengths.numel())
    out["cu_seqlens"] = cu_seqlens_of(lengths)
    return out


def gdn_step_inputs(B: int, H: int, K: int = 64, V: int = 64,
                    dtype: torch.dtype = torch.bfloat16, seed: int = 6, step: int = 0):
    """One Gated DeltaNet decode step: q, k [B,H,K], v [B,H,V], g, beta [B,H]."""
    g = torch.Generator().manual_seed(seed * 1_000_003 + 1 + step)
    return _gdn_vectors(g, (B, H, K), (B, H, V), dtype)


def sane_tau(B: int, C: int, H: int, seed: int) -> torch.Tensor:
    """fp32 [B, C, H] SANE clip levels, softplus(z) + 1 with z ~ N(0, 1) (the README's
    preprocessing of tau: softplus(param) + 1, so tau > 1)."""
    g = torch.Generator().manual_seed(seed * 7177 + 11)
    return (F.softplus(torch.randn(B, C, H, generator=g)) + 1.0).contiguous()


def padding_mask(B: int, T: int, seed: int, max_suffix: int = 1024,
                 interior_p: float = 0.05) -> torch.Tensor:
    """uint8 [B,T]: 0 on a random suffix of length U{0..max_suffix} per row and
    on a Bernoulli(interior_p) set of the earlier tokens, 1 elsewhere."""
    g = torch.Generator().manual_seed(seed * 7919 + 17)
    suffix = torch.randint(0, max_suffix + 1, (B,), generator=g)
    holes = torch.rand(B, T, generator=g) < interior_p
    t = torch.arange(T)[None, :]
    keep = (t < (T - suffix)[:, None]) & ~holes
    return keep.to(torch.uint8).contiguous()


def varlen_lengths(n: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    """int64 [n]: round(exp(U(ln lo, ln hi))) clipped to [lo, hi]."""
    g = torch.Generator().manual_seed(seed * 104729 + 3)
    u = torch.rand(n, generator=g, dtype=torch.float64)
    lengths = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))).round()
    return lengths.clamp(lo, hi).to(torch.int64)


def cu_seqlens_of(lengths: torch.Tensor) -> torch.Tensor:
    cu = torch.zeros(lengths.numel() + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lengths, 0).to(torch.int32)
    return cu


def varlen_inputs(lengths: torch.Tensor, H: int, K: int = 64, V: int = 64,
                  dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                  s0_std: float | None = 0.1):
    """Packed [1, sum(lengths), H, *] inputs, per-sequence s0 and cu_seqlens."""
    total = int(lengths.sum())
    out = fwd_inputs(1, total, H, K, V, dtype, seed, s0_std, n_states=lengths.numel())
    out["cu_seqlens"] = cu_seqlens_of(lengths)
    return out


def decode_state(B: int, H: int, K: int = 64, V: int = 64, seed: int = 4,
                 std: float = 0.1) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed * 31 + 5)
    return (torch.randn(B, H, K, V, generator=g) * std).contiguous()


def decode_step_inputs(B: int, H: int, K: int = 64, V: int = 64,
                       dtype: torch.dtype = torch.bfloat16, seed: int = 4,
                       step: int = 0):
    """One decode step's r,w,k,a,b [B,H,K] and v [B,H,V]; independent per step."""
    g = torch.Generator().manual_seed(seed * 1_000_003 + 1 + step)
    return _token_vectors(g, (B, H, K), (B, H, V), dtype)


# The workloads: name -> description of sizes (used by tests and bench).
WORKLOADS = {
    "fwd_fp32_small": dict(B=1, T=64, H=2, K=64, V=64, dtype="f32", seed=0, s0_std=0.0),
    "fwd_bf16_b8_t4096_h64": dict(B=8, T=4096, H=64, K=64, V=64, dtype="bf16", seed=1,
                                  s0_std=0.1),
    "fwd_bf16_masked_b16_t4096_h32": dict(B=16, T=4096, H=32, K=64, V=64, dtype="bf16",
                                          seed=2, s0_std=0.1, mask=True),
    "fwd_bf16_varlen_64seq_h32": dict(n_seqs=64, lo=16, hi=8192, H=32, K=64, V=64,
                                      dtype="bf16", seed=3, s0_std=0.1),
    "step_bf16_b1024_h32_256steps": dict(B=1024, H=32, K=64, V=64, dtype="bf16", seed=4,
                                         steps=256, s0_std=0.1),
    # Gated DeltaNet through the same kernels (same shapes as the WKV7 workloads)
    "gdn_fwd_bf16_b8_t4096_h64": dict(B=8, T=4096, H=64, K=64, V=64, dtype="bf16", seed=5,
                                      s0_std=0.1),
    "gdn_step_bf16_b1024_h32_256steps": dict(B=1024, H=32, K=64, V=64, dtype="bf16", seed=6,
                                             steps=256, s0_std=0.1),
}
