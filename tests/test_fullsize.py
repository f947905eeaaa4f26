"""Parity at the full workload sizes, in the launch configuration the benchmark
times.  The forward workloads are compared on every (sequence, head) unit with one
oracle call over the whole problem (a few seconds on the host's cores), so the
relative errors use the same denominators as the tolerances' definition; the decode
workload on sampled states.

Workloads: B=8,T=4096,H=64 bf16 (seed 1); B=16,T=4096,H=32 bf16 with a padding
mask (seed 2); 64 packed sequences of log-uniform length in [16, 8192], H=32
(seed 3); 1024 x 32 decode states (seed 4)."""
import functools

import numpy as np
import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import synth, wkv7_fwd, wkv7_step
from parity_util import check, rel_err, BF16_O_REL, BF16_S_REL

pytestmark = pytest.mark.gpu


def _sample_units(B, H, n, seed):
    g = np.random.default_rng(seed)
    units = {(0, 0), (B - 1, H - 1)}
    while len(units) < n:
        units.add((int(g.integers(B)), int(g.integers(H))))
    return sorted(units)


@functools.lru_cache(maxsize=1)
def _inputs(name):
    p = synth.WORKLOADS[name]
    x = synth.fwd_inputs(p["B"], p["T"], p["H"], dtype=torch.bfloat16, seed=p["seed"],
                         s0_std=p["s0_std"])
    mask = synth.padding_mask(p["B"], p["T"], seed=p["seed"]) if p.get("mask") else None
    return x, mask


def _fwd_full(cuda_device, name, algo):
    x, mask = _inputs(name)
    xd = {k: v.to(cuda_device) for k, v in x.items()}
    o, s = wkv7_fwd(xd["r"], xd["w"], xd["k"], xd["v"], xd["a"], xd["b"], s0=xd["s0"],
                    mask=None if mask is None else mask.to(cuda_device), algo=algo)
    o_ref, s_ref = _oracle_full(name)
    return check(o, s, o_ref, s_ref, torch.bfloat16, f"{name} {algo}")


@functools.lru_cache(maxsize=1)
def _oracle_full(name):
    x, mask = _inputs(name)
    o_ref, s_ref, _ = oracle.fwd(x["r"], x["w"], x["k"], x["v"], x["a"], x["b"], s0=x["s0"],
                                 mask=mask)
    return o_ref, s_ref


@pytest.mark.parametrize("algo", ["auto", "recurrent"])
def test_fwd_b8_t4096_h64(cuda_device, algo):
    _fwd_full(cuda_device, "fwd_bf16_b8_t4096_h64", algo)


@pytest.mark.parametrize("algo", ["auto", "recurrent"])
def test_fwd_masked_b16_t4096_h32(cuda_device, algo):
    _fwd_full(cuda_device, "fwd_bf16_masked_b16_t4096_h32", algo)


def test_fwd_varlen_64seq_h32(cuda_device):
    p = synth.WORKLOADS["fwd_bf16_varlen_64seq_h32"]
    lengths = synth.varlen_lengths(p["n_seqs"], p["lo"], p["hi"], seed=p["seed"])
    x = synth.varlen_inputs(lengths, p["H"], dtype=torch.bfloat16, seed=p["seed"],
                            s0_std=p["s0_std"])
    xd = {k: v.to(cuda_device) for k, v in x.items()}
    o, s = wkv7_fwd(xd["r"], xd["w"], xd["k"], xd["v"], xd["a"], xd["b"], s0=xd["s0"],
                    cu_seqlens=xd["cu_seqlens"])
    o_ref, s_ref, _ = oracle.fwd(x["r"], x["w"], x["k"], x["v"], x["a"], x["b"], s0=x["s0"],
                                 cu_seqlens=x["cu_seqlens"])
    check(o, s, o_ref, s_ref, torch.bfloat16, "varlen 64 sequences")


def test_step_b1024_h32(cuda_device):
    """The decode workload at its stated length: 256 consecutive in-place steps over
    1024 x 32 states.  o is compared at every step (rel <= 2e-2) and the state after
    the last step (rel <= 1e-3) on 64 sampled states, the first and last included;
    the oracle steps those states in fp64 from the same initial values."""
    p = synth.WORKLOADS["step_bf16_b1024_h32_256steps"]
    B, H, steps = p["B"], p["H"], p["steps"]
    assert steps == 256
    state = synth.decode_state(B, H, seed=p["seed"], std=p["s0_std"])
    units = _sample_units(B, H, 64, p["seed"])
    assert (0, 0) in units and (B - 1, H - 1) in units
    idx_b = [u[0] for u in units]
    idx_h = [u[1] for u in units]
    ref = state[idx_b, idx_h].double().numpy()[:, None]  # [U,1,K,V]
    st = state.to(cuda_device)
    worst_o = 0.0
    for i in range(steps):
        x = synth.decode_step_inputs(B, H, dtype=torch.bfloat16, seed=p["seed"], step=i)
        o = wkv7_step(*(x[n].to(cuda_device) for n in "rwkvab"), st)
        sub = {n: x[n][idx_b, idx_h][:, None] for n in "rwkvab"}  # [U,1,K]
        o_ref, ref = oracle.step(*(sub[n] for n in "rwkvab"), ref)
        e = rel_err(o[idx_b, idx_h][:, None], o_ref)
        worst_o = max(worst_o, e)
        assert e <= BF16_O_REL, f"step {i}: o rel {e:.3e}"
    es = rel_err(st[idx_b, idx_h][:, None], ref)
    assert es <= BF16_S_REL, f"state after {steps} steps: rel {es:.3e} (worst o {worst_o:.3e})"
