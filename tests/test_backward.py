"""GPU parity of wkv7_bwd (backward of the generalized delta rule) against the fp64
backward oracle, which is itself pinned by finite differences of the forward oracle.

Small problems are compared in full across checkpoint (8-token) and chunk
boundaries, with masks, a zero or given dL/dS_T, and s0 = None; the B=8, T=4096, H=64
bf16 workload is compared on a sample of units.  Tolerances: fp32 inputs
rel <= 1e-4; bf16 inputs (gradients rounded to bf16) rel <= 2e-2, where
rel(X) = max |X_gpu - X_ref| / max |X_ref|."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import (WKV7Error, generalized_delta_rule, synth,
                                            wkv7_bwd, wkv7_get_last_error)
from linear_attention_rnn_wkv7_b200.wkv7 import ERR_INVALID_ARG, OK
from parity_util import rel_err, to_dev

pytestmark = pytest.mark.gpu

NAMES = ("r", "w", "k", "v", "a", "b")
GRADS = ("dr", "dw", "dk", "dv", "da", "db", "ds0")


def tol(dtype):
    return 1e-4 if dtype == torch.float32 else 2e-2


def check_grads(g, ref, dtype, what):
    for n in GRADS:
        e = rel_err(g[n], ref[n])
        limit = tol(dtype) if n != "ds0" else (1e-4 if dtype == torch.float32 else 1e-3)
        assert e <= limit, f"{what}: {n} rel {e:.3e} > {limit}"


def upstream(B, T, H, dtype, seed):
    gen = torch.Generator().manual_seed(seed)
    dout = torch.randn(B, T, H, 64, generator=gen).to(dtype)
    dsT = torch.randn(B, H, 64, 64, generator=gen) * 0.1
    return dout, dsT


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [1, 7, 8, 9, 64, 130])
def test_bwd_matches_oracle(cuda_device, dtype, T):
    x = synth.fwd_inputs(2, T, 3, dtype=dtype, seed=600 + T, s0_std=0.1)
    dout, dsT = upstream(2, T, 3, dtype, 601 + T)
    ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], dsT=dsT)
    xd = to_dev(x, cuda_device)
    g = wkv7_bwd(*(xd[n] for n in NAMES), dout.to(cuda_device), s0=xd["s0"],
                 dsT=dsT.to(cuda_device))
    check_grads(g, ref, dtype, f"bwd T={T} {dtype}")
    assert wkv7_get_last_error() == OK


def test_bwd_mask_and_optional_states(cuda_device):
    """A mask (masked tokens pass the state gradient through), s0 = None and
    dsT = None."""
    T = 77
    x = synth.fwd_inputs(3, T, 2, dtype=torch.float32, seed=610, s0_std=0.1)
    mask = synth.padding_mask(3, T, seed=611, max_suffix=20)
    mask[1, 8] = 0  # a masked token at a checkpoint
    dout, dsT = upstream(3, T, 2, torch.float32, 612)
    xd = to_dev(x, cuda_device)
    for s0, d in ((x["s0"], dsT), (None, None)):
        ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=s0, mask=mask, dsT=d)
        g = wkv7_bwd(*(xd[n] for n in NAMES), dout.to(cuda_device),
                     s0=None if s0 is None else xd["s0"], mask=mask.to(cuda_device),
                     dsT=None if d is None else d.to(cuda_device))
        check_grads(g, ref, torch.float32, f"bwd mask s0={'set' if s0 is not None else None}")
        m = mask.bool().to(cuda_device)
        for n in ("dw", "dk", "dv", "da", "db"):
            assert float(g[n][~m].abs().max()) == 0.0


def test_bwd_full_size_sampled_units(cuda_device):
    """B=8, T=4096, H=64 bf16 (the forward benchmark's workload) with the launch the
    benchmark times; eight (b, h) units against the oracle."""
    p = synth.WORKLOADS["fwd_bf16_b8_t4096_h64"]
    x = synth.fwd_inputs(p["B"], p["T"], p["H"], dtype=torch.bfloat16, seed=p["seed"],
                         s0_std=p["s0_std"])
    dout, dsT = upstream(p["B"], p["T"], p["H"], torch.bfloat16, 620)
    xd = to_dev(x, cuda_device)
    g = wkv7_bwd(*(xd[n] for n in NAMES), dout.to(cuda_device), s0=xd["s0"],
                 dsT=dsT.to(cuda_device))
    for bb, h in [(0, 0), (1, 17), (2, 33), (3, 63), (4, 5), (5, 40), (6, 21), (7, 62)]:
        sl = lambda t: t[bb:bb + 1, :, h:h + 1]
        ref = oracle.bwd(*(sl(x[n]) for n in NAMES), sl(dout), s0=x["s0"][bb:bb + 1, h:h + 1],
                         dsT=dsT[bb:bb + 1, h:h + 1])
        gu = {n: (g[n][bb:bb + 1, :, h:h + 1] if n != "ds0" else g[n][bb:bb + 1, h:h + 1])
              for n in GRADS}
        check_grads(gu, ref, torch.bfloat16, f"bwd full size unit ({bb},{h})")


def test_autograd_wrapper(cuda_device):
    """generalized_delta_rule through torch.autograd gives wkv7_bwd's gradients."""
    x = to_dev(synth.fwd_inputs(2, 40, 2, dtype=torch.bfloat16, seed=630, s0_std=0.1),
               cuda_device)
    leaves = {n: x[n].clone().requires_grad_(True) for n in NAMES}
    s0 = x["s0"].clone().requires_grad_(True)
    o, sT = generalized_delta_rule(*(leaves[n] for n in NAMES), initial_state=s0)
    gen = torch.Generator().manual_seed(631)
    do = torch.randn(o.shape, generator=gen).to(o.dtype).to(cuda_device)
    dsT = (torch.randn(sT.shape, generator=gen) * 0.1).to(cuda_device)
    ((o.float() * do.float()).sum() + (sT * dsT).sum()).backward()
    g = wkv7_bwd(*(x[n] for n in NAMES), do, s0=x["s0"], dsT=dsT)
    for n in NAMES:
        torch.testing.assert_close(leaves[n].grad, g["d" + n], rtol=0, atol=0)
    torch.testing.assert_close(s0.grad, g["ds0"], rtol=0, atol=0)


def test_bwd_rejects_small_workspace(cuda_device):
    x = to_dev(synth.fwd_inputs(1, 16, 1, dtype=torch.float32, seed=640, s0_std=0.1), cuda_device)
    dout = torch.zeros(1, 16, 1, 64, device=cuda_device)
    ws = torch.empty(64, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(WKV7Error) as e:
        wkv7_bwd(*(x[n] for n in NAMES), dout, workspace=ws)
    assert e.value.status == ERR_INVALID_ARG


@pytest.mark.parametrize("head_first", [False, True])
def test_bwd_varlen(cuda_device, head_first):
    """Packed sequences (lengths 0 … 130, checkpoint boundaries inside and at the ends)
    with per-sequence s0 and dL/dS_T, token-major and head-first."""
    lengths = torch.tensor([17, 0, 8, 1, 130, 63])
    x = synth.varlen_inputs(lengths, 2, dtype=torch.float32, seed=650, s0_std=0.1)
    cu = x.pop("cu_seqlens")
    total, N = int(lengths.sum()), lengths.numel()
    dout, _ = upstream(1, total, 2, torch.float32, 651)
    dsT = torch.randn(N, 2, 64, 64, generator=torch.Generator().manual_seed(652)) * 0.1
    ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], dsT=dsT, cu_seqlens=cu)
    xd = to_dev(x, cuda_device)
    lay = (lambda t: t.transpose(1, 2).contiguous()) if head_first else (lambda t: t)
    g = wkv7_bwd(*(lay(xd[n]) for n in NAMES), lay(dout.to(cuda_device)), s0=xd["s0"],
                 dsT=dsT.to(cuda_device), cu_seqlens=cu.to(cuda_device), head_first=head_first)
    if head_first:
        g = {n: (t.transpose(1, 2) if n != "ds0" else t) for n, t in g.items()}
    check_grads(g, ref, torch.float32, f"bwd varlen head_first={head_first}")
    assert wkv7_get_last_error() == OK


def test_bwd_head_first_batched(cuda_device):
    x = synth.fwd_inputs(2, 45, 3, dtype=torch.bfloat16, seed=660, s0_std=0.1)
    dout, dsT = upstream(2, 45, 3, torch.bfloat16, 661)
    ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], dsT=dsT)
    xd = to_dev(x, cuda_device)
    hf = lambda t: t.transpose(1, 2).contiguous()
    g = wkv7_bwd(*(hf(xd[n]) for n in NAMES), hf(dout.to(cuda_device)), s0=xd["s0"],
                 dsT=dsT.to(cuda_device), head_first=True)
    g = {n: (t.transpose(1, 2) if n != "ds0" else t) for n, t in g.items()}
    check_grads(g, ref, torch.bfloat16, "bwd head_first")


def test_bwd_varlen_with_mask(cuda_device):
    """Packed sequences with a padding mask over the packed rows (masked tokens at
    sequence starts and ends and at checkpoint boundaries)."""
    lengths = torch.tensor([17, 0, 8, 1, 130, 63])
    x = synth.varlen_inputs(lengths, 2, dtype=torch.float32, seed=670, s0_std=0.1)
    cu = x.pop("cu_seqlens")
    total, N = int(lengths.sum()), lengths.numel()
    g = torch.Generator().manual_seed(671)
    mask = (torch.rand(1, total, generator=g) >= 0.2).to(torch.uint8)
    for s0_, L in zip(cu[:-1].tolist(), lengths.tolist()):
        if L > 0:
            mask[0, s0_] = 0
            mask[0, s0_ + L - 1] = 0
        if L > 16:
            mask[0, s0_ + 8] = 0
            mask[0, s0_ + 15] = 0
    dout, _ = upstream(1, total, 2, torch.float32, 672)
    dsT = torch.randn(N, 2, 64, 64, generator=torch.Generator().manual_seed(673)) * 0.1
    ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], mask=mask, dsT=dsT,
                     cu_seqlens=cu)
    xd = to_dev(x, cuda_device)
    gr = wkv7_bwd(*(xd[n] for n in NAMES), dout.to(cuda_device), s0=xd["s0"],
                  mask=mask.to(cuda_device), dsT=dsT.to(cuda_device),
                  cu_seqlens=cu.to(cuda_device))
    check_grads(gr, ref, torch.float32, "bwd varlen + mask")
    assert wkv7_get_last_error() == OK
