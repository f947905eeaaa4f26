"""GPU parity of the State Anomaly Neutralization kernels (wkv7_sane_fwd, wkv7_sane_step;
rwkv-ops 0.9.0 README, "rwkv7op_sane 使用方法" and "rwkv7_op_sane_rnn 使用方法") against
the fp64 SANE oracle on the same seeded inputs.  The clip function itself (tau *
tanh(S / tau)) is the reading both sides implement: parity for it is unpinned by the
pages; its placement (after every full 16-token chunk whose flag is set, outputs read
before the clip, a partial last chunk never clipped) is what these tests fix.  States
are drawn large enough (s0 ~ N(0, 2)) that the clip changes them."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import (synth, wkv7_fwd, wkv7_get_last_error, wkv7_sane_fwd,
                                            wkv7_sane_step)
from linear_attention_rnn_wkv7_b200.wkv7 import OK
from parity_util import abs_err, check, rel_err, to_dev, BF16_O_REL, BF16_S_REL, F32_ABS

pytestmark = pytest.mark.gpu
NAMES = ("r", "w", "k", "v", "a", "b")


def _problem(B, T, H, dtype, seed, K=64, s0_std=2.0):
    x = synth.fwd_inputs(B, T, H, K=K, V=K, dtype=dtype, seed=seed, s0_std=s0_std)
    C = T // 16
    tau = synth.sane_tau(B, C, H, seed)
    g = torch.Generator().manual_seed(seed + 1)
    flags = (torch.rand(B, C, generator=g) < 0.7).to(torch.uint8)
    return x, tau, flags


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [15, 16, 47, 64, 130])
def test_sane_fwd_matches_oracle(cuda_device, dtype, T):
    x, tau, flags = _problem(2, T, 3, dtype, 900 + T)
    o_ref, s_ref = oracle.sane_fwd(*(x[n] for n in NAMES), tau, sane_mask=flags, s0=x["s0"])
    xd = to_dev(x, cuda_device)
    o, s = wkv7_sane_fwd(*(xd[n] for n in NAMES), tau.to(cuda_device),
                         sane_mask=flags.to(cuda_device), s0=xd["s0"])
    check(o, s, o_ref, s_ref, dtype, f"sane fwd T={T}")
    assert wkv7_get_last_error() == OK


def test_sane_clip_is_active_and_placed(cuda_device):
    """Against the plain forward: identical through token 15 (the boundary token's output
    is read before the clip), different from token 16 on where the chunk is flagged,
    identical throughout where no chunk is flagged."""
    x, tau, _ = _problem(2, 64, 2, torch.float32, 950)
    flags = torch.tensor([[1, 1, 1, 1], [0, 0, 0, 0]], dtype=torch.uint8)
    xd = to_dev(x, cuda_device)
    o_s, s_s = wkv7_sane_fwd(*(xd[n] for n in NAMES), tau.to(cuda_device),
                             sane_mask=flags.to(cuda_device), s0=xd["s0"])
    o_p, s_p = wkv7_fwd(*(xd[n] for n in NAMES), s0=xd["s0"], algo="recurrent")
    assert abs_err(o_s[:, :16], o_p[:, :16].cpu().double().numpy()) <= 1e-5
    assert abs_err(o_s[1], o_p[1].cpu().double().numpy()) <= 1e-5
    assert abs_err(s_s[1], s_p[1].cpu().double().numpy()) <= 1e-5
    assert (o_s[0, 16:] - o_p[0, 16:]).abs().max().item() > 1e-2
    bound = tau[0, -1][:, None, None].to(cuda_device)
    assert bool((s_s[0].abs() <= bound).all())


@pytest.mark.parametrize("head_first", [False, True])
def test_sane_fwd_shared_state_no_flags(cuda_device, head_first):
    """sane_mask = None (every full chunk clipped), one [1, H, K, V] initial state shared
    by the batch, token-major and head-first layouts, bf16."""
    x, tau, _ = _problem(3, 80, 2, torch.bfloat16, 960)
    s0 = x["s0"][:1].contiguous()
    o_ref, s_ref = oracle.sane_fwd(*(x[n] for n in NAMES), tau, s0=s0.expand(3, -1, -1, -1))
    xd = to_dev(x, cuda_device)
    lay = (lambda t: t.transpose(1, 2).contiguous()) if head_first else (lambda t: t)
    o, s = wkv7_sane_fwd(*(lay(xd[n]) for n in NAMES), tau.to(cuda_device),
                         s0=s0.to(cuda_device), head_first=head_first)
    if head_first:
        o = o.transpose(1, 2)
    check(o, s, o_ref, s_ref, torch.bfloat16, f"sane shared s0 head_first={head_first}")


@pytest.mark.parametrize("K", [128, 256])
def test_sane_fwd_wide_heads(cuda_device, K):
    x, tau, flags = _problem(1, 40, 2, torch.float32, 970 + K, K=K)
    o_ref, s_ref = oracle.sane_fwd(*(x[n] for n in NAMES), tau, sane_mask=flags, s0=x["s0"])
    xd = to_dev(x, cuda_device)
    o, s = wkv7_sane_fwd(*(xd[n] for n in NAMES), tau.to(cuda_device),
                         sane_mask=flags.to(cuda_device), s0=xd["s0"])
    check(o, s, o_ref, s_ref, torch.float32, f"sane fwd K={K}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("K", [64, 128])
def test_sane_step_matches_oracle(cuda_device, dtype, K):
    """The README's loop: do_sane = (step % 16 == 15), as a per-row [B] flag tensor on even
    chunks and as one bool on odd chunks; o per step and the state after 33 steps."""
    B, H, steps = 5, 3, 33
    state = synth.decode_state(B, H, K=K, V=K, seed=980, std=2.0)
    ref = state.double().numpy()
    st = state.to(cuda_device)
    tau = synth.sane_tau(B, 1, H, 981)[:, 0].contiguous()
    rows = torch.tensor([1, 0, 1, 1, 0], dtype=torch.uint8)
    for i in range(steps):
        y = synth.decode_step_inputs(B, H, K=K, V=K, dtype=dtype, seed=982, step=i)
        boundary = i % 16 == 15
        flag = (rows if (i // 16) % 2 == 0 else True) if boundary else False
        flag_dev = flag.to(cuda_device) if isinstance(flag, torch.Tensor) else flag
        og = wkv7_sane_step(*(y[n].to(cuda_device) for n in NAMES), tau.to(cuda_device),
                            flag_dev, st)
        o_r, ref = oracle.sane_step(*(y[n] for n in NAMES), tau, flag, ref)
        if dtype == torch.float32:
            assert abs_err(og, o_r) <= F32_ABS, i
        else:
            assert rel_err(og, o_r) <= BF16_O_REL, i
    if dtype == torch.float32:
        assert abs_err(st, ref) <= F32_ABS
    else:
        assert rel_err(st, ref) <= BF16_S_REL


def test_sane_step_equals_sane_fwd_on_gpu(cuda_device):
    """T decode steps with do_sane at every 16th token == one SANE forward (fp32)."""
    B, T, H = 2, 48, 2
    x, tau, flags = _problem(B, T, H, torch.float32, 990)
    xd = to_dev(x, cuda_device)
    o, s = wkv7_sane_fwd(*(xd[n] for n in NAMES), tau.to(cuda_device),
                         sane_mask=flags.to(cuda_device), s0=xd["s0"])
    st = xd["s0"].clone()
    for t in range(T):
        c = t // 16
        f = flags[:, c].to(cuda_device) if t % 16 == 15 else False
        ot = wkv7_sane_step(*(xd[n][:, t].contiguous() for n in NAMES),
                            tau[:, c].contiguous().to(cuda_device), f, st)
        assert (ot - o[:, t]).abs().max().item() <= 1e-4, t
    assert (st - s).abs().max().item() <= 1e-4
