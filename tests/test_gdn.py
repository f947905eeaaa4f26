"""GPU parity of the Gated DeltaNet entry points (wkv7_gdn_fwd, wkv7_gdn_step) against
the fp64 Gated DeltaNet oracle on the same seeded inputs.

The operator is gated_delta_net_recurrent / _chunk / _single_step (rwkv-ops 0.9.0
README, "gdn_recurrent 使用方法" and "gdn_chunk 使用方法"), run by the same kernels as
the generalized delta rule.  Small problems are compared element by element in
full across chunk boundaries and ragged tails; the B=8, T=4096, H=64 bf16 workload
is compared on every unit.  Tolerances are those of the generalized rule: fp32
max-abs <= 1e-4; bf16 rel(o) <= 2e-2, rel(final state) <= 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import (WKV7Error, synth, wkv7_gdn_fwd, wkv7_gdn_step,
                                            wkv7_get_last_error)
from linear_attention_rnn_wkv7_b200.wkv7 import ERR_UNSUPPORTED, OK
from parity_util import check, rel_err, to_dev

pytestmark = pytest.mark.gpu

ALGOS = ["recurrent", "chunked"]
NAMES = ("q", "k", "v", "g", "beta")


def run(x, algo, s0="own", cu=None, output_final_state=True):
    init = x["s0"] if s0 == "own" else s0
    return wkv7_gdn_fwd(*(x[n] for n in NAMES), s0=init, cu_seqlens=cu,
                        output_final_state=output_final_state, algo=algo)


def ref(x, s0="own", cu=None):
    init = x["s0"] if s0 == "own" else s0
    o, s, _ = oracle.gdn_fwd(*(x[n] for n in NAMES), s0=init, cu_seqlens=cu)
    return o, s


def test_fp32_recurrent(cuda_device):
    x = synth.gdn_inputs(1, 64, 2, dtype=torch.float32, seed=20, s0_std=0.1)
    o_ref, s_ref = ref(x)
    o, s = run(to_dev(x, cuda_device), "recurrent")
    check(o, s, o_ref, s_ref, torch.float32, "gdn fp32 recurrent")
    with pytest.raises(WKV7Error) as e:  # the chunked form is bf16 only
        run(to_dev(x, cuda_device), "chunked")
    assert e.value.status == ERR_UNSUPPORTED
    assert wkv7_get_last_error() == OK


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 200, 257])
def test_bf16_chunk_boundaries(cuda_device, algo, T):
    x = synth.gdn_inputs(2, T, 3, dtype=torch.bfloat16, seed=200 + T, s0_std=0.1)
    o_ref, s_ref = ref(x)
    o, s = run(to_dev(x, cuda_device), algo)
    check(o, s, o_ref, s_ref, torch.bfloat16, f"gdn {algo} T={T}")


@pytest.mark.parametrize("algo", ALGOS)
def test_initial_state_forms(cuda_device, algo):
    """s0 = None (zeros), one state per sequence, one [1,H,K,V] state shared by every
    sequence, and no final state."""
    x = synth.gdn_inputs(3, 150, 2, dtype=torch.bfloat16, seed=31, s0_std=0.1)
    xd = to_dev(x, cuda_device)
    shared = torch.randn(1, 2, 64, 64, generator=torch.Generator().manual_seed(32)) * 0.1
    for init, name in ((None, "none"), ("own", "own"), (shared, "shared")):
        o_ref, s_ref = ref(x, s0=init)
        dinit = init.to(cuda_device) if isinstance(init, torch.Tensor) else init
        o, s = run(xd, algo, s0=dinit)
        check(o, s, o_ref, s_ref, torch.bfloat16, f"gdn {algo} s0={name}")
    o, s = run(xd, algo, output_final_state=False)
    assert s is None
    check(o, None, ref(x)[0], None, torch.bfloat16, f"gdn {algo} no final state")


@pytest.mark.parametrize("algo", ALGOS)
def test_varlen(cuda_device, algo):
    lengths = torch.tensor([64, 1, 0, 130, 65, 7, 200, 63])
    x = synth.gdn_varlen_inputs(lengths, 3, dtype=torch.bfloat16, seed=33, s0_std=0.1)
    cu = x.pop("cu_seqlens")
    o_ref, s_ref = ref(x, cu=cu)
    o, s = run(to_dev(x, cuda_device), algo, cu=cu.to(cuda_device))
    check(o, s, o_ref, s_ref, torch.bfloat16, f"gdn varlen {algo}")
    shared = x["s0"][:1].clone()
    o_ref, s_ref = ref(x, s0=shared, cu=cu)
    o, s = run(to_dev(x, cuda_device), algo, s0=shared.to(cuda_device), cu=cu.to(cuda_device))
    check(o, s, o_ref, s_ref, torch.bfloat16, f"gdn varlen shared s0 {algo}")
    assert wkv7_get_last_error() == OK


@pytest.mark.parametrize("algo", ALGOS)
def test_degenerate_tokens(cuda_device, algo):
    """Zero query and zero key vectors (normalised to zero: no read, no write or
    erase), beta at 0 and 1, and a gate of 0 (no decay)."""
    x = synth.gdn_inputs(2, 130, 2, dtype=torch.bfloat16, seed=34, s0_std=0.1)
    x["q"][0, 5] = 0
    x["k"][0, 6] = 0
    x["k"][1, 64:70] = 0
    x["beta"][0, 10:20] = 0
    x["beta"][1, 20:40] = 1
    x["g"][0, 30:100] = 0
    o_ref, s_ref = ref(x)
    o, s = run(to_dev(x, cuda_device), algo)
    check(o, s, o_ref, s_ref, torch.bfloat16, f"gdn degenerate {algo}")
    assert float(o[0, 5].abs().max()) == 0.0


def test_empty_and_state_copy(cuda_device):
    x = synth.gdn_inputs(2, 0, 2, dtype=torch.bfloat16, seed=35, s0_std=0.1)
    xd = to_dev(x, cuda_device)
    for algo in ALGOS:
        o, s = run(xd, algo)
        assert o.shape == (2, 0, 2, 64)
        torch.testing.assert_close(s, xd["s0"], rtol=0, atol=0)
    shared = xd["s0"][:1].contiguous()
    _, s = run(xd, "auto", s0=shared)
    torch.testing.assert_close(s, shared.expand(2, -1, -1, -1), rtol=0, atol=0)


def test_chunked_is_deterministic(cuda_device):
    x = to_dev(synth.gdn_inputs(2, 333, 4, dtype=torch.bfloat16, seed=36, s0_std=0.1),
               cuda_device)
    o1, s1 = run(x, "chunked")
    o2, s2 = run(x, "chunked")
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_full_size_workload_all_units(cuda_device):
    """B=8, T=4096, H=64 bf16 (the GDN benchmark's workload, in its launch
    configuration): every one of the 512 (b, h) units against one oracle call."""
    p = synth.WORKLOADS["gdn_fwd_bf16_b8_t4096_h64"]
    x = synth.gdn_inputs(p["B"], p["T"], p["H"], dtype=torch.bfloat16, seed=p["seed"],
                         s0_std=p["s0_std"])
    o, s = run(to_dev(x, cuda_device), "auto")
    o_ref, s_ref = ref(x)
    eo, es = check(o, s, o_ref, s_ref, torch.bfloat16, "gdn full size")
    print(f"gdn full size: rel(o) {eo:.3e} rel(sT) {es:.3e}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_step_matches_oracle(cuda_device, dtype):
    B, H = 37, 4
    state = torch.randn(B, H, 64, 64, generator=torch.Generator().manual_seed(40)) * 0.1
    x = synth.gdn_step_inputs(B, H, dtype=dtype, seed=41, step=0)
    o_ref, s_ref = oracle.gdn_step(*(x[n] for n in NAMES), state)
    sd = state.to(cuda_device)
    o = wkv7_gdn_step(*(to_dev(x, cuda_device)[n] for n in NAMES), sd)
    check(o, sd, o_ref, s_ref, dtype, f"gdn step {dtype}")


def test_steps_equal_forward(cuda_device):
    """Eight consecutive decode steps reproduce the forward over the same tokens."""
    x = synth.gdn_inputs(5, 8, 3, dtype=torch.float32, seed=42, s0_std=0.1)
    xd = to_dev(x, cuda_device)
    o_fwd, s_fwd = run(xd, "recurrent")
    state = xd["s0"].clone()
    for t in range(8):
        ot = wkv7_gdn_step(*(xd[n][:, t].contiguous() for n in NAMES), state)
        torch.testing.assert_close(ot, o_fwd[:, t], rtol=0, atol=2e-5)
    torch.testing.assert_close(state, s_fwd, rtol=0, atol=2e-5)
    o_ref, s_ref = ref(x)
    assert rel_err(state, s_ref) < 1e-5


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("T", [1, 65, 200])
def test_head_first_layout(cuda_device, algo, T):
    """head_first=True (README: q, k, v [B,H,T,*], g and beta [B,H,T]) gives the
    token-major results."""
    x = synth.gdn_inputs(2, T, 3, dtype=torch.bfloat16, seed=400 + T, s0_std=0.1)
    o_ref, s_ref = ref(x)
    xd = to_dev(x, cuda_device)
    hf = {n: (xd[n].transpose(1, 2).contiguous() if n != "s0" else xd[n]) for n in xd}
    o, s = wkv7_gdn_fwd(*(hf[n] for n in NAMES), s0=hf["s0"], algo=algo, head_first=True)
    assert o.shape == (2, 3, T, 64)
    check(o.transpose(1, 2), s, o_ref, s_ref, torch.bfloat16, f"gdn head_first {algo} T={T}")


# --- the Gated DeltaNet backward (wkv7_gdn_bwd) against its fp64 oracle --------------

GD = ("dq", "dk", "dv", "dg", "dbeta", "ds0")


def check_gdn_grads(g, ref, dtype, what):
    for n in GD:
        e = rel_err(g[n], ref[n])
        limit = (1e-4 if dtype == torch.float32 else (1e-3 if n == "ds0" else 2e-2))
        assert e <= limit, f"{what}: {n} rel {e:.3e} > {limit}"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [1, 9, 70])
def test_gdn_bwd_matches_oracle(cuda_device, dtype, T):
    from linear_attention_rnn_wkv7_b200 import wkv7_gdn_bwd
    x = synth.gdn_inputs(2, T, 3, dtype=dtype, seed=700 + T, s0_std=0.1)
    gen = torch.Generator().manual_seed(701 + T)
    dout = torch.randn(2, T, 3, 64, generator=gen).to(dtype)
    dsT = torch.randn(2, 3, 64, 64, generator=gen) * 0.1
    ref = oracle.gdn_bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], dsT=dsT)
    xd = to_dev(x, cuda_device)
    g = wkv7_gdn_bwd(*(xd[n] for n in NAMES), dout.to(cuda_device), s0=xd["s0"],
                     dsT=dsT.to(cuda_device))
    check_gdn_grads(g, ref, dtype, f"gdn bwd T={T} {dtype}")


@pytest.mark.parametrize("head_first", [False, True])
def test_gdn_bwd_varlen_shared_state(cuda_device, head_first):
    from linear_attention_rnn_wkv7_b200 import wkv7_gdn_bwd
    lengths = torch.tensor([9, 0, 40, 1])
    x = synth.gdn_varlen_inputs(lengths, 2, dtype=torch.float32, seed=710, s0_std=0.1)
    cu = x.pop("cu_seqlens")
    shared = x["s0"][:1].clone()
    total = int(lengths.sum())
    gen = torch.Generator().manual_seed(711)
    dout = torch.randn(1, total, 2, 64, generator=gen)
    dsT = torch.randn(4, 2, 64, 64, generator=gen) * 0.1
    ref = oracle.gdn_bwd(*(x[n] for n in NAMES), dout, s0=shared, dsT=dsT, cu_seqlens=cu)
    xd = to_dev(x, cuda_device)
    lay = (lambda t: t.transpose(1, 2).contiguous()) if head_first else (lambda t: t)
    g = wkv7_gdn_bwd(*(lay(xd[n]) for n in NAMES), lay(dout.to(cuda_device)),
                     s0=shared.to(cuda_device), dsT=dsT.to(cuda_device),
                     cu_seqlens=cu.to(cuda_device), head_first=head_first)
    if head_first:
        g = {n: (t.transpose(1, 2) if n not in ("ds0",) else t) for n, t in g.items()}
    assert g["ds0"].shape == (1, 2, 64, 64)
    check_gdn_grads(g, ref, torch.float32, f"gdn bwd varlen shared head_first={head_first}")


def test_gdn_autograd(cuda_device):
    from linear_attention_rnn_wkv7_b200 import gated_delta_net, wkv7_gdn_bwd
    x = to_dev(synth.gdn_inputs(2, 30, 2, dtype=torch.bfloat16, seed=720, s0_std=0.1),
               cuda_device)
    leaves = {n: x[n].clone().requires_grad_(True) for n in NAMES}
    s0 = x["s0"].clone().requires_grad_(True)
    o, sT = gated_delta_net(*(leaves[n] for n in NAMES), initial_state=s0)
    gen = torch.Generator().manual_seed(721)
    do = torch.randn(o.shape, generator=gen).to(o.dtype).to(cuda_device)
    dsT = (torch.randn(sT.shape, generator=gen) * 0.1).to(cuda_device)
    ((o.float() * do.float()).sum() + (sT * dsT).sum()).backward()
    g = wkv7_gdn_bwd(*(x[n] for n in NAMES), do, s0=x["s0"], dsT=dsT)
    for n in NAMES:
        torch.testing.assert_close(leaves[n].grad, g["d" + n], rtol=0, atol=0)
    torch.testing.assert_close(s0.grad, g["ds0"], rtol=0, atol=0)
