"""GPU parity for head sizes 128 and 256 (the README's head_size argument; rwkv-ops
0.9.0 README, "rwkv7op 使用方法") against the fp64 oracles, which are written for any
K and V.  These sizes run on the CUDA-core kernels (recurrent forward, decode step);
the chunked tensor-core kernel is built for K = V = 64 and refuses other sizes."""
import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import (WKV7Error, synth, wkv7_fwd, wkv7_gdn_fwd,
                                            wkv7_gdn_step, wkv7_step)
from linear_attention_rnn_wkv7_b200.wkv7 import ERR_UNSUPPORTED
from parity_util import check, to_dev

pytestmark = pytest.mark.gpu

SIZES = [128, 256]


@pytest.mark.parametrize("D", SIZES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_fwd_head_sizes(cuda_device, D, dtype):
    x = synth.fwd_inputs(2, 37, 2, K=D, V=D, dtype=dtype, seed=500 + D, s0_std=0.1)
    mask = torch.ones(2, 37, dtype=torch.uint8)
    mask[0, 10:14] = 0
    o_ref, s_ref, _ = oracle.fwd(*(x[n] for n in "rwkvab"), s0=x["s0"], mask=mask)
    xd = to_dev(x, cuda_device)
    o, s = wkv7_fwd(*(xd[n] for n in "rwkvab"), s0=xd["s0"], mask=mask.to(cuda_device))
    tol_dtype = torch.bfloat16 if dtype == torch.bfloat16 else torch.float32
    check(o, s, o_ref, s_ref, tol_dtype, f"fwd D={D} {dtype}")
    with pytest.raises(WKV7Error) as e:
        wkv7_fwd(*(xd[n] for n in "rwkvab"), s0=xd["s0"], algo="chunked")
    assert e.value.status == ERR_UNSUPPORTED


@pytest.mark.parametrize("D", SIZES)
def test_fwd_head_sizes_varlen_head_first(cuda_device, D):
    lengths = torch.tensor([5, 0, 40])
    x = synth.varlen_inputs(lengths, 2, K=D, V=D, dtype=torch.bfloat16, seed=510 + D,
                            s0_std=0.1)
    cu = x.pop("cu_seqlens")
    o_ref, s_ref, _ = oracle.fwd(*(x[n] for n in "rwkvab"), s0=x["s0"], cu_seqlens=cu)
    xd = to_dev(x, cuda_device)
    hf = {n: (xd[n].transpose(1, 2).contiguous() if n != "s0" else xd[n]) for n in xd}
    o, s = wkv7_fwd(*(hf[n] for n in "rwkvab"), s0=hf["s0"], cu_seqlens=cu.to(cuda_device),
                    head_first=True)
    check(o.transpose(1, 2), s, o_ref, s_ref, torch.bfloat16, f"varlen head_first D={D}")


@pytest.mark.parametrize("D", SIZES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_step_head_sizes(cuda_device, D, dtype):
    state = synth.decode_state(9, 3, K=D, V=D, seed=520 + D)
    x = synth.decode_step_inputs(9, 3, K=D, V=D, dtype=dtype, seed=521 + D)
    o_ref, s_ref = oracle.step(*(x[n] for n in "rwkvab"), state)
    sd = state.to(cuda_device)
    o = wkv7_step(*(to_dev(x, cuda_device)[n] for n in "rwkvab"), sd)
    check(o, sd, o_ref, s_ref, dtype, f"step D={D} {dtype}")


@pytest.mark.parametrize("D", SIZES)
def test_gdn_head_sizes(cuda_device, D):
    names = ("q", "k", "v", "g", "beta")
    x = synth.gdn_inputs(2, 45, 2, K=D, V=D, dtype=torch.float32, seed=530 + D, s0_std=0.1)
    o_ref, s_ref, _ = oracle.gdn_fwd(*(x[n] for n in names), s0=x["s0"])
    xd = to_dev(x, cuda_device)
    o, s = wkv7_gdn_fwd(*(xd[n] for n in names), s0=xd["s0"])
    check(o, s, o_ref, s_ref, torch.float32, f"gdn fwd D={D}")
    state = synth.decode_state(7, 2, K=D, V=D, seed=540 + D)
    y = synth.gdn_step_inputs(7, 2, K=D, V=D, dtype=torch.bfloat16, seed=541 + D)
    o_ref, s_ref = oracle.gdn_step(*(y[n] for n in names), state)
    sd = state.to(cuda_device)
    o = wkv7_gdn_step(*(to_dev(y, cuda_device)[n] for n in names), sd)
    check(o, sd, o_ref, s_ref, torch.bfloat16, f"gdn step D={D}")
