"""GPU parity of wkv7_step (single-token decode, state updated in place)
against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import synth, wkv7_fwd, wkv7_step
from parity_util import abs_err, rel_err, BF16_O_REL, BF16_S_REL, F32_ABS

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,H", [(1, 1), (3, 5), (37, 2)])
def test_step_matches_oracle(cuda_device, dtype, B, H):
    state = synth.decode_state(B, H, seed=9, std=0.1)
    st_dev = state.to(cuda_device)
    ref_state = state.double().numpy()
    for step in range(6):
        x = synth.decode_step_inputs(B, H, dtype=dtype, seed=9, step=step)
        o = wkv7_step(*(x[n].to(cuda_device) for n in "rwkvab"), st_dev)
        o_ref, ref_state = oracle.step(x["r"], x["w"], x["k"], x["v"], x["a"], x["b"], ref_state)
        if dtype == torch.float32:
            assert abs_err(o, o_ref) <= F32_ABS
            assert abs_err(st_dev, ref_state) <= F32_ABS
        else:
            assert rel_err(o, o_ref) <= BF16_O_REL
            assert rel_err(st_dev, ref_state) <= BF16_S_REL


def test_steps_equal_forward_on_gpu(cuda_device):
    """T decode steps == one forward over the same T tokens (both on the GPU)."""
    B, H, T = 4, 3, 70
    x = synth.fwd_inputs(B, T, H, dtype=torch.bfloat16, seed=13, s0_std=0.1)
    xd = {k: v.to(cuda_device) for k, v in x.items()}
    o_fwd, s_fwd = wkv7_fwd(xd["r"], xd["w"], xd["k"], xd["v"], xd["a"], xd["b"], s0=xd["s0"],
                            algo="recurrent")
    st = xd["s0"].clone()
    outs = []
    for t in range(T):
        outs.append(wkv7_step(*(xd[n][:, t].contiguous() for n in "rwkvab"), st))
    o_steps = torch.stack(outs, 1)
    assert rel_err(o_steps, o_fwd.double().cpu().numpy()) <= 1e-2
    assert rel_err(st, s_fwd.double().cpu().numpy()) <= 1e-5
