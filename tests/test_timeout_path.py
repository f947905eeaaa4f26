"""The chunked kernel's failure path on the GPU, made to run without any fault.

Every wait of the chunked kernel on a TMA copy or a tcgen05 MMA is bounded.  A thread
that gives up raises WKV7_ERR_DEVICE_TIMEOUT; its CTA agrees on abandoning the
sequence at the next barrier (__syncthreads_or), waits (bounded) for the copies and
MMAs it issued, frees its tensor memory and returns.  The test hook makes one thread
of the first CTA wait, with a 2 ms limit, on an mbarrier that nothing arrives at, at a
point where no copy or MMA is in flight: nothing faults, traps or hangs.  The status
must come back, the other sequences must be right, and the next call must be exact."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import library, synth, wkv7_fwd, wkv7_get_last_error
from linear_attention_rnn_wkv7_b200.wkv7 import ERR_DEVICE_TIMEOUT, OK
from parity_util import check, rel_err, to_dev, BF16_O_REL, BF16_S_REL

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tid", [0, 37, 200])
def test_timeout_is_reported_and_context_stays_usable(cuda_device, tid):
    x = synth.fwd_inputs(2, 200, 3, dtype=torch.bfloat16, seed=700 + tid, s0_std=0.1)
    o_ref, s_ref, _ = oracle.fwd(x["r"], x["w"], x["k"], x["v"], x["a"], x["b"], s0=x["s0"])
    xd = to_dev(x, cuda_device)
    assert wkv7_get_last_error() == OK
    assert library().wkv7_test_stall_next_chunked(tid) == OK
    o, s = wkv7_fwd(*(xd[n] for n in "rwkvab"), s0=xd["s0"], algo="chunked")
    assert wkv7_get_last_error() == ERR_DEVICE_TIMEOUT
    assert wkv7_get_last_error() == OK  # cleared once read
    # The first CTA is unit (b=0, h=0); every other unit ran to completion.
    for b in range(2):
        for h in range(3):
            if (b, h) == (0, 0):
                continue
            assert rel_err(o[b, :, h], o_ref[b, :, h]) <= BF16_O_REL
            assert rel_err(s[b, h], s_ref[b, h]) <= BF16_S_REL
    # The hook was consumed: the next call is a normal one, and exact.
    o2, s2 = wkv7_fwd(*(xd[n] for n in "rwkvab"), s0=xd["s0"], algo="chunked")
    check(o2, s2, o_ref, s_ref, torch.bfloat16, "after the timeout")
    assert wkv7_get_last_error() == OK
