"""wkv7_bwd_noalloc: the backward on the library's static scratch (a file-scope device
array) instead of a caller workspace.  It must give exactly wkv7_bwd's results on
problems that fit, and refuse larger ones before touching the device."""
import ctypes
import threading

import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import build as wkv7_build
from linear_attention_rnn_wkv7_b200 import library, synth, wkv7_bwd
from linear_attention_rnn_wkv7_b200.wkv7 import (ERR_UNSUPPORTED, BF16, WKV7Error,
                                                 wkv7_bwd_noalloc, wkv7_bwd_workspace_bytes)
from parity_util import rel_err, to_dev

NAMES = ("r", "w", "k", "v", "a", "b")
STATIC_SCRATCH_BYTES = 64 << 20  # WKV7_STATIC_SCRATCH_BYTES in include/wkv7.h


def test_header_constant_and_refusal_on_cpu():
    """The header's scratch size; a problem whose workspace exceeds it is refused by the
    host check (nothing is launched, so this runs without a GPU)."""
    import os
    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "wkv7.h")).read()
    assert "#define WKV7_STATIC_SCRATCH_BYTES (64u << 20)" in hdr
    wkv7_build.build()
    lib = library()
    B, T, H = 8, 4096, 64
    assert wkv7_bwd_workspace_bytes(B, T, H) > STATIC_SCRATCH_BYTES
    fake = [ctypes.c_void_p(0x7f0000000000 + 0x1000 * i) for i in range(16)]
    st = lib.wkv7_bwd_noalloc(*fake[:6], None, None, fake[6], None, *fake[7:13], None,
                              B, T, H, 64, 64, None, B, 0, BF16, None)
    assert st == ERR_UNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_noalloc_equals_workspace_call(cuda_device, dtype):
    B, T, H = 2, 100, 3
    assert wkv7_bwd_workspace_bytes(B, T, H) <= STATIC_SCRATCH_BYTES
    x = synth.fwd_inputs(B, T, H, dtype=dtype, seed=800, s0_std=0.1)
    gen = torch.Generator().manual_seed(801)
    dout = torch.randn(B, T, H, 64, generator=gen).to(dtype)
    dsT = torch.randn(B, H, 64, 64, generator=gen) * 0.1
    xd = to_dev(x, cuda_device)
    args = [xd[n] for n in NAMES] + [dout.to(cuda_device)]
    g0 = wkv7_bwd(*args, s0=xd["s0"], dsT=dsT.to(cuda_device))
    g1 = wkv7_bwd_noalloc(*args, s0=xd["s0"], dsT=dsT.to(cuda_device))
    for n in g0:
        assert torch.equal(g0[n], g1[n]), n
    ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], dsT=dsT)
    limit = 1e-4 if dtype == torch.float32 else 2e-2
    for n in ("dr", "dw", "dk", "dv", "da", "db"):
        assert rel_err(g1[n], ref[n]) <= limit, n


@pytest.mark.gpu
def test_noalloc_refuses_large_problem(cuda_device):
    B, T, H = 4, 4096, 32  # the bf16 (chunked) workspace is over the static scratch
    assert wkv7_bwd_workspace_bytes(B, T, H, dtype=torch.bfloat16, algo="auto") > STATIC_SCRATCH_BYTES
    x = to_dev(synth.fwd_inputs(B, T, H, dtype=torch.bfloat16, seed=802, s0_std=0.1),
               cuda_device)
    dout = torch.zeros(B, T, H, 64, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(WKV7Error) as e:
        wkv7_bwd_noalloc(*(x[n] for n in NAMES), dout, s0=x["s0"])
    assert e.value.status == ERR_UNSUPPORTED


@pytest.mark.gpu
def test_noalloc_makes_no_handoff_area(cuda_device):
    """More (sequence, head) units than the GPU holds CTAs at once: wkv7_bwd runs its
    two chunked forward runs on the balanced schedule (with the library's handoff area),
    while wkv7_bwd_noalloc, called from a host thread that has no handoff area yet, must
    not make one and runs them one unit per CTA.  The results are the same bits."""
    B, T, H = 5, 200, 64
    assert wkv7_bwd_workspace_bytes(B, T, H, dtype=torch.bfloat16, algo="auto") <= STATIC_SCRATCH_BYTES
    x = to_dev(synth.fwd_inputs(B, T, H, dtype=torch.bfloat16, seed=803, s0_std=0.1), cuda_device)
    gen = torch.Generator().manual_seed(804)
    dout = torch.randn(B, T, H, 64, generator=gen).to(torch.bfloat16).to(cuda_device)
    dsT = (torch.randn(B, H, 64, 64, generator=gen) * 0.1).to(cuda_device)
    args = [x[n] for n in NAMES] + [dout]
    g0 = wkv7_bwd(*args, s0=x["s0"], dsT=dsT)
    torch.cuda.synchronize()
    out = {}

    def run():
        try:
            torch.cuda.set_device(cuda_device)
            out["g"] = wkv7_bwd_noalloc(*args, s0=x["s0"], dsT=dsT)
            torch.cuda.synchronize()
        except Exception as e:  # re-raised below, in the test's thread
            out["err"] = e

    t = threading.Thread(target=run)
    t.start()
    t.join()
    if "err" in out:
        raise out["err"]
    for n in g0:
        assert torch.equal(g0[n], out["g"][n]), n
