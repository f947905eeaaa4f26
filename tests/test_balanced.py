"""The balanced schedule of the chunked kernel (units of one length, more units than
resident CTAs): the units' chunks are cut into equal runs, one per CTA, and a unit cut
between two CTAs passes its fp32 state from one to the other.

B=5, T=200 (four chunks, the last ragged), H=64 gives 320 units for the 296 CTAs a
B200 holds (two per SM): runs of five chunks, so most units are cut, at every offset
inside the unit.  The same problem given as packed sequences of equal length runs one
unit per CTA, with the same per-chunk arithmetic: the two must agree bit for bit (the
handoff is an exact fp32 copy), and both must match the oracle within the bf16
tolerances of the other parity tests."""
import ctypes

import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import (library, synth, wkv7_bwd, wkv7_fwd, wkv7_gdn_fwd,
                                            wkv7_get_last_error)
from linear_attention_rnn_wkv7_b200.wkv7 import ERR_DEVICE_TIMEOUT, OK
from parity_util import BF16_O_REL, BF16_S_REL, check, rel_err, to_dev
from test_backward import GRADS, check_grads, upstream

pytestmark = pytest.mark.gpu

BF = torch.bfloat16
B, T, H = 5, 200, 64
NAMES = ("r", "w", "k", "v", "a", "b")
GDN = ("q", "k", "v", "g", "beta")


def _packed(t):
    """[B, T, ...] -> [1, B*T, ...] (the packed form of equal-length sequences)."""
    return t.reshape(1, t.shape[0] * t.shape[1], *t.shape[2:])


def _cu(device):
    return torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device=device)


def _schedule(units, length):
    """(resident CTAs, CTAs, chunks per CTA) of the chunked kernel for this problem."""
    res, ctas, cmax = ctypes.c_int(), ctypes.c_longlong(), ctypes.c_longlong()
    assert library().wkv7_test_chunked_schedule(units, length, ctypes.byref(res),
                                                ctypes.byref(ctas), ctypes.byref(cmax)) == OK
    return res.value, ctas.value, cmax.value


def test_schedule_geometry(cuda_device):
    """Two CTAs per SM; the problem here takes the balanced schedule; runs of at least
    one unit's chunks, every chunk covered, no more CTAs than are resident."""
    res, ctas, cmax = _schedule(B * H, T)
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    assert res == 2 * sms, (res, sms)
    C = (T + 63) // 64
    assert B * H > res and cmax >= C and 0 < ctas <= res
    assert ctas * cmax >= B * H * C > (ctas - 1) * cmax
    assert _schedule(res, T)[1:] == (0, 0)  # as many units as slots: one unit per CTA


@pytest.fixture(scope="module")
def problem():
    return synth.fwd_inputs(B, T, H, dtype=BF, seed=900, s0_std=0.1)


def test_forward_balanced_is_exact_and_matches_oracle(cuda_device, problem):
    x = problem
    xd = to_dev(x, cuda_device)
    o, s = wkv7_fwd(*(xd[n] for n in NAMES), s0=xd["s0"], algo="chunked")
    op, sp = wkv7_fwd(*(_packed(xd[n]) for n in NAMES), s0=xd["s0"], cu_seqlens=_cu(cuda_device),
                      algo="chunked")
    assert torch.equal(o, op.reshape(o.shape)), "o: balanced vs one unit per CTA"
    assert torch.equal(s, sp), "sT: balanced vs one unit per CTA"
    o_ref, s_ref, _ = oracle.fwd(*(x[n] for n in NAMES), s0=x["s0"])
    check(o, s, o_ref, s_ref, BF, "balanced forward")
    assert wkv7_get_last_error() == OK


def test_forward_balanced_mask_head_first_in_place(cuda_device, problem):
    """Masked tokens (including whole masked chunks), the head-first layout, and the
    final state written over s0."""
    x = problem
    g = torch.Generator().manual_seed(901)
    mask = (torch.rand(B, T, generator=g) >= 0.1).to(torch.uint8)
    mask[1, 64:128] = 0
    mask[3, 150:] = 0
    o_ref, s_ref, _ = oracle.fwd(*(x[n] for n in NAMES), s0=x["s0"], mask=mask)
    xd = to_dev(x, cuda_device)
    hf = {n: xd[n].transpose(1, 2).contiguous() for n in NAMES}
    st = xd["s0"].clone()
    o, s = wkv7_fwd(*(hf[n] for n in NAMES), s0=st, sT=st, mask=mask.to(cuda_device),
                    head_first=True, algo="chunked")
    assert s.data_ptr() == st.data_ptr()
    check(o.transpose(1, 2), s, o_ref, s_ref, BF, "balanced, masked, head first, in place")


def test_gdn_forward_balanced(cuda_device):
    x = synth.gdn_inputs(B, T, H, dtype=BF, seed=902, s0_std=0.1)
    xd = to_dev(x, cuda_device)
    o, s = wkv7_gdn_fwd(*(xd[n] for n in GDN), s0=xd["s0"], algo="chunked")
    op, sp = wkv7_gdn_fwd(*(_packed(xd[n]) for n in GDN), s0=xd["s0"],
                          cu_seqlens=_cu(cuda_device), algo="chunked")
    assert torch.equal(o, op.reshape(o.shape))
    assert torch.equal(s, sp)
    o_ref, s_ref, _ = oracle.gdn_fwd(*(x[n] for n in GDN), s0=x["s0"])
    check(o, s, o_ref, s_ref, BF, "balanced Gated DeltaNet forward")


def test_backward_balanced(cuda_device, problem):
    """Both forward runs of the chunked backward (the checkpointing run and the reversed
    run, 256 tokens per reversed sequence) take the balanced schedule here."""
    x = problem
    xd = to_dev(x, cuda_device)
    dout, dsT = upstream(B, T, H, BF, 903)
    g = wkv7_bwd(*(xd[n] for n in NAMES), dout.to(cuda_device), s0=xd["s0"],
                 dsT=dsT.to(cuda_device), algo="chunked")
    gp = wkv7_bwd(*(_packed(xd[n]) for n in NAMES), _packed(dout.to(cuda_device)), s0=xd["s0"],
                  dsT=dsT.to(cuda_device), cu_seqlens=_cu(cuda_device), algo="chunked")
    for n in GRADS:
        assert torch.equal(g[n], gp[n].reshape(g[n].shape)), n
    ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], dsT=dsT)
    check_grads(g, ref, BF, "balanced backward")


def test_timeout_in_balanced_run(cuda_device, problem):
    """The first CTA gives up at its first chunk (the test hook).  Its run is unit 0
    onwards and ends with the last chunks of a unit whose first chunks the second CTA
    ran and handed over; every unit outside that run must be right, and the next call
    (whose handoff flags carry a new value) exact."""
    x = problem
    xd = to_dev(x, cuda_device)
    o_ref, s_ref, _ = oracle.fwd(*(x[n] for n in NAMES), s0=x["s0"])
    assert wkv7_get_last_error() == OK
    assert library().wkv7_test_stall_next_chunked(0) == OK
    o, s = wkv7_fwd(*(xd[n] for n in NAMES), s0=xd["s0"], algo="chunked")
    assert wkv7_get_last_error() == ERR_DEVICE_TIMEOUT
    _, _, cmax = _schedule(B * H, T)
    first_ctas_units = -(-cmax // ((T + 63) // 64))  # units with chunks in the first CTA's run
    for b in range(B):
        for h in range(H):
            if b * H + h < first_ctas_units:
                continue
            assert rel_err(o[b, :, h], o_ref[b, :, h]) <= BF16_O_REL, (b, h)
            assert rel_err(s[b, h], s_ref[b, h]) <= BF16_S_REL, (b, h)
    o2, s2 = wkv7_fwd(*(xd[n] for n in NAMES), s0=xd["s0"], algo="chunked")
    check(o2, s2, o_ref, s_ref, BF, "after the timeout")
    assert wkv7_get_last_error() == OK


def test_graph_replay_balanced(cuda_device, problem):
    """A captured balanced launch replays correctly: each consumer clears its handoff
    flag, so a replay (same flag value) never reads the previous replay's state."""
    xd = to_dev(problem, cuda_device)
    side = torch.cuda.Stream(device=cuda_device)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # the handoff area of this stream exists before capture
        o0, s0 = wkv7_fwd(*(xd[n] for n in NAMES), s0=xd["s0"], algo="chunked")
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        og, sg = wkv7_fwd(*(xd[n] for n in NAMES), s0=xd["s0"], algo="chunked")
    for _ in range(3):
        og.zero_()
        sg.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(og, o0)
        assert torch.equal(sg, s0)
    del graph
    assert wkv7_get_last_error() == OK
