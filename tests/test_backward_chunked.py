"""GPU parity of the tensor-core (chunked) backward, wkv7_bwd for bf16 inputs, against
the fp64 backward oracle, on the cases the fp32 tests of test_backward.py cover for the
recurrent kernels: masks (masked tokens at and next to 64-token chunk boundaries),
packed sequences (empty, 1-token, exactly 64, ragged), packed sequences with a mask,
both layouts, optional states, and decays at both ends of the chunked form's range.
The bf16 recurrent kernels stay covered here too (algo="recurrent").

Tolerances as in test_backward.py: rel <= 2e-2 for the bf16 gradients, rel <= 1e-3 for
ds0, rel(X) = max |X_gpu - X_ref| / max |X_ref|; masked tokens have exactly zero dw,
dk, dv, da, db."""
import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import WKV7Error, synth, wkv7_bwd, wkv7_get_last_error
from linear_attention_rnn_wkv7_b200.wkv7 import ERR_UNSUPPORTED, OK
from parity_util import to_dev
from test_backward import GRADS, NAMES, check_grads, upstream

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


def _run(xd, dout, dev, **kw):
    return wkv7_bwd(*(xd[n] for n in NAMES), dout.to(dev), **kw)


def _chunk_mask(B, T, seed):
    """Random masked tokens plus masked tokens at 63, 64, 127 and the last token."""
    g = torch.Generator().manual_seed(seed)
    m = (torch.rand(B, T, generator=g) >= 0.15).to(torch.uint8)
    for t in (0, 63, 64, 127, T - 1):
        if t < T:
            m[0, t] = 0
    return m


@pytest.mark.parametrize("algo", ["chunked", "recurrent"])
def test_bwd_bf16_mask_and_optional_states(cuda_device, algo):
    B, T, H = 3, 200, 2
    x = synth.fwd_inputs(B, T, H, dtype=BF, seed=700, s0_std=0.1)
    mask = _chunk_mask(B, T, 701)
    dout, dsT = upstream(B, T, H, BF, 702)
    xd = to_dev(x, cuda_device)
    for s0, d in ((x["s0"], dsT), (None, None), (x["s0"], None)):
        ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=s0, mask=mask, dsT=d)
        g = _run(xd, dout, cuda_device, s0=None if s0 is None else xd["s0"],
                 mask=mask.to(cuda_device), dsT=None if d is None else d.to(cuda_device),
                 algo=algo)
        check_grads(g, ref, BF, f"{algo} mask s0={s0 is not None} dsT={d is not None}")
        m = mask.bool().to(cuda_device)
        for n in ("dw", "dk", "dv", "da", "db"):
            assert float(g[n][~m].abs().max()) == 0.0, n
    assert wkv7_get_last_error() == OK


@pytest.mark.parametrize("head_first", [False, True])
@pytest.mark.parametrize("with_mask", [False, True])
def test_chunked_bwd_varlen(cuda_device, head_first, with_mask):
    """Packed sequences of lengths 0, 1, 17, 64, 130, 63, 200 (chunk boundaries inside,
    at and next to the sequence ends), per-sequence s0 and dL/dS_T."""
    lengths = torch.tensor([17, 0, 64, 1, 130, 63, 200])
    H = 2
    x = synth.varlen_inputs(lengths, H, dtype=BF, seed=710, s0_std=0.1)
    cu = x.pop("cu_seqlens")
    total, N = int(lengths.sum()), lengths.numel()
    dout, _ = upstream(1, total, H, BF, 711)
    dsT = torch.randn(N, H, 64, 64, generator=torch.Generator().manual_seed(712)) * 0.1
    mask = None
    if with_mask:
        g = torch.Generator().manual_seed(713)
        mask = (torch.rand(1, total, generator=g) >= 0.2).to(torch.uint8)
        for s0_, L in zip(cu[:-1].tolist(), lengths.tolist()):
            for t in (0, L - 1, 63, 64):
                if 0 <= t < L:
                    mask[0, s0_ + t] = 0
    ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], mask=mask, dsT=dsT,
                     cu_seqlens=cu)
    xd = to_dev(x, cuda_device)
    lay = (lambda t: t.transpose(1, 2).contiguous()) if head_first else (lambda t: t)
    g = wkv7_bwd(*(lay(xd[n]) for n in NAMES), lay(dout.to(cuda_device)), s0=xd["s0"],
                 dsT=dsT.to(cuda_device), cu_seqlens=cu.to(cuda_device),
                 mask=None if mask is None else mask.to(cuda_device), head_first=head_first,
                 algo="chunked")
    if head_first:
        g = {n: (t.transpose(1, 2) if n != "ds0" else t) for n, t in g.items()}
    check_grads(g, ref, BF, f"chunked varlen head_first={head_first} mask={with_mask}")
    assert wkv7_get_last_error() == OK


@pytest.mark.parametrize("decay", ["none", "strong", "mixed"])
def test_chunked_bwd_extreme_decays(cuda_device, decay):
    """w = 0 (E_t = 1), w = -1.2 (a chunk's decay spans e^{-76}, near the exponent clamp)
    and channels mixing the two: the gradient kernel's E_t, 1/E_t and e^{g} factors at
    both ends of their range."""
    B, T, H = 2, 200, 2
    x = synth.fwd_inputs(B, T, H, dtype=BF, seed=720, s0_std=0.1)
    w = x["w"].float()
    if decay == "none":
        w = torch.zeros_like(w)
    elif decay == "strong":
        w = torch.full_like(w, -1.2)
    else:
        w = torch.where(torch.arange(64) % 2 == 0, torch.zeros_like(w), torch.full_like(w, -1.2))
    x["w"] = w.to(BF).contiguous()
    dout, dsT = upstream(B, T, H, BF, 721)
    ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], dsT=dsT)
    g = _run(to_dev(x, cuda_device), dout, cuda_device, s0=to_dev(x, cuda_device)["s0"],
             dsT=dsT.to(cuda_device), algo="chunked")
    check_grads(g, ref, BF, f"chunked decay={decay}")


def test_chunked_bwd_matches_recurrent_at_full_size(cuda_device):
    """B=8, T=4096, H=64 bf16: the two kernel families agree on every unit (the oracle
    comparison of sampled units is test_backward.py's; this covers all 512)."""
    p = synth.WORKLOADS["fwd_bf16_b8_t4096_h64"]
    x = to_dev(synth.fwd_inputs(p["B"], p["T"], p["H"], dtype=BF, seed=p["seed"],
                                s0_std=p["s0_std"]), cuda_device)
    dout, dsT = upstream(p["B"], p["T"], p["H"], BF, 730)
    gc = _run(x, dout, cuda_device, s0=x["s0"], dsT=dsT.to(cuda_device), algo="chunked")
    gr = _run(x, dout, cuda_device, s0=x["s0"], dsT=dsT.to(cuda_device), algo="recurrent")
    for n in GRADS:
        a, b = gc[n].double(), gr[n].double()
        e = float((a - b).abs().max() / b.abs().max())
        limit = 2e-3 if n == "ds0" else 4e-2  # both sides carry their own error
        assert e <= limit, f"{n}: chunked vs recurrent rel {e:.3e} > {limit}"


def test_chunked_bwd_rejects_fp32(cuda_device):
    x = to_dev(synth.fwd_inputs(1, 16, 1, dtype=torch.float32, seed=740, s0_std=0.1),
               cuda_device)
    dout = torch.zeros(1, 16, 1, 64, device=cuda_device)
    with pytest.raises(WKV7Error) as e:
        wkv7_bwd(*(x[n] for n in NAMES), dout, algo="chunked")
    assert e.value.status == ERR_UNSUPPORTED


def test_chunked_bwd_is_deterministic(cuda_device):
    x = to_dev(synth.fwd_inputs(2, 300, 3, dtype=BF, seed=750, s0_std=0.1), cuda_device)
    dout, dsT = upstream(2, 300, 3, BF, 751)
    g0 = _run(x, dout, cuda_device, s0=x["s0"], dsT=dsT.to(cuda_device))
    g1 = _run(x, dout, cuda_device, s0=x["s0"], dsT=dsT.to(cuda_device))
    for n in GRADS:
        assert torch.equal(g0[n], g1[n]), n


def test_chunked_bwd_larger_magnitudes(cuda_device):
    """States around 10 and values around 100 (the gradient kernel carries V, dO, S0 and
    dSL as fp16 operands, exact in range up to 65504), as the forward's test does."""
    B, T, H = 2, 200, 2
    x = synth.fwd_inputs(B, T, H, dtype=BF, seed=760, s0_std=10.0)
    x["v"] = (x["v"].float() * 100.0).to(BF).contiguous()
    dout, dsT = upstream(B, T, H, BF, 761)
    ref = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], dsT=dsT)
    xd = to_dev(x, cuda_device)
    g = _run(xd, dout, cuda_device, s0=xd["s0"], dsT=dsT.to(cuda_device), algo="chunked")
    check_grads(g, ref, BF, "chunked larger magnitudes")
