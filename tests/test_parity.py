"""GPU parity of wkv7_fwd against the fp64 oracle on the same seeded inputs.

Small problems are compared element by element in full; they span several
64-token chunks with ragged tails, masks, packed varlen sequences, null
initial / final states and the fp32 workload.  Edge cases: empty batches,
zero-length sequences, all-masked rows, bad cu_seqlens (flagged on the
device, never faulting), determinism, and canaries around the outputs."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_rnn_wkv7_b200 import synth, wkv7_fwd, wkv7_get_last_error, WKV7Error
from linear_attention_rnn_wkv7_b200.wkv7 import ERR_DEVICE_BAD_SEQLENS, ERR_UNSUPPORTED, OK
from parity_util import check, to_dev

pytestmark = pytest.mark.gpu

ALGOS = ["recurrent", "chunked"]


def run(x, algo, mask=None, cu=None, output_final_state=True, use_s0=True):
    try:
        return wkv7_fwd(x["r"], x["w"], x["k"], x["v"], x["a"], x["b"],
                        s0=x["s0"] if use_s0 else None, mask=mask, cu_seqlens=cu,
                        output_final_state=output_final_state, algo=algo)
    except WKV7Error as e:
        if e.status == ERR_UNSUPPORTED and algo == "chunked" and x["r"].dtype != torch.float32:
            pytest.skip("chunked kernel not built")
        raise


def ref(x, mask=None, cu=None, use_s0=True):
    o, s, _ = oracle.fwd(x["r"], x["w"], x["k"], x["v"], x["a"], x["b"],
                         s0=x["s0"] if use_s0 else None, mask=mask, cu_seqlens=cu)
    return o, s


def test_fp32_small_workload(cuda_device):
    """B=1, T=64, H=2, K=V=64, fp32, s0 = 0, no mask (seed 0): max-abs <= 1e-4."""
    p = synth.WORKLOADS["fwd_fp32_small"]
    x = synth.fwd_inputs(p["B"], p["T"], p["H"], dtype=torch.float32, seed=p["seed"], s0_std=0.0)
    o_ref, s_ref = ref(x)
    xd = to_dev(x, cuda_device)
    for use_s0 in (True, False):  # explicit zero state and s0 = NULL
        o, s = run(xd, "recurrent", use_s0=use_s0)
        check(o, s, o_ref, s_ref, torch.float32, f"fp32 workload use_s0={use_s0}")
    assert wkv7_get_last_error() == OK


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 200, 257])
def test_bf16_chunk_boundaries(cuda_device, algo, T):
    x = synth.fwd_inputs(2, T, 3, dtype=torch.bfloat16, seed=100 + T, s0_std=0.1)
    o_ref, s_ref = ref(x)
    o, s = run(to_dev(x, cuda_device), algo)
    check(o, s, o_ref, s_ref, torch.bfloat16, f"{algo} T={T}")


@pytest.mark.parametrize("algo", ALGOS)
def test_bf16_null_states(cuda_device, algo):
    x = synth.fwd_inputs(2, 130, 2, dtype=torch.bfloat16, seed=5, s0_std=0.1)
    o_ref, s_ref = ref(x, use_s0=False)
    o, s = run(to_dev(x, cuda_device), algo, use_s0=False, output_final_state=False)
    assert s is None
    check(o, None, o_ref, None, torch.bfloat16, f"{algo} null states")


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("decay", ["none", "strong", "mixed"])
def test_extreme_decays(cuda_device, algo, decay):
    """Per-step log decays at both ends of the range the chunked form is exact for:
    w = 0 (no decay: E_t = 1, a pure delta rule), w = -1.2 (a chunk's decay spans
    e^{-76}, near the exponent clamp of 80), and channels mixing the two."""
    x = synth.fwd_inputs(2, 200, 2, dtype=torch.bfloat16, seed=11, s0_std=0.1)
    w = x["w"].float()
    if decay == "none":
        w = torch.zeros_like(w)
    elif decay == "strong":
        w = torch.full_like(w, -1.2)
    else:
        w = torch.where(torch.arange(64) % 2 == 0, torch.zeros_like(w), torch.full_like(w, -1.2))
    x["w"] = w.to(torch.bfloat16).contiguous()
    o_ref, s_ref = ref(x)
    o, s = run(to_dev(x, cuda_device), algo)
    check(o, s, o_ref, s_ref, torch.bfloat16, f"{algo} decay={decay}")


@pytest.mark.parametrize("algo", ALGOS)
def test_larger_magnitudes(cuda_device, algo):
    """State entries around 10 and values around 100 (the chunked form carries S0 and
    V as fp16 operands, exact in range up to 65504)."""
    x = synth.fwd_inputs(2, 200, 2, dtype=torch.bfloat16, seed=13, s0_std=10.0)
    x["v"] = (x["v"].float() * 100.0).to(torch.bfloat16).contiguous()
    o_ref, s_ref = ref(x)
    o, s = run(to_dev(x, cuda_device), algo)
    check(o, s, o_ref, s_ref, torch.bfloat16, f"{algo} larger magnitudes")


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_mask(cuda_device, algo, dtype):
    if algo == "chunked" and dtype == torch.float32:
        pytest.skip("chunked form is bf16 only")
    B, T = 4, 300
    x = synth.fwd_inputs(B, T, 2, dtype=dtype, seed=21, s0_std=0.1)
    mask = synth.padding_mask(B, T, seed=2, max_suffix=100, interior_p=0.1)
    mask[1] = 0  # an all-masked row: state passes through unchanged
    mask[2] = 1  # an unmasked row
    o_ref, s_ref = ref(x, mask=mask)
    o, s = run(to_dev(x, cuda_device), algo, mask=mask.to(cuda_device))
    check(o, s, o_ref, s_ref, dtype, f"{algo} mask")
    torch.testing.assert_close(s[1].cpu(), x["s0"][1], rtol=0, atol=0)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_varlen(cuda_device, algo, dtype):
    if algo == "chunked" and dtype == torch.float32:
        pytest.skip("chunked form is bf16 only")
    lengths = torch.tensor([1, 15, 16, 64, 65, 0, 300, 129], dtype=torch.int64)
    x = synth.varlen_inputs(lengths, H=2, dtype=dtype, seed=31, s0_std=0.1)
    cu = x["cu_seqlens"]
    o_ref, s_ref = ref(x, cu=cu)
    o, s = run(to_dev(x, cuda_device), algo, cu=cu.to(cuda_device))
    check(o, s, o_ref, s_ref, dtype, f"{algo} varlen")


@pytest.mark.parametrize("algo", ALGOS)
def test_state_passing_on_gpu(cuda_device, algo):
    """Running [0, tau) then [tau, T) with sT fed back as s0 == running [0, T)."""
    x = synth.fwd_inputs(2, 200, 2, dtype=torch.bfloat16, seed=41, s0_std=0.1)
    xd = to_dev(x, cuda_device)
    o_full, s_full = run(xd, algo)
    tau = 77
    first = {k: (v[:, :tau].contiguous() if k != "s0" else v) for k, v in xd.items()}
    o1, s1 = run(first, algo)
    second = {k: (v[:, tau:].contiguous() if k != "s0" else s1) for k, v in xd.items()}
    o2, s2 = run(second, algo)
    o_ref, s_ref = ref(x)
    check(torch.cat([o1, o2], 1), s2, o_ref, s_ref, torch.bfloat16, f"{algo} state passing")


@pytest.mark.parametrize("algo", ALGOS)
def test_deterministic_and_fully_written(cuda_device, algo):
    x = to_dev(synth.fwd_inputs(3, 190, 2, dtype=torch.bfloat16, seed=51, s0_std=0.1),
               cuda_device)
    B, T, H, K = x["r"].shape
    # canaries: outputs live in the middle of larger NaN-filled buffers
    pad = 4096
    o_buf = torch.full((B * T * H * K + 2 * pad,), float("nan"), dtype=torch.bfloat16,
                       device=cuda_device)
    s_buf = torch.full((B * H * K * K + 2 * pad,), float("nan"), dtype=torch.float32,
                       device=cuda_device)
    o = o_buf[pad:pad + B * T * H * K].view(B, T, H, K)
    s = s_buf[pad:pad + B * H * K * K].view(B, H, K, K)
    try:
        wkv7_fwd(x["r"], x["w"], x["k"], x["v"], x["a"], x["b"], s0=x["s0"], algo=algo,
                 o=o, sT=s)
    except WKV7Error as e:
        if e.status == ERR_UNSUPPORTED:
            pytest.skip("chunked kernel not built")
        raise
    torch.cuda.synchronize()
    assert not torch.isnan(o).any() and not torch.isnan(s).any()
    assert torch.isnan(o_buf[:pad]).all() and torch.isnan(o_buf[-pad:]).all()
    assert torch.isnan(s_buf[:pad]).all() and torch.isnan(s_buf[-pad:]).all()
    o2, s2 = run(x, algo)
    assert torch.equal(o, o2) and torch.equal(s, s2)


def test_in_place_state(cuda_device):
    """s0 and sT may be the same buffer."""
    x = synth.fwd_inputs(2, 70, 2, dtype=torch.bfloat16, seed=61, s0_std=0.1)
    o_ref, s_ref = ref(x)
    xd = to_dev(x, cuda_device)
    st = xd["s0"].clone()
    for algo in ALGOS:
        st.copy_(xd["s0"])
        try:
            o, s = wkv7_fwd(xd["r"], xd["w"], xd["k"], xd["v"], xd["a"], xd["b"], s0=st, sT=st,
                            algo=algo)
        except WKV7Error as e:
            if e.status == ERR_UNSUPPORTED:
                continue
            raise
        check(o, st, o_ref, s_ref, torch.bfloat16, f"{algo} in-place state")


def test_empty_problems(cuda_device):
    x = to_dev(synth.fwd_inputs(2, 0, 2, dtype=torch.bfloat16, seed=1, s0_std=0.1), cuda_device)
    o, s = wkv7_fwd(x["r"], x["w"], x["k"], x["v"], x["a"], x["b"], s0=x["s0"])
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(s, x["s0"])  # T = 0: state passes through
    y = to_dev(synth.fwd_inputs(0, 16, 2, dtype=torch.bfloat16, seed=1, s0_std=None), cuda_device)
    o, s = wkv7_fwd(y["r"], y["w"], y["k"], y["v"], y["a"], y["b"])
    assert o.numel() == 0 and s.numel() == 0


@pytest.mark.parametrize("algo", ALGOS)
def test_bad_cu_seqlens_flagged_not_faulting(cuda_device, algo):
    lengths = torch.tensor([10, 20, 30])
    x = to_dev(synth.varlen_inputs(lengths, H=2, seed=71, s0_std=0.1), cuda_device)
    bad = torch.tensor([0, 25, 12, 60], dtype=torch.int32, device=cuda_device)  # decreasing
    try:
        wkv7_fwd(x["r"], x["w"], x["k"], x["v"], x["a"], x["b"], s0=x["s0"], cu_seqlens=bad,
                 algo=algo)
    except WKV7Error as e:
        if e.status == ERR_UNSUPPORTED:
            pytest.skip("chunked kernel not built")
        raise
    assert wkv7_get_last_error() == ERR_DEVICE_BAD_SEQLENS
    assert wkv7_get_last_error() == OK  # the flag is cleared once read


def _head_first(t):
    return t.transpose(1, 2).contiguous()


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("T", [1, 64, 130])
def test_head_first_layout(cuda_device, algo, T):
    """head_first=True ([B,H,T,*] inputs and output, README generalized_delta_rule
    argument): the same results as the token-major run, with and without a mask."""
    x = synth.fwd_inputs(2, T, 3, dtype=torch.bfloat16, seed=300 + T, s0_std=0.1)
    mask = torch.ones(2, T, dtype=torch.uint8)
    mask[1, T // 3:T // 2] = 0
    for m in (None, mask):
        o_ref, s_ref = ref(x, mask=m)
        xd = to_dev(x, cuda_device)
        hf = {n: (_head_first(xd[n]) if n != "s0" else xd[n]) for n in xd}
        o, s = wkv7_fwd(*(hf[n] for n in "rwkvab"), s0=hf["s0"],
                        mask=None if m is None else m.to(cuda_device), algo=algo,
                        head_first=True)
        assert o.shape == (2, 3, T, 64)
        check(o.transpose(1, 2), s, o_ref, s_ref, torch.bfloat16, f"head_first {algo} T={T}")


@pytest.mark.parametrize("algo", ALGOS)
def test_head_first_varlen(cuda_device, algo):
    lengths = torch.tensor([70, 0, 1, 129])
    x = synth.varlen_inputs(lengths, 2, dtype=torch.bfloat16, seed=310, s0_std=0.1)
    cu = x.pop("cu_seqlens")
    o_ref, s_ref = ref(x, cu=cu)
    xd = to_dev(x, cuda_device)
    hf = {n: (_head_first(xd[n]) if n != "s0" else xd[n]) for n in xd}
    o, s = wkv7_fwd(*(hf[n] for n in "rwkvab"), s0=hf["s0"], cu_seqlens=cu.to(cuda_device),
                    algo=algo, head_first=True)
    check(o.transpose(1, 2), s, o_ref, s_ref, torch.bfloat16, f"head_first varlen {algo}")


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("head_first", [False, True])
def test_varlen_with_mask(cuda_device, algo, head_first):
    """Packed sequences (cu_seqlens) together with a padding mask: the mask is [1, sum L]
    over the packed token rows (rwkv-ops 0.9.0 README, "rwkv7op 使用方法": mask[b, t] = 0
    leaves the state unchanged at that token).  Masked tokens fall at sequence starts,
    ends, chunk boundaries and the interior; one sequence is masked throughout."""
    lengths = torch.tensor([70, 0, 1, 129, 64, 200, 33], dtype=torch.int64)
    x = synth.varlen_inputs(lengths, 2, dtype=torch.bfloat16, seed=320, s0_std=0.1)
    cu = x.pop("cu_seqlens")
    total = int(lengths.sum())
    g = torch.Generator().manual_seed(321)
    mask = (torch.rand(1, total, generator=g) >= 0.15).to(torch.uint8)
    starts = cu[:-1].tolist()
    for s0_, L in zip(starts, lengths.tolist()):
        if L > 0:
            mask[0, s0_] = 0               # first token of every sequence
            mask[0, s0_ + L - 1] = 0       # last token
        if L > 64:
            mask[0, s0_ + 63] = 0          # a chunk's last token
            mask[0, s0_ + 64] = 0          # and the next chunk's first
    mask[0, starts[4]:starts[4] + 64] = 0  # the 64-token sequence is masked throughout
    o_ref, s_ref = ref(x, mask=mask, cu=cu)
    xd = to_dev(x, cuda_device)
    if head_first:
        xd = {n: (_head_first(xd[n]) if n != "s0" else xd[n]) for n in xd}
    o, s = wkv7_fwd(*(xd[n] for n in "rwkvab"), s0=xd["s0"], mask=mask.to(cuda_device),
                    cu_seqlens=cu.to(cuda_device), algo=algo, head_first=head_first)
    if head_first:
        o = o.transpose(1, 2)
    check(o, s, o_ref, s_ref, torch.bfloat16, f"varlen+mask {algo} head_first={head_first}")
    torch.testing.assert_close(s[4].cpu(), x["s0"][4], rtol=0, atol=0)
