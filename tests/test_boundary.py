"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every
entry point that include/wkv7.h declares, and rejects bad arguments with the
documented status codes before touching the device."""
import ctypes
import os
import re

import pytest
import torch

import linear_attention_rnn_wkv7_b200 as wkv7
from linear_attention_rnn_wkv7_b200 import build as wkv7_build
from linear_attention_rnn_wkv7_b200.wkv7 import (BF16, ERR_CUDA, ERR_INVALID_ARG, ERR_UNSUPPORTED,
                                                 F32, OK)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    wkv7_build.build()
    return wkv7.library()


def declared_functions():
    names = []
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*"
                            r"(wkv7_[A-Za-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("wkv7_fwd", "wkv7_step", "wkv7_bwd", "wkv7_bwd_workspace_bytes",
                     "wkv7_gdn_fwd", "wkv7_gdn_step", "wkv7_gdn_bwd",
                     "wkv7_gdn_bwd_workspace_bytes", "wkv7_get_last_error",
                     "wkv7_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libwkv7.so does not export {name}"


def test_status_strings(lib):
    assert wkv7.status_string(OK) == "WKV7_OK"
    assert wkv7.status_string(ERR_UNSUPPORTED) == "WKV7_ERR_UNSUPPORTED"
    assert lib.wkv7_version() >= 10000


# Fake, 16-byte aligned device addresses: every call below must be rejected by
# the host-side checks, so nothing is ever dereferenced or launched.
P = 0x7f0000000000
MIS = P + 2


def fwd(lib, ptrs=None, B=1, T=8, H=2, K=64, V=64, cu=None, N=None, dtype=BF16, algo=0,
        s0=None, sT=None, o=None, mask=None, layout=0):
    ptrs = ptrs or [P + 0x1000 * i for i in range(6)]
    o = P + 0x10000 if o is None else o
    N = B if N is None else N
    return lib.wkv7_fwd(*[ctypes.c_void_p(x) if x else None for x in ptrs],
                        ctypes.c_void_p(s0) if s0 else None, ctypes.c_void_p(mask) if mask else None,
                        ctypes.c_void_p(o) if o else None, ctypes.c_void_p(sT) if sT else None,
                        B, T, H, K, V, ctypes.c_void_p(cu) if cu else None, N, layout, dtype, algo,
                        None)


def test_fwd_rejects_bad_arguments(lib):
    assert fwd(lib, K=32, V=32) == ERR_UNSUPPORTED
    assert fwd(lib, K=64, V=128) == ERR_UNSUPPORTED
    assert fwd(lib, H=0) == ERR_INVALID_ARG
    assert fwd(lib, B=-1) == ERR_INVALID_ARG
    assert fwd(lib, T=-3) == ERR_INVALID_ARG
    assert fwd(lib, dtype=7) == ERR_INVALID_ARG
    assert fwd(lib, algo=9) == ERR_INVALID_ARG
    assert fwd(lib, layout=2) == ERR_INVALID_ARG
    assert fwd(lib, ptrs=[P, 0, P + 32, P + 48, P + 64, P + 80]) == ERR_INVALID_ARG  # null w
    assert fwd(lib, ptrs=[P, MIS, P + 32, P + 48, P + 64, P + 80]) == ERR_INVALID_ARG
    assert fwd(lib, o=0) == ERR_INVALID_ARG
    assert fwd(lib, o=P) == ERR_INVALID_ARG  # o aliases r
    assert fwd(lib, s0=MIS) == ERR_INVALID_ARG
    assert fwd(lib, sT=MIS) == ERR_INVALID_ARG
    assert fwd(lib, B=2, N=3) == ERR_INVALID_ARG  # N must equal B without cu_seqlens
    assert fwd(lib, B=2, cu=P + 0x20000, N=2) == ERR_INVALID_ARG  # varlen needs B == 1
    assert fwd(lib, cu=P + 0x20001, N=2) == ERR_INVALID_ARG  # misaligned cu_seqlens
    assert fwd(lib, dtype=F32, algo=2) == ERR_UNSUPPORTED  # chunked form is bf16 only
    # nothing to do: zero sequences, no launch
    assert fwd(lib, B=0, N=0) == OK
    assert fwd(lib, cu=P + 0x20000, N=0, T=0) == OK


def test_step_rejects_bad_arguments(lib):
    ptrs = [ctypes.c_void_p(P + 0x1000 * i) for i in range(6)]
    st, o = ctypes.c_void_p(P + 0x10000), ctypes.c_void_p(P + 0x20000)
    assert lib.wkv7_step(*ptrs, st, o, 4, 2, 32, 32, BF16, None) == ERR_UNSUPPORTED
    assert lib.wkv7_step(*ptrs, st, o, 4, 0, 64, 64, BF16, None) == ERR_INVALID_ARG
    assert lib.wkv7_step(*ptrs, st, o, 4, 2, 64, 64, 5, None) == ERR_INVALID_ARG
    assert lib.wkv7_step(*ptrs, st, st, 4, 2, 64, 64, BF16, None) == ERR_INVALID_ARG  # o == state
    assert lib.wkv7_step(*ptrs, None, o, 4, 2, 64, 64, BF16, None) == ERR_INVALID_ARG
    assert lib.wkv7_step(*ptrs, ctypes.c_void_p(P + 0x10004), o, 4, 2, 64, 64, BF16,
                         None) == ERR_INVALID_ARG
    assert lib.wkv7_step(*ptrs, st, o, 0, 2, 64, 64, BF16, None) == OK  # empty batch


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        wkv7.wkv7_fwd(x, x, x, x, x, x)
    with pytest.raises(ValueError, match="CUDA"):
        wkv7.wkv7_step(x[:, 0], x[:, 0], x[:, 0], x[:, 0], x[:, 0], x[:, 0],
                       torch.zeros(1, 1, 64, 64))


def gdn(lib, ptrs=None, B=1, T=8, H=2, K=64, V=64, cu=None, N=None, dtype=BF16, algo=0,
        s0=None, shared=0, sT=None, o=None, layout=0):
    ptrs = ptrs or [P + 0x1000 * i for i in range(5)]
    o = P + 0x10000 if o is None else o
    N = B if N is None else N
    return lib.wkv7_gdn_fwd(*[ctypes.c_void_p(x) if x else None for x in ptrs],
                            ctypes.c_void_p(s0) if s0 else None, shared,
                            ctypes.c_void_p(o) if o else None, ctypes.c_void_p(sT) if sT else None,
                            B, T, H, K, V, ctypes.c_void_p(cu) if cu else None, N, layout, dtype,
                            algo, None)


def test_gdn_fwd_rejects_bad_arguments(lib):
    assert gdn(lib, K=128) == ERR_UNSUPPORTED
    assert gdn(lib, H=0) == ERR_INVALID_ARG
    assert gdn(lib, dtype=3) == ERR_INVALID_ARG
    assert gdn(lib, algo=5) == ERR_INVALID_ARG
    assert gdn(lib, shared=2) == ERR_INVALID_ARG
    assert gdn(lib, layout=-1) == ERR_INVALID_ARG
    assert gdn(lib, ptrs=[P, P + 16, P + 32, 0, P + 64]) == ERR_INVALID_ARG  # null g
    assert gdn(lib, ptrs=[P, P + 16, P + 32, P + 49, P + 64]) == ERR_INVALID_ARG  # odd bf16 g
    assert gdn(lib, ptrs=[P, P + 16, P + 32, P + 50, P + 66], dtype=F32) == ERR_INVALID_ARG
    assert gdn(lib, ptrs=[P, P + 8, P + 32, P + 48, P + 64]) == ERR_INVALID_ARG  # k not 16-aligned
    assert gdn(lib, o=P) == ERR_INVALID_ARG  # o aliases q
    assert gdn(lib, B=2, N=3) == ERR_INVALID_ARG
    assert gdn(lib, B=2, s0=P + 0x30000, sT=P + 0x30000, shared=1) == ERR_INVALID_ARG
    assert gdn(lib, dtype=F32, algo=2) == ERR_UNSUPPORTED
    assert gdn(lib, B=0, N=0) == OK


def test_gdn_step_rejects_bad_arguments(lib):
    ptrs = [ctypes.c_void_p(P + 0x1000 * i) for i in range(5)]
    st, o = ctypes.c_void_p(P + 0x10000), ctypes.c_void_p(P + 0x20000)
    assert lib.wkv7_gdn_step(*ptrs, st, o, 4, 2, 32, 64, BF16, None) == ERR_UNSUPPORTED
    assert lib.wkv7_gdn_step(*ptrs, st, o, 4, 0, 64, 64, BF16, None) == ERR_INVALID_ARG
    assert lib.wkv7_gdn_step(*ptrs, st, st, 4, 2, 64, 64, BF16, None) == ERR_INVALID_ARG
    bad = ptrs[:3] + [ctypes.c_void_p(P + 0x3001), ptrs[4]]
    assert lib.wkv7_gdn_step(*bad, st, o, 4, 2, 64, 64, BF16, None) == ERR_INVALID_ARG
    assert lib.wkv7_gdn_step(*ptrs, st, o, 0, 2, 64, 64, BF16, None) == OK


def test_gdn_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 64, dtype=torch.bfloat16)
    s = torch.zeros(1, 4, 1, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        wkv7.wkv7_gdn_fwd(x, x, x, s, s)
    with pytest.raises(ValueError, match="CUDA"):
        wkv7.wkv7_gdn_step(x[:, 0], x[:, 0], x[:, 0], s[:, 0], s[:, 0],
                           torch.zeros(1, 1, 64, 64))


def test_bwd_rejects_bad_arguments(lib):
    ins = [ctypes.c_void_p(P + 0x1000 * i) for i in range(6)]
    dout = ctypes.c_void_p(P + 0x8000)
    outs = [ctypes.c_void_p(P + 0x10000 + 0x1000 * i) for i in range(6)]
    ws = ctypes.c_void_p(P + 0x100000)
    need = lib.wkv7_bwd_workspace_bytes(1, 16, 2, 64, 64, 1)
    # the larger of the two families' needs: the fp32 recurrences (checkpoints every
    # 8 tokens and every token's u) and the chunked form (reversed-sequence offsets and
    # the fp16 state checkpoints of both passes; every region 256-byte aligned)
    rows, N, H = 16, 1, 2
    rec = (H * (rows // 8 + 2 * N + 1) * 4096 + rows * H * 64) * 4
    al = lambda x: (x + 255) // 256 * 256
    rows_r = rows + 64 * N
    ck_f = al(4 * (N + 1))
    ck_r = al(ck_f + H * (rows // 64 + N + 1) * 8192)
    chk = al(ck_r + H * (rows_r // 64 + N + 1) * 8192)
    assert need == max(rec, chk)
    q = lib.wkv7_bwd_workspace_bytes_algo
    q.restype = ctypes.c_size_t
    AUTO, RECURRENT, CHUNKED = 0, 1, 2
    assert q(1, 16, 2, 64, 64, 1, BF16, AUTO) == chk
    assert q(1, 16, 2, 64, 64, 1, BF16, CHUNKED) == chk
    assert q(1, 16, 2, 64, 64, 1, BF16, RECURRENT) == rec
    assert q(1, 16, 2, 64, 64, 1, F32, AUTO) == rec
    assert q(1, 16, 2, 64, 64, 1, F32, CHUNKED) == 0
    assert q(1, 16, 2, 128, 128, 1, BF16, AUTO) == 0
    assert lib.wkv7_bwd_workspace_bytes(1, 16, 2, 128, 128, 1) == 0

    def call(B=1, T=16, H=2, K=64, V=64, dtype=BF16, d=dout, o=outs, w=ws, n=need, N=None,
             layout=0):
        return lib.wkv7_bwd(*ins, None, None, d, None, *o, None, B, T, H, K, V, None,
                            B if N is None else N, layout, dtype, w, n, None)

    assert call(K=128, V=128) == ERR_UNSUPPORTED
    assert call(H=0) == ERR_INVALID_ARG
    assert call(dtype=4) == ERR_INVALID_ARG
    assert call(d=None) == ERR_INVALID_ARG
    assert call(d=ctypes.c_void_p(P + 0x8008)) == ERR_INVALID_ARG  # misaligned dout
    assert call(o=[ins[0]] + outs[1:]) == ERR_INVALID_ARG  # dr aliases r
    assert call(n=chk - 1) == ERR_INVALID_ARG  # workspace too small (bf16: the chunked form)
    assert call(n=rec - 1, dtype=F32) == ERR_INVALID_ARG  # (fp32: the recurrences)
    assert call(w=None) == ERR_INVALID_ARG
    assert call(N=2) == ERR_INVALID_ARG  # N must equal B without cu_seqlens
    assert call(layout=3) == ERR_INVALID_ARG
    assert call(B=0) == OK


def test_stall_hook_arguments(lib):
    """The timeout-path test hook takes a thread index of the chunked kernel's CTA, or
    -1 to cancel; nothing is launched by the call itself."""
    assert lib.wkv7_test_stall_next_chunked(-2) == ERR_INVALID_ARG
    assert lib.wkv7_test_stall_next_chunked(256) == ERR_INVALID_ARG
    assert lib.wkv7_test_stall_next_chunked(5) == OK
    assert lib.wkv7_test_stall_next_chunked(-1) == OK


def test_schedule_hook_arguments(lib):
    """The chunked kernel's schedule query checks its arguments on the host; with no
    device to query it reports WKV7_ERR_CUDA and writes nothing."""
    r, c, m = ctypes.c_int(-7), ctypes.c_longlong(-7), ctypes.c_longlong(-7)
    out = (ctypes.byref(r), ctypes.byref(c), ctypes.byref(m))
    assert lib.wkv7_test_chunked_schedule(512, 4096, None, out[1], out[2]) == ERR_INVALID_ARG
    assert lib.wkv7_test_chunked_schedule(512, 4096, out[0], None, out[2]) == ERR_INVALID_ARG
    assert lib.wkv7_test_chunked_schedule(-1, 4096, *out) == ERR_INVALID_ARG
    assert lib.wkv7_test_chunked_schedule(512, -1, *out) == ERR_INVALID_ARG
    if not torch.cuda.is_available():
        assert lib.wkv7_test_chunked_schedule(512, 4096, *out) == ERR_CUDA
    assert (r.value, c.value, m.value) == (-7, -7, -7)


def test_sane_entry_points_reject_bad_arguments(lib):
    """wkv7_sane_fwd / wkv7_sane_step: host checks before any launch."""
    p = [ctypes.c_void_p(P + 0x1000 * i) for i in range(8)]
    tau = ctypes.c_void_p(P + 0x20000)
    o = ctypes.c_void_p(P + 0x30000)
    # forward: T >= 16 needs tau; layout, dtype and s0_shared range; head size; aliasing
    assert lib.wkv7_sane_fwd(*p[:6], None, None, None, 0, o, None, 1, 32, 2, 64, 64, 0, 0,
                             None) == ERR_INVALID_ARG
    assert lib.wkv7_sane_fwd(*p[:6], tau, None, None, 0, o, None, 1, 32, 2, 64, 64, 2, 0,
                             None) == ERR_INVALID_ARG
    assert lib.wkv7_sane_fwd(*p[:6], tau, None, None, 2, o, None, 1, 32, 2, 64, 64, 0, 0,
                             None) == ERR_INVALID_ARG
    assert lib.wkv7_sane_fwd(*p[:6], tau, None, None, 0, o, None, 1, 32, 2, 96, 96, 0, 0,
                             None) == ERR_UNSUPPORTED
    assert lib.wkv7_sane_fwd(*p[:6], tau, None, None, 0, p[0], None, 1, 32, 2, 64, 64, 0, 0,
                             None) == ERR_INVALID_ARG
    assert lib.wkv7_sane_fwd(*p[:6], ctypes.c_void_p(P + 2), None, None, 0, o, None, 1, 32, 2,
                             64, 64, 0, 0, None) == ERR_INVALID_ARG
    # T < 16 needs no tau; B = 0 launches nothing
    assert lib.wkv7_sane_fwd(*p[:6], None, None, None, 0, o, None, 0, 15, 2, 64, 64, 0, 0,
                             None) == OK
    # step: tau required, do_sane_all in {0, 1}, state and o distinct
    st = ctypes.c_void_p(P + 0x40000)
    assert lib.wkv7_sane_step(*p[:6], None, None, 1, st, o, 2, 2, 64, 64, 0, None) == ERR_INVALID_ARG
    assert lib.wkv7_sane_step(*p[:6], tau, None, 2, st, o, 2, 2, 64, 64, 0, None) == ERR_INVALID_ARG
    assert lib.wkv7_sane_step(*p[:6], tau, None, 1, st, st, 2, 2, 64, 64, 0, None) == ERR_INVALID_ARG
    assert lib.wkv7_sane_step(*p[:6], tau, None, 1, st, o, 2, 2, 96, 96, 0, None) == ERR_UNSUPPORTED
