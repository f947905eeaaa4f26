"""Shared helpers of the GPU parity tests: error measures and the oracle call on
a sample of (sequence, head) units."""
import numpy as np
import torch

import oracle

# Tolerances (max over the compared tensor):
#   fp32 inputs: max |gpu - oracle| <= 1e-4 on o and the final state;
#   bf16 inputs: rel(o) <= 2e-2 and rel(final state) <= 1e-3, where
#   rel(X) = max |X_gpu - X_ref| / max(max |X_ref|, 1e-6).
F32_ABS = 1e-4
BF16_O_REL = 2e-2
BF16_S_REL = 1e-3


def rel_err(x, ref) -> float:
    x = x.detach().double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-6)) if ref.size else 0.0


def abs_err(x, ref) -> float:
    x = x.detach().double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(x - ref).max()) if ref.size else 0.0


def check(o_gpu, s_gpu, o_ref, s_ref, dtype, what=""):
    if dtype == torch.float32:
        eo, es = abs_err(o_gpu, o_ref), (abs_err(s_gpu, s_ref) if s_ref is not None else 0.0)
        assert eo <= F32_ABS, f"{what}: o max-abs {eo:.3e} > {F32_ABS}"
        assert es <= F32_ABS, f"{what}: sT max-abs {es:.3e} > {F32_ABS}"
    else:
        eo, es = rel_err(o_gpu, o_ref), (rel_err(s_gpu, s_ref) if s_ref is not None else 0.0)
        assert eo <= BF16_O_REL, f"{what}: o rel {eo:.3e} > {BF16_O_REL}"
        assert es <= BF16_S_REL, f"{what}: sT rel {es:.3e} > {BF16_S_REL}"
    return eo, es


def oracle_units(x, units, mask=None):
    """Oracle on a sample of (b, h) units of a [B,T,H,*] problem.
    Returns o [len(units),T,V] and sT [len(units),K,V] (float64)."""
    os_, ss = [], []
    for (bb, h) in units:
        sl = lambda t: t[bb:bb + 1, :, h:h + 1]
        s0 = None if x.get("s0") is None else x["s0"][bb:bb + 1, h:h + 1]
        m = None if mask is None else mask[bb:bb + 1]
        o, s, _ = oracle.fwd(sl(x["r"]), sl(x["w"]), sl(x["k"]), sl(x["v"]), sl(x["a"]),
                             sl(x["b"]), s0=s0, mask=m)
        os_.append(o[0, :, 0])
        ss.append(s[0, 0])
    return np.stack(os_), np.stack(ss)


def to_dev(x, device):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
