"""The chunked (WY-form) algebra in fp64, checked against the oracles (no GPU).

The forward kernel rewrites each 64-token chunk exactly: with g_t the in-chunk prefix
of w, E_t = e^{g_t - g_L}, r~ = r E_t, a~ = a E_{t-1}, k~ = k / E_t, b~ = b / E_t, the
masked Gram products A_rk, A_rb (s <= t), A_ak, A_ab (s < t), T = (I - A_ab)^-1,
W = T Abar, Z = T A_ak, U = W S0 + Z V:
    O = Rbar S0 + A_rb U + A_rk V,   S_L = diag(e^{g_L}) S0 + Bhat^T U + Khat^T V.
This test runs that algebra in fp64 (torch on CPU) chunk by chunk and compares it with
the sequential oracle; then it runs the chunked backward (the adjoint of the same
algebra, written out by hand, carried across chunks in reverse) against the backward
oracle.  Both are independent routes to the oracles' results."""
import numpy as np
import pytest
import torch

import oracle


def _terms(r, w, k, a, b):
    g = torch.cumsum(w, 0)
    gL = g[-1]
    gm1 = torch.cat([torch.zeros_like(g[:1]), g[:-1]])
    E, Em1 = torch.exp(g - gL), torch.exp(gm1 - gL)
    return dict(g=g, gL=gL, gm1=gm1, E=E, Em1=Em1, rt=r * E, at=a * Em1, kt=k / E, bt=b / E,
                Abar=a * torch.exp(gm1), Rbar=r * torch.exp(g), gam=torch.exp(gL))


def _chunk_forward(S0, v, t):
    L = v.shape[0]
    low, slow = torch.tril(torch.ones(L, L)), torch.tril(torch.ones(L, L), -1)
    f = dict(A_rk=(t["rt"] @ t["kt"].T) * low, A_rb=(t["rt"] @ t["bt"].T) * low,
             A_ak=(t["at"] @ t["kt"].T) * slow, A_ab=(t["at"] @ t["bt"].T) * slow)
    f["T"] = torch.linalg.inv(torch.eye(L) - f["A_ab"])
    f["W"], f["Z"] = f["T"] @ t["Abar"], f["T"] @ f["A_ak"]
    f["U"] = f["W"] @ S0 + f["Z"] @ v
    O = t["Rbar"] @ S0 + f["A_rb"] @ f["U"] + f["A_rk"] @ v
    SL = t["gam"][:, None] * S0 + t["bt"].T @ f["U"] + t["kt"].T @ v
    return O, SL, f


def _chunk_backward(dO, dSL, S0, v, r, k, a, b, t, f):
    L = v.shape[0]
    low, slow = torch.tril(torch.ones(L, L)), torch.tril(torch.ones(L, L), -1)
    dU = f["A_rb"].T @ dO + t["bt"] @ dSL
    dV = f["A_rk"].T @ dO + t["kt"] @ dSL + f["Z"].T @ dU
    dS0 = t["Rbar"].T @ dO + t["gam"][:, None] * dSL + f["W"].T @ dU
    dA_rb, dA_rk = (dO @ f["U"].T) * low, (dO @ v.T) * low
    dRbar, dBhat, dKhat = dO @ S0.T, f["U"] @ dSL.T, v @ dSL.T
    dgam = (dSL * S0).sum(1)
    dW, dZ = dU @ S0.T, dU @ v.T
    dT = dW @ t["Abar"].T + dZ @ f["A_ak"].T
    dAbar = f["T"].T @ dW
    dA_ak = (f["T"].T @ dZ) * slow
    dA_ab = (f["T"].T @ dT @ f["T"].T) * slow
    drt = dA_rk @ t["kt"] + dA_rb @ t["bt"]
    dkt = dA_rk.T @ t["rt"] + dA_ak.T @ t["at"] + dKhat
    dat = dA_ak @ t["kt"] + dA_ab @ t["bt"]
    dbt = dA_rb.T @ t["rt"] + dA_ab.T @ t["at"] + dBhat
    E, Em1, g, gm1 = t["E"], t["Em1"], t["g"], t["gm1"]
    dr = drt * E + dRbar * torch.exp(g)
    da = dat * Em1 + dAbar * torch.exp(gm1)
    dk, db = dkt / E, dbt / E
    te = drt * r * E - dkt * k / E - dbt * b / E
    tm = dat * a * Em1
    dg = te + dRbar * r * torch.exp(g)
    dg[:-1] += tm[1:] + (dAbar * a * torch.exp(gm1))[1:]
    dg[-1] += -(te.sum(0) + tm.sum(0)) + dgam * t["gam"]
    dw = torch.flip(torch.cumsum(torch.flip(dg, [0]), 0), [0])
    return dict(dr=dr, dw=dw, dk=dk, dv=dV, da=da, db=db), dS0


def _problem(seed, T, K, V, asymmetric):
    rng = np.random.default_rng(seed)
    r, k, v = (rng.standard_normal((T, n)) for n in (K, K, V))
    w = -0.6 * rng.random((T, K))
    if asymmetric:
        a, b = 0.5 * rng.standard_normal((T, K)), 0.5 * rng.standard_normal((T, K))
    else:
        kh = k / np.linalg.norm(k, axis=1, keepdims=True)
        a, b = -kh, kh * rng.random((T, 1))
    s0 = 0.1 * rng.standard_normal((K, V))
    return dict(r=r, w=w, k=k, v=v, a=a, b=b), s0, rng


@pytest.mark.parametrize("T,asym", [(64, False), (150, False), (100, True)])
def test_chunked_forward_and_backward_match_the_oracles(T, asym):
    torch.set_default_dtype(torch.float64)
    try:
        x, s0, rng = _problem(T, T, 8, 6, asym)
        dout = rng.standard_normal((T, 6))
        dsT = 0.1 * rng.standard_normal((8, 6))
        lift = lambda z: z[None, :, None]
        o_ref, sT_ref, _ = oracle.fwd(*(lift(x[n]) for n in "rwkvab"), s0=s0[None, None])
        g_ref = oracle.bwd(*(lift(x[n]) for n in "rwkvab"), lift(dout), s0=s0[None, None],
                           dsT=dsT[None, None])
        X = {n: torch.tensor(z) for n, z in x.items()}
        starts = list(range(0, T, 64))
        S, S0s, O = torch.tensor(s0), [], []
        for c0 in starts:
            sl = {n: z[c0:c0 + 64] for n, z in X.items()}
            S0s.append(S)
            o, S, _ = _chunk_forward(S, sl["v"], _terms(sl["r"], sl["w"], sl["k"], sl["a"], sl["b"]))
            O.append(o)
        np.testing.assert_allclose(torch.cat(O).numpy(), o_ref[0, :, 0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S.numpy(), sT_ref[0, 0], rtol=1e-12, atol=1e-12)
        dS = torch.tensor(dsT)
        grads = {n: np.zeros_like(z) for n, z in x.items()}
        for ci in reversed(range(len(starts))):
            c0 = starts[ci]
            sl = {n: z[c0:c0 + 64] for n, z in X.items()}
            t = _terms(sl["r"], sl["w"], sl["k"], sl["a"], sl["b"])
            _, _, f = _chunk_forward(S0s[ci], sl["v"], t)
            g, dS = _chunk_backward(torch.tensor(dout[c0:c0 + 64]), dS, S0s[ci], sl["v"], sl["r"],
                                    sl["k"], sl["a"], sl["b"], t, f)
            for n in grads:
                grads[n][c0:c0 + 64] = g["d" + n].numpy()
        for n in grads:
            np.testing.assert_allclose(grads[n], g_ref["d" + n][0, :, 0], rtol=1e-10,
                                       atol=1e-10 * np.abs(g_ref["d" + n]).max(), err_msg=n)
        np.testing.assert_allclose(dS.numpy(), g_ref["ds0"][0, 0], rtol=1e-10, atol=1e-12)
    finally:
        torch.set_default_dtype(torch.float32)
