"""The state gradient as a forward run over the reversed sequence, in fp64 (no GPU).

With G_t = dL/dS_t for L = sum(o . dout) + sum(S_T . dsT), the backward of the
generalized delta rule is again a recurrence of the same form read backwards:
    G_t = r_t do_t^T + M_{t+1}^T G_{t+1},   G_{L-1} = r do^T + dsT,   ds0 = M_0^T G_0,
with M_t = diag(e^{w_t}) + b_t a_t^T (the transition) and dv_t = G_t^T k_t.  The
transpose of M_t is diag(e^{w_t}) + a_t b_t^T, so X_tau = G_{L-1-tau} is the forward
recurrence with w' = w_{L-tau}, a' = b_{L-tau}, b' = a_{L-tau} (tau >= 1; the identity
at tau = 0 and for a masked token), write pair k' = r_{L-1-tau}, v' = do_{L-1-tau}
(tau < L), read vector r' = k_{L-1-tau}, started from dsT; one more transition with no
write (tau = L) gives ds0.  The tensor-core backward runs it on sequences padded at
the start with p = 63 - L mod 64 identity steps (length 64 (L // 64 + 1)), so that the
reversed chunks end right after the original chunks' last tokens.

This test builds those reversed, padded sequences, runs the forward oracle over them
and compares ds0 and dv with the backward oracles (generalized rule with masks, and
Gated DeltaNet, whose transition e^{g} (I - beta kh kh^T) is symmetric, with write key
beta kh, a = kh, b = -e^{g} beta kh, read vector qh)."""
import numpy as np
import pytest

import oracle


def _reversed_run(w, a, b, r, k, dout, dsT, mask=None):
    """Forward oracle over the reversed, padded sequence of one (sequence, head).
    w, a, b, r, k [L, K]; dout [L, V]; dsT [K, V].  Returns (dv [L, V], ds0)."""
    L, K = w.shape
    V = dout.shape[1]
    p = 63 - L % 64
    n = p + L + 1
    assert n % 64 == 0
    wr, ar, br, kr, vr, rr = (np.zeros((n, d)) for d in (K, K, K, K, V, K))
    for tau in range(L + 1):
        j = p + tau
        t1, t2 = L - tau, L - 1 - tau
        if tau >= 1 and (mask is None or mask[t1]):
            wr[j], ar[j], br[j] = w[t1], b[t1], a[t1]
        if tau < L:
            kr[j], vr[j], rr[j] = r[t2], dout[t2], k[t2]
    lift = lambda z: z[None, :, None]
    o, sT, _ = oracle.fwd(lift(rr), lift(wr), lift(kr), lift(vr), lift(ar), lift(br),
                          s0=dsT[None, None])
    dv = o[0, p:p + L, 0][::-1].copy()  # step p + tau reads dv of token L - 1 - tau
    if mask is not None:
        dv[~mask.astype(bool)] = 0.0
    return dv, sT[0, 0]


@pytest.mark.parametrize("L", [1, 63, 64, 65, 150])
def test_wkv7_state_gradient_is_a_reversed_forward_run(L):
    rng = np.random.default_rng(L)
    K, V = 8, 6
    r, k, a, b = (rng.standard_normal((L, K)) for _ in range(4))
    a, b = 0.4 * a, 0.4 * b  # asymmetric: the a / b swap matters
    w = -0.6 * rng.random((L, K))
    v, dout = rng.standard_normal((L, V)), rng.standard_normal((L, V))
    s0, dsT = 0.1 * rng.standard_normal((K, V)), 0.1 * rng.standard_normal((K, V))
    mask = (rng.random(L) >= 0.2).astype(np.uint8)
    mask[L // 2] = 0
    lift = lambda z: z[None, :, None]
    g = oracle.bwd(*(lift(x) for x in (r, w, k, v, a, b)), lift(dout), s0=s0[None, None],
                   mask=mask[None], dsT=dsT[None, None])
    dv, ds0 = _reversed_run(w, a, b, r, k, dout, dsT, mask)
    np.testing.assert_allclose(ds0, g["ds0"][0, 0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv, g["dv"][0, :, 0], rtol=1e-12, atol=1e-13)


def test_swapping_a_and_b_is_needed():
    """The same run without the a / b swap misses ds0 (asymmetric transition)."""
    rng = np.random.default_rng(7)
    L, K, V = 40, 8, 6
    r, k, a, b = (rng.standard_normal((L, K)) for _ in range(4))
    w = -0.6 * rng.random((L, K))
    v, dout = rng.standard_normal((L, V)), rng.standard_normal((L, V))
    dsT = 0.1 * rng.standard_normal((K, V))
    lift = lambda z: z[None, :, None]
    g = oracle.bwd(*(lift(x) for x in (r, w, k, v, 0.4 * a, 0.4 * b)), lift(dout),
                   dsT=dsT[None, None])
    _, ds0 = _reversed_run(w, 0.4 * b, 0.4 * a, r, k, dout, dsT)  # roles not swapped
    assert np.abs(ds0 - g["ds0"][0, 0]).max() > 1e-3 * np.abs(g["ds0"]).max()


@pytest.mark.parametrize("L", [1, 64, 100])
def test_gated_deltanet_state_gradient_is_a_reversed_forward_run(L):
    rng = np.random.default_rng(100 + L)
    K, V = 8, 6
    q, k = rng.standard_normal((L, K)), rng.standard_normal((L, K))
    v, dout = rng.standard_normal((L, V)), rng.standard_normal((L, V))
    gate = -0.5 * rng.random(L)
    beta = rng.random(L)
    s0, dsT = 0.1 * rng.standard_normal((K, V)), 0.1 * rng.standard_normal((K, V))
    qh = q / np.linalg.norm(q, axis=1, keepdims=True)
    kh = k / np.linalg.norm(k, axis=1, keepdims=True)
    eg, bt = np.exp(gate)[:, None], beta[:, None]
    g = oracle.gdn_bwd(q[None, :, None], k[None, :, None], v[None, :, None],
                       gate[None, :, None], beta[None, :, None], dout[None, :, None],
                       s0=s0[None, None], dsT=dsT[None, None])
    # generalized-rule inputs of Gated DeltaNet: w = g on every channel, a = kh,
    # b = -e^g beta kh, write key beta kh, read vector qh
    w = np.repeat(gate[:, None], K, axis=1)
    dv, ds0 = _reversed_run(w, kh, -eg * bt * kh, qh, bt * kh, dout, dsT)
    np.testing.assert_allclose(ds0, g["ds0"][0, 0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv, g["dv"][0, :, 0], rtol=1e-12, atol=1e-13)
