"""Property-based pins of the oracles over random small shapes (hypothesis, CPU): the
sequential oracle against the dense-product form, the Gated DeltaNet oracle against the
generalized rule under its substitution, and the backward against finite differences.
Shapes include K != V, single tokens and single heads."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
from oracle import brute

shapes = st.tuples(st.integers(1, 2), st.integers(1, 9), st.integers(1, 2), st.integers(1, 4),
                   st.integers(1, 4), st.integers(0, 2**31 - 1))


def _inputs(B, T, H, K, V, seed):
    rng = np.random.default_rng(seed)
    x = {n: rng.standard_normal((B, T, H, V if n == "v" else K)) for n in "rkvab"}
    x["w"] = -rng.random((B, T, H, K))
    x["a"] *= 0.5
    x["b"] *= 0.5
    return x, rng.standard_normal((B, H, K, V)), rng


@settings(max_examples=25, deadline=None)
@given(shapes)
def test_sequential_equals_dense_products(sh):
    B, T, H, K, V, seed = sh
    x, s0, _ = _inputs(B, T, H, K, V, seed)
    o, sT, _ = oracle.fwd(*(x[n] for n in "rwkvab"), s0=s0)
    ob, sb = brute.fwd(*(x[n] for n in "rwkvab"), s0=s0)
    np.testing.assert_allclose(o, ob, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(sT, sb, rtol=1e-10, atol=1e-10)


@settings(max_examples=25, deadline=None)
@given(shapes)
def test_gdn_equals_generalized_substitution(sh):
    B, T, H, K, V, seed = sh
    rng = np.random.default_rng(seed)
    q, k = rng.standard_normal((B, T, H, K)), rng.standard_normal((B, T, H, K))
    v = rng.standard_normal((B, T, H, V))
    g, beta = -rng.random((B, T, H)), rng.random((B, T, H))
    s0 = rng.standard_normal((B, H, K, V))
    o, sT, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s0)
    unit = lambda z: z / np.linalg.norm(z, axis=-1, keepdims=True)
    qh, kh = unit(q), unit(k)
    og, sg, _ = oracle.fwd(qh, np.repeat(g[..., None], K, -1), beta[..., None] * kh, v, kh,
                           -np.exp(g)[..., None] * beta[..., None] * kh, s0=s0)
    np.testing.assert_allclose(o, og, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(sT, sg, rtol=1e-10, atol=1e-10)


@settings(max_examples=10, deadline=None)
@given(st.tuples(st.integers(1, 5), st.integers(1, 3), st.integers(1, 3),
                 st.integers(0, 2**31 - 1)))
def test_backward_equals_finite_differences(sh):
    T, K, V, seed = sh
    x, s0, rng = _inputs(1, T, 1, K, V, seed)
    dout = rng.standard_normal((1, T, 1, V))
    dsT = rng.standard_normal((1, 1, K, V))
    g = oracle.bwd(*(x[n] for n in "rwkvab"), dout, s0=s0, dsT=dsT)

    def loss():
        o, sT, _ = oracle.fwd(*(x[n] for n in "rwkvab"), s0=s0)
        return float(np.sum(o * dout) + np.sum(sT * dsT))

    eps = 1e-6
    for n in "rwkvab":
        idx = tuple(rng.integers(0, d) for d in x[n].shape)  # one random coordinate each
        keep = x[n][idx]
        x[n][idx] = keep + eps
        lp = loss()
        x[n][idx] = keep - eps
        lm = loss()
        x[n][idx] = keep
        np.testing.assert_allclose(g["d" + n][idx], (lp - lm) / (2 * eps), rtol=1e-5, atol=1e-6)


@settings(max_examples=10, deadline=None)
@given(st.tuples(st.integers(1, 5), st.integers(1, 3), st.integers(1, 3), st.booleans(),
                 st.integers(0, 2**31 - 1)))
def test_gdn_backward_equals_finite_differences(sh):
    T, K, V, shared, seed = sh
    rng = np.random.default_rng(seed)
    x = {"q": rng.standard_normal((2, T, 1, K)), "k": rng.standard_normal((2, T, 1, K)),
         "v": rng.standard_normal((2, T, 1, V)), "g": -rng.random((2, T, 1)),
         "beta": rng.random((2, T, 1)),
         "s0": rng.standard_normal((1 if shared else 2, 1, K, V))}
    dout = rng.standard_normal((2, T, 1, V))
    dsT = rng.standard_normal((2, 1, K, V))
    names = ("q", "k", "v", "g", "beta")
    g = oracle.gdn_bwd(*(x[n] for n in names), dout, s0=x["s0"], dsT=dsT)

    def loss():
        o, sT, _ = oracle.gdn_fwd(*(x[n] for n in names), s0=x["s0"])
        return float(np.sum(o * dout) + np.sum(sT * dsT))

    eps = 1e-6
    for n in names + ("s0",):
        idx = tuple(rng.integers(0, d) for d in x[n].shape)
        keep = x[n][idx]
        x[n][idx] = keep + eps
        lp = loss()
        x[n][idx] = keep - eps
        lm = loss()
        x[n][idx] = keep
        np.testing.assert_allclose(g["d" + n][idx], (lp - lm) / (2 * eps), rtol=1e-5, atol=1e-6)
