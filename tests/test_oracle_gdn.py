"""Pins for the Gated DeltaNet oracle (no GPU).  Each test checks ``oracle.gdn_fwd``
against something other than itself: a hand-worked example, an independent
dense-product form, the generalized delta rule oracle under the substitution
that makes it Gated DeltaNet, closed forms, and invariants of the operator.

The operator is gated_delta_net_recurrent / _chunk / _single_step (rwkv-ops 0.9.0
README, "gdn_recurrent 使用方法" and "gdn_chunk 使用方法"): q, k [B,T,H,K]
L2-normalised inside, v [B,T,H,V], g [B,T,H] a log-space decay gate, beta [B,T,H]
a write strength in (0, 1), initial state [N,H,K,V] or [1,H,K,V].
"""
import json
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from linear_attention_rnn_wkv7_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "gdn_hand_worked.json")


def rand_gdn(rng, B, T, H, K, V, s0=True, g_scale=1.0):
    q = rng.standard_normal((B, T, H, K))
    k = rng.standard_normal((B, T, H, K))
    v = rng.standard_normal((B, T, H, V))
    g = -g_scale * rng.random((B, T, H))
    beta = rng.random((B, T, H))
    st = rng.standard_normal((B, H, K, V)) if s0 else None
    return q, k, v, g, beta, st


def unit(x):
    n = np.linalg.norm(x, axis=-1, keepdims=True)
    return np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)


def as_generalized(q, k, v, g, beta):
    """The generalized delta rule inputs that give Gated DeltaNet: r = qh, w = g on
    every channel, write key beta kh, read vector a = kh, b = -exp(g) beta kh, so that
    diag(exp w) + b a^T = exp(g) (I - beta kh kh^T)."""
    qh, kh = unit(q), unit(k)
    K = q.shape[-1]
    w = np.repeat(g[..., None], K, axis=-1)
    return qh, w, beta[..., None] * kh, v, kh, -np.exp(g)[..., None] * beta[..., None] * kh


# --- hand-worked golden ---------------------------------------------------------

@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_worked_golden(case):
    K, V = case["K"], case["V"]
    vec = lambda x: np.array(x, dtype=np.float64)[None, :, None, :]
    sca = lambda x: np.array(x, dtype=np.float64)[None, :, None]
    o, sT, _ = oracle.gdn_fwd(vec(case["q"]), vec(case["k"]), vec(case["v"]), sca(case["g"]),
                              sca(case["beta"]),
                              s0=np.array(case["s0"], dtype=np.float64).reshape(1, 1, K, V))
    np.testing.assert_allclose(o[0, :, 0], np.array(case["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(sT[0, 0], np.array(case["sT"]), rtol=0, atol=1e-12)


# --- independent forms ----------------------------------------------------------

@pytest.mark.parametrize("K,V,T,seed", [(2, 2, 5, 0), (3, 2, 8, 1), (4, 4, 7, 2), (5, 3, 6, 3)])
def test_matches_dense_products(K, V, T, seed):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, s0 = rand_gdn(rng, 2, T, 2, K, V)
    o, sT, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s0)
    ob, sb = brute.gdn_fwd(q, k, v, g, beta, s0=s0)
    np.testing.assert_allclose(o, ob, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(sT, sb, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("T,K,V,seed", [(1, 4, 4, 0), (37, 8, 5, 1), (130, 64, 64, 2)])
def test_equals_generalized_rule_substitution(T, K, V, seed):
    """Two separately written oracles agree: Gated DeltaNet is the generalized delta
    rule with a scalar decay, a = kh, b = -exp(g) beta kh and write key beta kh."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, s0 = rand_gdn(rng, 2, T, 3, K, V)
    o, sT, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s0)
    og, sg, _ = oracle.fwd(*as_generalized(q, k, v, g, beta), s0=s0)
    np.testing.assert_allclose(o, og, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(sT, sg, rtol=1e-10, atol=1e-10)


# --- closed forms and special cases ----------------------------------------------

@pytest.mark.parametrize("T,K,V", [(1, 4, 4), (40, 8, 5)])
def test_closed_form_no_writes(T, K, V):
    """beta = 0: nothing is written or erased, the state only decays:
    S_t = exp(sum_{j<=t} g_j) S_0 and o_t = S_t^T qh_t."""
    rng = np.random.default_rng(7)
    q, k, v, g, beta, s0 = rand_gdn(rng, 1, T, 2, K, V)
    beta[:] = 0.0
    o, sT, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s0)
    G = np.cumsum(g, axis=1)  # [1,T,H]
    qh = unit(q)
    want = np.exp(G)[..., None] * np.einsum("bhkv,bthk->bthv", s0, qh)
    np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sT, np.exp(G[:, -1])[..., None, None] * s0, rtol=1e-12)


def test_single_write_from_zero():
    """One token from a zero state: S_1 = beta kh v^T, o_1 = beta (kh . qh) v."""
    rng = np.random.default_rng(8)
    q, k, v, g, beta, _ = rand_gdn(rng, 3, 1, 2, 6, 5, s0=False)
    o, sT, _ = oracle.gdn_fwd(q, k, v, g, beta)
    qh, kh = unit(q), unit(k)
    dot = np.sum(qh * kh, axis=-1)  # [B,1,H]
    np.testing.assert_allclose(o, (beta * dot)[..., None] * v, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sT, beta[:, 0, :, None, None] * np.einsum(
        "bhk,bhv->bhkv", kh[:, 0], v[:, 0]), rtol=1e-12, atol=1e-12)


def test_delta_rule_projection():
    """beta = 1: after each token the state maps its own key onto its value,
    S_t^T kh_t = v_t, whatever the gate; with q = c k (c > 0) the output is v_t."""
    rng = np.random.default_rng(9)
    q, k, v, g, beta, s0 = rand_gdn(rng, 2, 33, 2, 8, 6)
    beta[:] = 1.0
    q = 2.5 * k
    o, _, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s0)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


def test_normalisation_inside():
    """q and k are L2-normalised inside: positive per-token rescaling of q and k
    changes nothing; a zero key neither writes nor erases."""
    rng = np.random.default_rng(10)
    q, k, v, g, beta, s0 = rand_gdn(rng, 2, 20, 2, 8, 8)
    o, sT, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s0)
    cq = rng.uniform(0.1, 10.0, size=q.shape[:-1] + (1,))
    ck = rng.uniform(0.1, 10.0, size=k.shape[:-1] + (1,))
    o2, sT2, _ = oracle.gdn_fwd(q * cq, k * ck, v, g, beta, s0=s0)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sT2, sT, rtol=1e-12, atol=1e-12)
    k0 = np.zeros_like(k)
    _, sT0, _ = oracle.gdn_fwd(q, k0, v, g, beta, s0=s0)
    np.testing.assert_allclose(sT0, np.exp(g.sum(axis=1))[..., None, None] * s0, rtol=1e-12)


@pytest.mark.parametrize("split", [1, 17, 63, 64, 65, 100])
def test_state_passing(split):
    rng = np.random.default_rng(11)
    q, k, v, g, beta, s0 = rand_gdn(rng, 1, 150, 2, 8, 8)
    o, sT, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s0)
    cut = lambda x, a, b: x[:, a:b]
    o1, s1, _ = oracle.gdn_fwd(*(cut(x, 0, split) for x in (q, k, v, g, beta)), s0=s0)
    o2, s2, _ = oracle.gdn_fwd(*(cut(x, split, 150) for x in (q, k, v, g, beta)), s0=s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s2, sT, rtol=1e-12, atol=1e-12)


def test_varlen_and_shared_initial_state():
    """Packed sequences equal separate runs; a [1,H,K,V] initial state is shared by
    every sequence (README: initial_state (B,H,K,V) or (1,H,K,V))."""
    rng = np.random.default_rng(12)
    lens = [5, 1, 70, 0, 33]
    T = sum(lens)
    q, k, v, g, beta, _ = rand_gdn(rng, 1, T, 2, 8, 4, s0=False)
    s_shared = rng.standard_normal((1, 2, 8, 4))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, sT, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s_shared, cu_seqlens=cu)
    for n, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        on, sn, _ = oracle.gdn_fwd(*(x[:, a:b] for x in (q, k, v, g, beta)), s0=s_shared)
        np.testing.assert_allclose(o[:, a:b], on, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(sT[n], sn[0], rtol=1e-12, atol=1e-12)
    # batched form with a shared state equals the explicitly repeated state
    qb, kb, vb, gb, bb, _ = rand_gdn(rng, 3, 9, 2, 8, 4, s0=False)
    o1, s1, _ = oracle.gdn_fwd(qb, kb, vb, gb, bb, s0=s_shared)
    o2, s2, _ = oracle.gdn_fwd(qb, kb, vb, gb, bb, s0=np.repeat(s_shared, 3, axis=0))
    np.testing.assert_allclose(o1, o2, rtol=0, atol=0)
    np.testing.assert_allclose(s1, s2, rtol=0, atol=0)


def test_step_equals_forward():
    rng = np.random.default_rng(13)
    q, k, v, g, beta, s0 = rand_gdn(rng, 2, 6, 2, 8, 8)
    o, sT, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s0)
    state = s0
    for t in range(6):
        ot, state = oracle.gdn_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], state)
        np.testing.assert_allclose(ot, o[:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(state, sT, rtol=1e-12, atol=1e-12)


def test_contraction_on_workload_inputs():
    """With beta in (0,1) and g < 0 every transition has spectral norm <= 1, so
    |S_t|_F <= |S_0|_F + sum_s beta_s |v_s| (the write beta kh v^T has norm beta |v|)."""
    x = synth.gdn_inputs(1, 256, 4, dtype=torch.float32, seed=5, s0_std=0.1)
    o, sT, _ = oracle.gdn_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], s0=x["s0"])
    bound = (np.linalg.norm(x["s0"].double().numpy(), axis=(-2, -1)) +
             (x["beta"].double()[..., None] * x["v"].double()).norm(dim=-1).sum(dim=1).numpy())
    assert np.all(np.linalg.norm(sT, axis=(-2, -1)) <= bound[0] + 1e-9)


def test_synth_recipe():
    x = synth.gdn_inputs(2, 64, 3, dtype=torch.float32, seed=5, s0_std=0.1)
    g, beta = x["g"], x["beta"]
    assert g.shape == (2, 64, 3) and beta.shape == (2, 64, 3)
    assert float(g.max()) < 0 and float(g.min()) > -np.exp(-0.5) - 1e-6
    assert float(beta.min()) > 0 and float(beta.max()) < 1
    y = synth.gdn_inputs(2, 64, 3, dtype=torch.float32, seed=5, s0_std=0.1)
    torch.testing.assert_close(x["q"], y["q"], rtol=0, atol=0)


# --- the pins catch plausible mistakes in the oracle -----------------------------

GDN_MUTANTS = {
    "gate_dropped": ("for (size_t i = 0; i < (size_t)K * V; ++i) S[i] *= alpha;", ""),
    "gate_not_log_space": ("const double alpha = exp(g[tok]);", "const double alpha = g[tok];"),
    "gate_after_write": ("        for (size_t i = 0; i < (size_t)K * V; ++i) S[i] *= alpha;\n", ""),
    "q_not_normalised": ("unit_normalise(q + tok * K, qh, K);",
                         "for (int i = 0; i < K; ++i) qh[i] = q[tok * K + i];"),
    "k_not_normalised": ("unit_normalise(k + tok * K, kh, K);",
                         "for (int i = 0; i < K; ++i) kh[i] = k[tok * K + i];"),
    "beta_dropped": ("S[(size_t)i * V + j] += bt * kh[i] * e[j];",
                     "S[(size_t)i * V + j] += kh[i] * e[j];"),
    "error_sign": ("e[j] = v[tok * V + j] - pred;", "e[j] = v[tok * V + j] + pred;"),
    "write_transposed": ("S[(size_t)i * V + j] += bt * kh[i] * e[j];",
                         "S[(size_t)i * V + j] += bt * kh[j] * e[i];"),
    "every_sequence_from_state_0": ("(s0_shared ? 0 : n)", "(s0_shared ? 0 : 0)"),
}


def _gdn_mutant(tmp_path, name):
    old, new = GDN_MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, name
    if name == "gate_after_write":
        # decay after the delta write instead of before it
        src = src.replace(old, new)
        src = src.replace("        for (int j = 0; j < V; ++j) {\n            double acc = 0.0;\n"
                          "            for (int i = 0; i < K; ++i) acc += S[(size_t)i * V + j] * qh[i];",
                          "        for (size_t i = 0; i < (size_t)K * V; ++i) S[i] *= alpha;\n"
                          "        for (int j = 0; j < V; ++j) {\n            double acc = 0.0;\n"
                          "            for (int i = 0; i < K; ++i) acc += S[(size_t)i * V + j] * qh[i];", 1)
    else:
        src = src.replace(old, new)
    c = tmp_path / f"gdn_{name}.c"
    so = tmp_path / f"gdn_{name}.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-fPIC", "-shared", "-o", str(so), str(c),
                           "-lm"])
    return oracle.load_library(str(so))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(GDN_MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    lib = _gdn_mutant(tmp_path, name)
    failures = 0
    case = json.load(open(GOLDEN))["cases"][0]
    vec = lambda x: np.array(x, dtype=np.float64)[None, :, None, :]
    sca = lambda x: np.array(x, dtype=np.float64)[None, :, None]
    o, sT, _ = oracle.gdn_fwd(vec(case["q"]), vec(case["k"]), vec(case["v"]), sca(case["g"]),
                              sca(case["beta"]), s0=np.array(case["s0"]).reshape(1, 1, 2, 2),
                              library=lib)
    failures += not (np.allclose(o[0, :, 0], case["o"], atol=1e-9) and
                     np.allclose(sT[0, 0], case["sT"], atol=1e-9))
    rng = np.random.default_rng(14)
    q, k, v, g, beta, s0 = rand_gdn(rng, 2, 6, 1, 3, 3)
    o, sT, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s0, library=lib)
    ob, sb = brute.gdn_fwd(q, k, v, g, beta, s0=s0)
    failures += not (np.allclose(o, ob, atol=1e-9) and np.allclose(sT, sb, atol=1e-9))
    # a shared initial state must equal the repeated one
    s1 = rng.standard_normal((1, 1, 3, 3))
    o1, _, _ = oracle.gdn_fwd(q, k, v, g, beta, s0=s1, library=lib)
    ob1, _ = brute.gdn_fwd(q, k, v, g, beta, s0=np.repeat(s1, 2, axis=0))
    failures += not np.allclose(o1, ob1, atol=1e-9)
    assert failures > 0, f"mutant {name} passed every pin"


# --- the Gated DeltaNet backward --------------------------------------------------

def _gdn_loss(x, dout, dsT):
    o, sT, _ = oracle.gdn_fwd(*(x[n] for n in ("q", "k", "v", "g", "beta")), s0=x["s0"])
    return float(np.sum(o * dout) + np.sum(sT * dsT))


@pytest.mark.parametrize("seed,shared", [(20, False), (21, True)])
def test_gdn_bwd_matches_finite_differences(seed, shared):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, _ = rand_gdn(rng, 2, 6, 1, 3, 2, s0=False)
    s0 = rng.standard_normal((1 if shared else 2, 1, 3, 2))
    x = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "s0": s0}
    dout = rng.standard_normal(v.shape)
    dsT = rng.standard_normal((2, 1, 3, 2))
    gr = oracle.gdn_bwd(q, k, v, g, beta, dout, s0=s0, dsT=dsT)
    eps = 1e-6
    for n in ("q", "k", "v", "g", "beta", "s0"):
        fd = np.zeros_like(x[n])
        for idx in np.ndindex(x[n].shape):
            keep = x[n][idx]
            x[n][idx] = keep + eps
            lp = _gdn_loss(x, dout, dsT)
            x[n][idx] = keep - eps
            lm = _gdn_loss(x, dout, dsT)
            x[n][idx] = keep
            fd[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(gr["d" + n], fd, rtol=1e-6, atol=1e-7, err_msg=n)
