"""Pins for the fp64 CPU oracle (no GPU).  Each test checks the oracle against
something other than itself: hand-worked values, an independent dense-product
form, closed forms, invariants and a textbook special case.

The recurrence being pinned is the generalized delta rule behind
generalized_delta_rule(r, w, k, v, a, b, initial_state, output_final_state,
head_first, mask) (rwkv-ops 0.9.0 README, "rwkv7op 使用方法"): per head a K x V
state, log-space decay w, mask[B,T] with 1 = update and 0 = keep, initial and
final states [N, H, K, V], and its length-one decode form rwkv7_op_rnn
(same README, "rwkv7_op_rnn 使用方法").
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

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def rand_inputs(rng, B, T, H, K, V, w_scale=1.0, s0=True, symmetric=False):
    r = rng.standard_normal((B, T, H, K))
    k = rng.standard_normal((B, T, H, K))
    v = rng.standard_normal((B, T, H, V))
    w = -w_scale * rng.random((B, T, H, K))
    if symmetric:
        kh = k / np.linalg.norm(k, axis=-1, keepdims=True)
        a, b = -kh, kh * rng.random((B, T, H, 1))
    else:
        a = 0.5 * rng.standard_normal((B, T, H, K))
        b = 0.5 * rng.standard_normal((B, T, H, K))
    st = rng.standard_normal((B, H, K, V)) if s0 else None
    return r, w, k, v, a, b, st


# --- hand-worked goldens -------------------------------------------------------

@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_worked_golden(case):
    K, V = case["K"], case["V"]
    arr = lambda x: np.array(x, dtype=np.float64)[None, :, None, :]  # [1,T,1,*]
    mask = None if case["mask"] is None else np.array(case["mask"], dtype=np.uint8)[None]
    o, sT, _ = oracle.fwd(arr(case["r"]), arr(case["w"]), arr(case["k"]), arr(case["v"]),
                          arr(case["a"]), arr(case["b"]),
                          s0=np.array(case["s0"], dtype=np.float64).reshape(1, 1, K, V),
                          mask=mask)
    np.testing.assert_allclose(o[0, :, 0], np.array(case["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(sT[0, 0], np.array(case["sT"]), rtol=0, atol=1e-12)


# --- P1: brute-force dense transition products --------------------------------

@pytest.mark.parametrize("K,V,T,seed", [(2, 2, 5, 0), (3, 2, 8, 1), (4, 4, 7, 2),
                                        (2, 3, 1, 3), (4, 3, 8, 4)])
def test_matches_dense_products(K, V, T, seed):
    rng = np.random.default_rng(seed)
    r, w, k, v, a, b, s0 = rand_inputs(rng, 2, T, 2, K, V)
    o, sT, _ = oracle.fwd(r, w, k, v, a, b, s0=s0)
    ob, sb = brute.fwd(r, w, k, v, a, b, s0=s0)
    np.testing.assert_allclose(o, ob, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(sT, sb, rtol=1e-10, atol=1e-12)


def test_matches_dense_products_with_mask():
    rng = np.random.default_rng(11)
    r, w, k, v, a, b, s0 = rand_inputs(rng, 2, 8, 1, 3, 3)
    mask = (rng.random((2, 8)) > 0.4).astype(np.uint8)
    o, sT, _ = oracle.fwd(r, w, k, v, a, b, s0=s0, mask=mask)
    ob, sb = brute.fwd(r, w, k, v, a, b, s0=s0, mask=mask)
    np.testing.assert_allclose(o, ob, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(sT, sb, rtol=1e-10, atol=1e-12)


# --- P2 / P3: closed forms with a = b = 0 -------------------------------------

@pytest.mark.parametrize("T,K,V", [(1, 4, 4), (37, 8, 5), (130, 64, 64)])
def test_closed_form_cumulative_linear_attention(T, K, V):
    """a = b = 0, w = 0: o_t = S0^T r_t + sum_{s<=t} (r_t . k_s) v_s."""
    rng = np.random.default_rng(T)
    r, _, k, v, _, _, s0 = rand_inputs(rng, 1, T, 1, K, V)
    z = np.zeros_like(r)
    o, sT, _ = oracle.fwd(r, z, k, v, z, z, s0=s0)
    R, Kk, Vv, S0 = r[0, :, 0], k[0, :, 0], v[0, :, 0], s0[0, 0]
    expect = R @ S0 + np.tril(R @ Kk.T) @ Vv
    np.testing.assert_allclose(o[0, :, 0], expect, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(sT[0, 0], S0 + Kk.T @ Vv, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("T,K,V", [(9, 4, 3), (64, 16, 8)])
def test_closed_form_gated_linear_attention(T, K, V):
    """a = b = 0, w != 0: with G_t = sum_{j<=t} w_j (log space),
    o_t = S0^T (r_t * e^{G_t}) + sum_{s<=t} (r_t * e^{G_t - G_s} . k_s) v_s."""
    rng = np.random.default_rng(100 + T)
    r, w, k, v, _, _, s0 = rand_inputs(rng, 1, T, 1, K, V, w_scale=0.7)
    z = np.zeros_like(r)
    o, sT, _ = oracle.fwd(r, w, k, v, z, z, s0=s0)
    R, W, Kk, Vv, S0 = r[0, :, 0], w[0, :, 0], k[0, :, 0], v[0, :, 0], s0[0, 0]
    G = np.cumsum(W, axis=0)
    expect = np.zeros((T, V))
    for t in range(T):
        expect[t] = (R[t] * np.exp(G[t])) @ S0
        for s in range(t + 1):
            expect[t] += np.dot(R[t] * np.exp(G[t] - G[s]), Kk[s]) * Vv[s]
    np.testing.assert_allclose(o[0, :, 0], expect, rtol=1e-10, atol=1e-10)
    expect_S = np.exp(G[-1])[:, None] * S0 + sum(
        np.outer(Kk[s] * np.exp(G[-1] - G[s]), Vv[s]) for s in range(T))
    np.testing.assert_allclose(sT[0, 0], expect_S, rtol=1e-10, atol=1e-10)


# --- P4: state passing (checkpoint / resume) ----------------------------------

@pytest.mark.parametrize("split", [1, 17, 63, 64, 65, 100])
def test_state_passing(split):
    rng = np.random.default_rng(7)
    r, w, k, v, a, b, s0 = rand_inputs(rng, 2, 129, 3, 8, 8, symmetric=True)
    o, sT, _ = oracle.fwd(r, w, k, v, a, b, s0=s0)
    cut = lambda x, sl: x[:, sl]
    o1, s1, _ = oracle.fwd(*(cut(x, slice(0, split)) for x in (r, w, k, v, a, b)), s0=s0)
    o2, s2, _ = oracle.fwd(*(cut(x, slice(split, None)) for x in (r, w, k, v, a, b)), s0=s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s2, sT, rtol=1e-12, atol=1e-12)


def test_decode_steps_equal_forward():
    """T single-token steps (rwkv7_op_rnn) == one forward over the T tokens."""
    rng = np.random.default_rng(8)
    r, w, k, v, a, b, s0 = rand_inputs(rng, 3, 12, 2, 8, 8, symmetric=True)
    o, sT, _ = oracle.fwd(r, w, k, v, a, b, s0=s0)
    state = s0
    for t in range(12):
        ot, state = oracle.step(r[:, t], w[:, t], k[:, t], v[:, t], a[:, t], b[:, t], state)
        np.testing.assert_allclose(ot, o[:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(state, sT, rtol=1e-12, atol=1e-12)


def test_varlen_equals_separate_sequences():
    rng = np.random.default_rng(9)
    lens = [5, 1, 64, 0, 23]
    total = sum(lens)
    r, w, k, v, a, b, _ = rand_inputs(rng, 1, total, 2, 4, 4, symmetric=True)
    s0 = rng.standard_normal((len(lens), 2, 4, 4))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, sT, _ = oracle.fwd(r, w, k, v, a, b, s0=s0, cu_seqlens=cu)
    for n, (lo, hi) in enumerate(zip(cu[:-1], cu[1:])):
        on, sn, _ = oracle.fwd(*(x[:, lo:hi] for x in (r, w, k, v, a, b)), s0=s0[n:n + 1])
        np.testing.assert_allclose(o[:, lo:hi], on, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(sT[n], sn[0], rtol=1e-12, atol=1e-12)


# --- P5: mask invariants -------------------------------------------------------

def test_mask_invariants():
    rng = np.random.default_rng(10)
    B, T, H, K = 2, 40, 2, 6
    r, w, k, v, a, b, s0 = rand_inputs(rng, B, T, H, K, K, symmetric=True)
    o_ref, s_ref, _ = oracle.fwd(r, w, k, v, a, b, s0=s0)
    # (i) all-ones mask == no mask
    o1, s1, _ = oracle.fwd(r, w, k, v, a, b, s0=s0, mask=np.ones((B, T), np.uint8))
    np.testing.assert_array_equal(o1, o_ref)
    np.testing.assert_array_equal(s1, s_ref)
    # (iv) all-zero mask: state unchanged, o_t = s0^T r_t
    o0, s0_out, _ = oracle.fwd(r, w, k, v, a, b, s0=s0, mask=np.zeros((B, T), np.uint8))
    np.testing.assert_array_equal(s0_out, s0)
    np.testing.assert_allclose(o0, np.einsum("bthk,bhkv->bthv", r, s0), rtol=1e-12, atol=1e-12)
    # (ii) masked tokens == deleted tokens for state and unmasked outputs;
    # (iii) at a masked step o_t = S_{t-1}^T r_t
    mask = (rng.random((B, T)) > 0.3).astype(np.uint8)
    om, sm, _ = oracle.fwd(r, w, k, v, a, b, s0=s0, mask=mask)
    for bb in range(B):
        keep = mask[bb].astype(bool)
        od, sd, _ = oracle.fwd(*(x[bb:bb + 1, keep] for x in (r, w, k, v, a, b)),
                               s0=s0[bb:bb + 1])
        np.testing.assert_allclose(om[bb, keep], od[0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(sm[bb], sd[0], rtol=1e-12, atol=1e-12)
        # state before each token = state after the kept prefix before it
        for t in np.nonzero(~keep)[0]:
            prefix = keep.copy()
            prefix[t:] = False
            _, sp, _ = oracle.fwd(*(x[bb:bb + 1, prefix] for x in (r, w, k, v, a, b)),
                                  s0=s0[bb:bb + 1])
            np.testing.assert_allclose(om[bb, t], np.einsum("hk,hkv->hv", r[bb, t], sp[0]),
                                       rtol=1e-12, atol=1e-12)


# --- P6: textbook delta rule ----------------------------------------------------

def test_delta_rule_overwrite():
    """w = 0, a = -k_hat, b = k_hat, key k_hat: S_t = (I - k k^T) S + k v^T, so
    S_t^T k_hat == v_t exactly (the classic delta-rule projection property)."""
    rng = np.random.default_rng(12)
    T, K, V = 10, 8, 5
    r, _, k, v, _, _, s0 = rand_inputs(rng, 1, T, 1, K, V)
    kh = k / np.linalg.norm(k, axis=-1, keepdims=True)
    z = np.zeros_like(r)
    for t in range(1, T + 1):
        _, sT, _ = oracle.fwd(r[:, :t], z[:, :t], kh[:, :t], v[:, :t], -kh[:, :t], kh[:, :t],
                              s0=s0)
        np.testing.assert_allclose(sT[0, 0].T @ kh[0, t - 1, 0], v[0, t - 1, 0],
                                   rtol=1e-12, atol=1e-12)


# --- P7: linearity in (v, s0) -------------------------------------------------

def test_linearity_in_values_and_state():
    rng = np.random.default_rng(13)
    r, w, k, v1, a, b, s1 = rand_inputs(rng, 1, 50, 2, 8, 8)
    v2 = rng.standard_normal(v1.shape)
    s2 = rng.standard_normal(s1.shape)
    al, be = 0.7, -1.9
    oa, sa, _ = oracle.fwd(r, w, k, v1, a, b, s0=s1)
    ob, sb, _ = oracle.fwd(r, w, k, v2, a, b, s0=s2)
    oc, sc, _ = oracle.fwd(r, w, k, al * v1 + be * v2, a, b, s0=al * s1 + be * s2)
    np.testing.assert_allclose(oc, al * oa + be * ob, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(sc, al * sa + be * sb, rtol=1e-9, atol=1e-9)


# --- P8: contraction bound on the workload distributions ------------------------

def test_contraction_bound_on_workload_inputs():
    """With a = -k_hat, b = eta k_hat (0 <= eta <= 1) and w < 0 the transition
    diag(e^w) - eta k_hat k_hat^T has spectral norm <= 1, so
    ||S_t||_F <= ||S_0||_F + sum_s ||k_s|| ||v_s||."""
    x = synth.fwd_inputs(2, 200, 3, 16, 16, dtype=torch.float32, seed=0, s0_std=0.1)
    o, sT, _ = oracle.fwd(x["r"], x["w"], x["k"], x["v"], x["a"], x["b"], s0=x["s0"])
    k, v, s0 = x["k"].double().numpy(), x["v"].double().numpy(), x["s0"].double().numpy()
    bound = (np.linalg.norm(s0, axis=(-2, -1)) +
             np.einsum("bth,bth->bh", np.linalg.norm(k, axis=-1), np.linalg.norm(v, axis=-1)))
    assert np.all(np.linalg.norm(sT, axis=(-2, -1)) <= bound * (1 + 1e-12))
    assert np.all(np.isfinite(o))


def test_synth_recipe():
    x = synth.fwd_inputs(1, 64, 2, dtype=torch.float32, seed=0, s0_std=0.0)
    k = x["k"].double()
    np.testing.assert_allclose(k.norm(dim=-1).numpy(), 1.0, rtol=1e-6)
    w = x["w"]
    assert float(w.max()) < 0 and float(w.min()) > -np.exp(-0.5) - 1e-6
    torch.testing.assert_close(x["a"], -x["k"])
    eta = (x["b"] / x["k"]).nan_to_num(0.5)
    assert float(eta.min()) >= 0 and float(eta.max()) <= 1
    y = synth.fwd_inputs(1, 64, 2, dtype=torch.float32, seed=0, s0_std=0.0)
    torch.testing.assert_close(x["r"], y["r"], rtol=0, atol=0)
    m = synth.padding_mask(4, 256, seed=2, max_suffix=64)
    assert m.dtype == torch.uint8 and m.shape == (4, 256)
    lens = synth.varlen_lengths(64, 16, 8192, seed=3)
    assert int(lens.min()) >= 16 and int(lens.max()) <= 8192


# --- the pins themselves catch plausible mistakes in the oracle ----------------

MUTANTS = {
    "decay_dropped": ("*s = di * (*s) + bi * u[j] + ki * v[rowV + j];",
                      "*s = (*s) + bi * u[j] + ki * v[rowV + j];"),
    "decay_not_log_space": ("const double di = exp(w[rowK + i]);",
                            "const double di = w[rowK + i];"),
    "rank1_sign_flipped": ("*s = di * (*s) + bi * u[j] + ki * v[rowV + j];",
                           "*s = di * (*s) - bi * u[j] + ki * v[rowV + j];"),
    "a_b_roles_swapped": ("const double ai = a[rowK + i];", "const double ai = b[rowK + i];"),
    "write_transposed": ("ki * v[rowV + j]", "k[rowK + j] * v[rowV + i]"),
    "output_before_update": ("        /* o = S^T r */", "        continue; /* o = S^T r */"),
    "mask_ignored": ("mask ? (mask[(size_t)bb * T + t] != 0) : 1", "1"),
}


def _mutant_results(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, name
    if name == "output_before_update":
        # compute o before the update instead of after it
        src = src.replace("        if (update) {", "        for (int j = 0; j < V; ++j) {"
                          " double acc = 0.0; for (int i = 0; i < K; ++i) acc += "
                          "S[(size_t)i * V + j] * r[rowK + i]; o[rowV + j] = acc; }\n"
                          "        if (update) {", 1)
        src = src.replace("        /* o = S^T r */\n        for (int j = 0; j < V; ++j) {",
                          "        for (int j = 0; j < 0; ++j) {", 1)
    else:
        src = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-fPIC", "-shared", "-o", str(so), str(c),
                           "-lm"])
    return oracle.load_library(str(so))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    lib = _mutant_results(tmp_path, name)
    failures = 0
    # hand-worked goldens
    for case in json.load(open(GOLDEN))["cases"]:
        K, V = case["K"], case["V"]
        arr = lambda x: np.array(x, dtype=np.float64)[None, :, None, :]
        mask = None if case["mask"] is None else np.array(case["mask"], np.uint8)[None]
        o, sT, _ = oracle.fwd(arr(case["r"]), arr(case["w"]), arr(case["k"]), arr(case["v"]),
                              arr(case["a"]), arr(case["b"]),
                              s0=np.array(case["s0"], np.float64).reshape(1, 1, K, V),
                              mask=mask, library=lib)
        failures += not (np.allclose(o[0, :, 0], case["o"], atol=1e-9) and
                         np.allclose(sT[0, 0], case["sT"], atol=1e-9))
    # dense products (asymmetric a, b)
    rng = np.random.default_rng(5)
    r, w, k, v, a, b, s0 = rand_inputs(rng, 1, 6, 1, 3, 3)
    mask = np.array([[1, 0, 1, 1, 0, 1]], np.uint8)
    o, sT, _ = oracle.fwd(r, w, k, v, a, b, s0=s0, mask=mask, library=lib)
    ob, sb = brute.fwd(r, w, k, v, a, b, s0=s0, mask=mask)
    failures += not (np.allclose(o, ob, atol=1e-9) and np.allclose(sT, sb, atol=1e-9))
    assert failures > 0, f"mutant {name} passed every pin"
