"""Pins for the backward oracle (no GPU): ``oracle.bwd`` against central finite
differences of ``oracle.fwd`` (an independent route to the same derivatives), a
closed form for the linear-attention special case, and planted mistakes.

The loss is L = sum(o * dout) + sum(S_T * dsT); the backward returns dL/dr, dw, dk,
dv, da, db and dL/ds0 of the generalized delta rule (rwkv-ops 0.9.0 README,
"rwkv7op 使用方法": the training entry supports backpropagation)."""
import shutil
import subprocess

import numpy as np
import pytest

import oracle

NAMES = ("r", "w", "k", "v", "a", "b")


def rand_problem(rng, B=1, T=5, H=1, K=3, V=3, mask=False):
    x = {n: rng.standard_normal((B, T, H, V if n == "v" else K)) for n in NAMES}
    x["w"] = -rng.random((B, T, H, K))
    x["a"] *= 0.5
    x["b"] *= 0.5
    x["s0"] = rng.standard_normal((B, H, K, V))
    dout = rng.standard_normal((B, T, H, V))
    dsT = rng.standard_normal((B, H, K, V))
    m = None
    if mask:
        m = (rng.random((B, T)) > 0.3).astype(np.uint8)
        m[:, 0] = 0
    return x, dout, dsT, m


def loss(x, dout, dsT, mask, library=None):
    o, sT, _ = oracle.fwd(*(x[n] for n in NAMES), s0=x["s0"], mask=mask, library=library)
    return float(np.sum(o * dout) + np.sum(sT * dsT))


def finite_difference(x, dout, dsT, mask, eps=1e-6):
    fd = {}
    for n in NAMES + ("s0",):
        g = np.zeros_like(x[n])
        for idx in np.ndindex(x[n].shape):
            keep = x[n][idx]
            x[n][idx] = keep + eps
            lp = loss(x, dout, dsT, mask)
            x[n][idx] = keep - eps
            lm = loss(x, dout, dsT, mask)
            x[n][idx] = keep
            g[idx] = (lp - lm) / (2 * eps)
        fd["d" + n] = g
    return fd


@pytest.mark.parametrize("seed,mask", [(0, False), (1, True), (2, False)])
def test_matches_finite_differences(seed, mask):
    rng = np.random.default_rng(seed)
    x, dout, dsT, m = rand_problem(rng, B=2, T=5, H=1, K=3, V=2, mask=mask)
    g = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], mask=m, dsT=dsT)
    fd = finite_difference(x, dout, dsT, m)
    for n in fd:
        np.testing.assert_allclose(g[n], fd[n], rtol=1e-6, atol=1e-7, err_msg=n)


def test_no_final_state_gradient_and_varlen():
    """dsT = None is a zero upstream state gradient; packed sequences equal separate
    runs, each with its own ds0."""
    rng = np.random.default_rng(3)
    x, dout, _, _ = rand_problem(rng, B=1, T=9, H=2, K=4, V=3)
    g0 = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"])
    g1 = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], dsT=np.zeros_like(x["s0"]))
    for n in g0:
        np.testing.assert_array_equal(g0[n], g1[n])
    cu = np.array([0, 4, 4, 9], dtype=np.int32)
    s0 = rng.standard_normal((3, 2, 4, 3))
    dsT = rng.standard_normal((3, 2, 4, 3))
    gv = oracle.bwd(*(x[n] for n in NAMES), dout, s0=s0, dsT=dsT, cu_seqlens=cu)
    for i, (lo, hi) in enumerate(zip(cu[:-1], cu[1:])):
        gi = oracle.bwd(*(x[n][:, lo:hi] for n in NAMES), dout[:, lo:hi], s0=s0[i:i + 1],
                        dsT=dsT[i:i + 1])
        for n in NAMES:
            np.testing.assert_allclose(gv["d" + n][:, lo:hi], gi["d" + n], rtol=1e-12,
                                       atol=1e-12)
        np.testing.assert_allclose(gv["ds0"][i], gi["ds0"][0], rtol=1e-12, atol=1e-12)


def test_closed_form_linear_attention():
    """a = b = 0, w = 0: o_t = S0^T r_t + sum_{s<=t} (r_t . k_s) v_s, so
    dr_t = S0 do_t + sum_{s<=t} (do_t . v_s) k_s, dk_s = sum_{t>=s} (do_t . v_s) r_t,
    dv_s = sum_{t>=s} (r_t . k_s) do_t, ds0 = sum_t r_t do_t^T, and da = db = 0."""
    rng = np.random.default_rng(4)
    T, K, V = 11, 5, 4
    r, k, v, do = (rng.standard_normal((T, K if n != "v" and n != "do" else V))
                   for n in ("r", "k", "v", "do"))
    s0 = rng.standard_normal((K, V))
    z = np.zeros((1, T, 1, K))
    g = oracle.bwd(r[None, :, None], z, k[None, :, None], v[None, :, None], z, z,
                   do[None, :, None], s0=s0[None, None])
    dr = np.stack([s0 @ do[t] + sum((do[t] @ v[s]) * k[s] for s in range(t + 1))
                   for t in range(T)])
    dk = np.stack([sum((do[t] @ v[s]) * r[t] for t in range(s, T)) for s in range(T)])
    dv = np.stack([sum((r[t] @ k[s]) * do[t] for t in range(s, T)) for s in range(T)])
    ds0 = sum(np.outer(r[t], do[t]) for t in range(T))
    np.testing.assert_allclose(g["dr"][0, :, 0], dr, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dk"][0, :, 0], dk, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dv"][0, :, 0], dv, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["ds0"][0, 0], ds0, rtol=1e-12, atol=1e-12)
    assert np.all(g["da"] == 0) and np.all(g["db"] == 0)


BWD_MUTANTS = {
    "dw_without_decay_factor": ("dw[rowK + i] = di * sw;", "dw[rowK + i] = sw;"),
    "adjoint_not_decayed": ("G[(size_t)i * V + j] = di * G[(size_t)i * V + j] + a[rowK + i] * du[j];",
                            "G[(size_t)i * V + j] = G[(size_t)i * V + j] + a[rowK + i] * du[j];"),
    "du_reads_a": ("sd += G[(size_t)i * V + j] * b[rowK + i];",
                   "sd += G[(size_t)i * V + j] * a[rowK + i];"),
    "da_uses_new_state": ("sa += Sp[(size_t)i * V + j] * du[j];",
                          "sa += St[(size_t)i * V + j] * du[j];"),
    "dr_uses_old_state": ("acc += St[(size_t)i * V + j] * dout[rowV + j];",
                          "acc += Sp[(size_t)i * V + j] * dout[rowV + j];"),
    "rank1_adjoint_dropped": ("G[(size_t)i * V + j] = di * G[(size_t)i * V + j] + a[rowK + i] * du[j];",
                              "G[(size_t)i * V + j] = di * G[(size_t)i * V + j];"),
}


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new = BWD_MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, name
    c = tmp_path / f"bwd_{name}.c"
    so = tmp_path / f"bwd_{name}.so"
    c.write_text(src.replace(old, new))
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-fPIC", "-shared", "-o", str(so), str(c),
                           "-lm"])
    lib = oracle.load_library(str(so))
    rng = np.random.default_rng(5)
    x, dout, dsT, m = rand_problem(rng, B=1, T=4, H=1, K=3, V=2)
    g = oracle.bwd(*(x[n] for n in NAMES), dout, s0=x["s0"], mask=m, dsT=dsT, library=lib)
    fd = finite_difference(x, dout, dsT, m)
    assert any(not np.allclose(g[n], fd[n], rtol=1e-5, atol=1e-6) for n in fd), \
        f"mutant {name} passed the finite-difference pin"
