"""Pins for the SANE oracle (no GPU).  The README (rwkv-ops 0.9.0, "rwkv7op_sane 使用方法"
and "rwkv7_op_sane_rnn 使用方法") fixes where and when the state is soft-clipped (after
every 16th token, per-chunk tau > 0, a per-chunk flag, outputs read before the clip)
but defers the clip function to an external paper.  The tests pin that structure
against the generalized-rule oracle; the clip function itself (the reading
tau * tanh(S / tau)) is parity unpinned."""
import numpy as np
import pytest

import oracle

NAMES = ("r", "w", "k", "v", "a", "b")


def problem(rng, B=2, T=40, H=2, K=4, V=3, scale=1.0):
    x = {n: scale * rng.standard_normal((B, T, H, V if n == "v" else K)) for n in NAMES}
    x["w"] = -rng.random((B, T, H, K))
    x["a"] *= 0.5
    x["b"] *= 0.5
    s0 = rng.standard_normal((B, H, K, V))
    tau = 1.0 + rng.random((B, T // 16, H))
    return x, s0, tau


def test_huge_tau_or_no_chunk_is_the_plain_rule():
    rng = np.random.default_rng(0)
    x, s0, tau = problem(rng)
    o, sT, _ = oracle.fwd(*(x[n] for n in NAMES), s0=s0)
    o1, s1 = oracle.sane_fwd(*(x[n] for n in NAMES), np.full_like(tau, 1e30), s0=s0)
    np.testing.assert_allclose(o1, o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s1, sT, rtol=1e-12, atol=1e-12)
    o2, s2 = oracle.sane_fwd(*(x[n] for n in NAMES), tau, sane_mask=np.zeros(tau.shape[:2]),
                             s0=s0)
    np.testing.assert_array_equal(o2, o)
    np.testing.assert_array_equal(s2, sT)
    short = {n: x[n][:, :15] for n in NAMES}  # no full chunk: never clipped
    o3, s3 = oracle.sane_fwd(*(short[n] for n in NAMES), tau[:, :0], s0=s0)
    o4, s4, _ = oracle.fwd(*(short[n] for n in NAMES), s0=s0)
    np.testing.assert_array_equal(o3, o4)
    np.testing.assert_array_equal(s3, s4)


def test_clip_happens_after_the_boundary_token_only():
    """Tokens 0..15 give the plain outputs (token 15's output is read before the clip);
    token 16 on differ when the clip is active (large state, small tau)."""
    rng = np.random.default_rng(1)
    x, s0, tau = problem(rng, scale=3.0)
    tau[:] = 1.0
    o, _, _ = oracle.fwd(*(x[n] for n in NAMES), s0=s0)
    o1, _ = oracle.sane_fwd(*(x[n] for n in NAMES), tau, s0=s0)
    np.testing.assert_array_equal(o1[:, :16], o[:, :16])
    assert np.abs(o1[:, 16:] - o[:, 16:]).max() > 1e-3


@pytest.mark.parametrize("split", [16, 32])
def test_state_passing_at_chunk_boundaries(split):
    """Running [0, split) then [split, T) from its final state (with the matching tau
    rows) equals one run: the clip belongs to the chunk that ends at the boundary."""
    rng = np.random.default_rng(2)
    x, s0, tau = problem(rng, T=48, scale=2.0)
    mask = np.array([[1, 0, 1], [1, 1, 0]])
    o, sT = oracle.sane_fwd(*(x[n] for n in NAMES), tau, sane_mask=mask, s0=s0)
    c = split // 16
    o1, s1 = oracle.sane_fwd(*(x[n][:, :split] for n in NAMES), tau[:, :c],
                             sane_mask=mask[:, :c], s0=s0)
    o2, s2 = oracle.sane_fwd(*(x[n][:, split:] for n in NAMES), tau[:, c:],
                             sane_mask=mask[:, c:], s0=s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s2, sT, rtol=1e-12, atol=1e-12)


def test_step_form_every_sixteenth_token():
    """The README's single-step loop (do_sane at step % 16 == 15, outputs before the
    clip) reproduces the forward: plain steps from the generalized-rule oracle, the
    clip applied to the carried state at the flagged steps."""
    rng = np.random.default_rng(3)
    x, s0, tau = problem(rng, T=32, scale=2.0)
    o, sT = oracle.sane_fwd(*(x[n] for n in NAMES), tau, s0=s0)
    state = s0.copy()
    for t in range(32):
        ot, state = oracle.step(*(x[n][:, t] for n in NAMES), state)
        np.testing.assert_allclose(ot, o[:, t], rtol=1e-12, atol=1e-12)
        if t % 16 == 15:
            tc = tau[:, t // 16][:, :, None, None]
            state = tc * np.tanh(state / tc)
    np.testing.assert_allclose(state, sT, rtol=1e-12, atol=1e-12)


def test_clip_bounds_the_state():
    """After a clipped boundary every state entry lies within [-tau, tau] (tanh rounds to
    1 for very large entries)."""
    rng = np.random.default_rng(4)
    x, s0, tau = problem(rng, T=16, scale=10.0)
    _, sT = oracle.sane_fwd(*(x[n] for n in NAMES), tau, s0=s0 * 10)
    assert np.all(np.abs(sT) <= tau[:, 0][:, :, None, None])
    assert np.abs(sT).max() > 0.5 * tau.min()


def test_sane_step_matches_the_forward():
    """oracle.sane_step (NumPy, per step) driven as the README's loop (do_sane at step %
    16 == 15, per-row flags) equals the C SANE forward on the same tokens."""
    rng = np.random.default_rng(5)
    x, s0, tau = problem(rng, B=3, T=48, scale=2.0)
    mask = np.array([[1, 1, 0], [0, 1, 1], [1, 0, 1]])
    o, sT = oracle.sane_fwd(*(x[n] for n in NAMES), tau, sane_mask=mask, s0=s0)
    state = s0.copy()
    for t in range(48):
        c = t // 16
        flags = mask[:, c] if t % 16 == 15 else np.zeros(3)
        ot, state = oracle.sane_step(*(x[n][:, t] for n in NAMES), tau[:, c], flags, state)
        np.testing.assert_allclose(ot, o[:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(state, sT, rtol=1e-12, atol=1e-12)
