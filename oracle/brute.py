"""Dense transition-product form of the WKV7 recurrence (tiny sizes only).

TEST INFRASTRUCTURE ONLY: used by the tests to pin the C oracle.  It writes the
same definition differently from ``wkv7_oracle.c``: instead of stepping a
read vector u_t through the state, it builds each token's dense K x K
transition matrix

    M_t = diag(exp(w_t)) + b_t a_t^T

(rwkv-ops 0.9.0 README, "rwkv7op 使用方法": a and b are the two rank-1 factors,
gk / w the log-space decay) and unrolls the recurrence S_t = M_t S_{t-1} + k_t v_t^T
into explicit matrix products:

    S_t = (M_t ... M_1) S_0 + sum_{s<=t} (M_t ... M_{s+1}) k_s v_s^T
    o_t = S_t^T r_t

Masked tokens (mask 0) contribute the identity transition and no write.  Cost is
O(T^2 K^3) per head, so keep K and T small.
"""
from __future__ import annotations

import numpy as np


def fwd_unit(r, w, k, v, a, b, s0, mask=None):
    """One (sequence, head): r,w,k,a,b [T,K]; v [T,V]; s0 [K,V]; mask [T] or None."""
    r, w, k, v, a, b, s0 = (np.asarray(x, dtype=np.float64) for x in (r, w, k, v, a, b, s0))
    T, K = r.shape
    V = v.shape[1]
    eye = np.eye(K)
    trans = []
    writes = []
    for t in range(T):
        if mask is not None and not mask[t]:
            trans.append(eye.copy())
            writes.append(np.zeros((K, V)))
        else:
            trans.append(np.diag(np.exp(w[t])) + np.outer(b[t], a[t]))
            writes.append(np.outer(k[t], v[t]))
    o = np.zeros((T, V))
    S_t = s0
    for t in range(T):
        # P(t, s) = M_t M_{t-1} ... M_{s+1}  (empty product = I)
        acc = np.zeros((K, V))
        prod = eye.copy()
        for s in range(t, -1, -1):
            acc = acc + prod @ writes[s]
            prod = prod @ trans[s]
        S_t = prod @ s0 + acc
        o[t] = S_t.T @ r[t]
    return o, S_t


def fwd(r, w, k, v, a, b, s0=None, mask=None):
    """Batched [B,T,H,K] inputs (no varlen).  Returns (o [B,T,H,V], sT [B,H,K,V])."""
    r = np.asarray(r, dtype=np.float64)
    B, T, H, K = r.shape
    V = np.asarray(v).shape[-1]
    o = np.zeros((B, T, H, V))
    sT = np.zeros((B, H, K, V))
    for bb in range(B):
        for h in range(H):
            init = np.zeros((K, V)) if s0 is None else np.asarray(s0, dtype=np.float64)[bb, h]
            m = None if mask is None else np.asarray(mask)[bb]
            o[bb, :, h], sT[bb, h] = fwd_unit(
                r[bb, :, h], np.asarray(w)[bb, :, h], np.asarray(k)[bb, :, h],
                np.asarray(v)[bb, :, h], np.asarray(a)[bb, :, h], np.asarray(b)[bb, :, h],
                init, m)
    return o, sT


def gdn_fwd_unit(q, k, v, g, beta, s0):
    """Gated DeltaNet, one (sequence, head), as dense products: q, k [T,K], v [T,V],
    g, beta [T], s0 [K,V].  Each token's transition and write are built explicitly
    from the unit vectors kh = k / |k| (numpy.linalg.norm):

        M_t = exp(g_t) (I - beta_t kh_t kh_t^T),   W_t = beta_t kh_t v_t^T
        S_t = M_t S_{t-1} + W_t,                   o_t = S_t^T (q_t / |q_t|)

    (the Gated DeltaNet rule of rwkv-ops 0.9.0 README, "gdn_recurrent 使用方法",
    written as a product of transitions instead of a delta-rule update)."""
    q, k, v, s0 = (np.asarray(x, dtype=np.float64) for x in (q, k, v, s0))
    g, beta = np.asarray(g, dtype=np.float64), np.asarray(beta, dtype=np.float64)
    T, K = q.shape

    def unit(x):
        n = np.linalg.norm(x)
        return x / n if n > 0 else np.zeros_like(x)

    eye = np.eye(K)
    trans, writes = [], []
    for t in range(T):
        kh = unit(k[t])
        trans.append(np.exp(g[t]) * (eye - beta[t] * np.outer(kh, kh)))
        writes.append(beta[t] * np.outer(kh, v[t]))
    o = np.zeros((T, v.shape[1]))
    S_t = s0
    for t in range(T):
        acc = np.zeros_like(s0)
        prod = eye.copy()
        for s in range(t, -1, -1):
            acc = acc + prod @ writes[s]
            prod = prod @ trans[s]
        S_t = prod @ s0 + acc
        o[t] = S_t.T @ unit(q[t])
    return o, S_t


def gdn_fwd(q, k, v, g, beta, s0=None):
    """Batched Gated DeltaNet: q, k [B,T,H,K], v [B,T,H,V], g, beta [B,T,H];
    s0 [B,H,K,V] or None.  Returns (o [B,T,H,V], sT [B,H,K,V])."""
    q = np.asarray(q, dtype=np.float64)
    B, T, H, K = q.shape
    V = np.asarray(v).shape[-1]
    o = np.zeros((B, T, H, V))
    sT = np.zeros((B, H, K, V))
    for bb in range(B):
        for h in range(H):
            init = np.zeros((K, V)) if s0 is None else np.asarray(s0, dtype=np.float64)[bb, h]
            o[bb, :, h], sT[bb, h] = gdn_fwd_unit(
                q[bb, :, h], np.asarray(k)[bb, :, h], np.asarray(v)[bb, :, h],
                np.asarray(g)[bb, :, h], np.asarray(beta)[bb, :, h], init)
    return o, sT
