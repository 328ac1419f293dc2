"""FP64 NumPy restatement of the chunkwise (WY / UT) evaluation order.

Test helper: it is neither the oracle nor the CUDA library.  It writes out,
in plain NumPy, the chunk algebra that the CUDA kernels implement, so a test
can check that algebra against the sequential oracle to ~1e-12 before any
kernel is trusted.  Nothing here is imported by the library or the oracle.

Per chunk of C tokens (chunk-local index i, state S entering the chunk):
  forward    g_i = sum_{m<=i} log a_m
             L_ij = b_i e^{g_i-g_j} (k_i.k_j)          j < i
             W = (I+L)^{-1} diag(b e^g) K,  U = (I+L)^{-1} diag(b) V
             D = U - W S
             O_i = e^{g_i} q_i^T S + sum_{j<=i} e^{g_i-g_j} (q_i.k_j) D_j
             S' = e^{g_last} S + sum_j e^{g_last-g_j} k_j D_j^T
  reverse    h_i = sum_{m>=i} log a_m  (h_C = 0), same chunk boundaries as
             the forward pass, chunks visited last to first
             L'_ij = b_i e^{h_i-h_j} (k_i.k_j)          j > i
             W' = (I+L')^{-1} diag(b e^h) K,  U' = (I+L')^{-1} diag(b) V
             D' = U' - W' R
             O'_i = e^{h_{i+1}} q_i^T R + sum_{j>i} e^{h_{i+1}-h_j} (q_i.k_j) D'_j
             R' = e^{h_0} R + sum_j e^{h_0-h_j} k_j D'_j^T
Padded tokens past the end of the sequence have a = 1, b = 0, k = q = v = 0,
which makes them identity steps in either direction.
"""
import numpy as np


def _pad(x, n):
    pad = [(0, 0)] * x.ndim
    pad[0] = (0, n - x.shape[0])
    return np.pad(x, pad)


def forward_one(q, k, v, a, b, S, C):
    """One sequence: q,k [T,dk], v [T,dv], a,b [T], S [dk,dv]. Returns (o, S_out)."""
    T = q.shape[0]
    n = -(-T // C)
    Tp = n * C
    q, k, v = _pad(q, Tp), _pad(k, Tp), _pad(v, Tp)
    la = _pad(np.log(a), Tp)            # log 1 = 0 on padding
    b = _pad(b, Tp)
    o = np.zeros((Tp, v.shape[1]))
    S = S.copy()
    for c in range(n):
        s = slice(c * C, (c + 1) * C)
        Q, K, V, bb = q[s], k[s], v[s], b[s]
        g = np.cumsum(la[s])
        low = np.tril(np.ones((C, C), bool))
        Gam = np.where(low, np.exp(np.where(low, g[:, None] - g[None, :], 0)), 0)  # e^{g_i-g_j}, j<=i
        L = np.tril(bb[:, None] * Gam * (K @ K.T), -1)
        Tinv = np.linalg.inv(np.eye(C) + L)
        W = Tinv @ ((bb * np.exp(g))[:, None] * K)
        U = Tinv @ (bb[:, None] * V)
        D = U - W @ S
        P = np.tril(Gam * (Q @ K.T))
        o[s] = np.exp(g)[:, None] * (Q @ S) + P @ D
        S = np.exp(g[-1]) * S + (np.exp(g[-1] - g)[:, None] * K).T @ D
    return o[:T], S


def reverse_one(q, k, v, a, b, R, C):
    """Reverse scan with the strict readout, chunks aligned with the forward
    pass (the padded tail chunk is visited first).  Returns (o, R_out)."""
    T = q.shape[0]
    n = -(-T // C)
    Tp = n * C
    q, k, v = _pad(q, Tp), _pad(k, Tp), _pad(v, Tp)
    la = _pad(np.log(a), Tp)
    b = _pad(b, Tp)
    o = np.zeros((Tp, v.shape[1]))
    R = R.copy()
    for c in reversed(range(n)):
        s = slice(c * C, (c + 1) * C)
        Q, K, V, bb = q[s], k[s], v[s], b[s]
        h = np.cumsum(la[s][::-1])[::-1]          # h_i = sum_{m>=i}
        h_next = np.append(h[1:], 0.0)            # h_{i+1}, h_C = 0
        i, j = np.meshgrid(np.arange(C), np.arange(C), indexing="ij")
        up = j > i
        Lp = np.where(up, bb[:, None] * np.exp(np.where(up, h[:, None] - h[None, :], 0)) * (K @ K.T), 0)
        Tinv = np.linalg.inv(np.eye(C) + Lp)
        W = Tinv @ ((bb * np.exp(h))[:, None] * K)
        U = Tinv @ (bb[:, None] * V)
        D = U - W @ R
        Pp = np.where(up, np.exp(np.where(up, h_next[:, None] - h[None, :], 0)) * (Q @ K.T), 0)
        o[s] = np.exp(h_next)[:, None] * (Q @ R) + Pp @ D
        R = np.exp(h[0]) * R + (np.exp(h[0] - h)[:, None] * K).T @ D
    return o[:T], R


def scan(q, k, v, alpha, beta, mode="causal", state_in=None, state_in_bwd=None, C=64):
    """Same interface as the oracle's scan on [B,T,H,*] float arrays."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    alpha, beta = np.asarray(alpha, np.float64), np.asarray(beta, np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    sb = np.zeros((B, H, dk, dv))
    for bb in range(B):
        for h in range(H):
            args = (q[bb, :, h], k[bb, :, h], v[bb, :, h], alpha[bb, :, h], beta[bb, :, h])
            if mode in ("causal", "bidir"):
                S0 = np.zeros((dk, dv)) if state_in is None else state_in[bb, h]
                of, sf[bb, h] = forward_one(*args, S0, C)
                o[bb, :, h] += of
            if mode in ("reverse", "bidir"):
                R0 = np.zeros((dk, dv)) if state_in_bwd is None else state_in_bwd[bb, h]
                ob, sb[bb, h] = reverse_one(*args, R0, C)
                o[bb, :, h] += ob
    return o, sf, sb
