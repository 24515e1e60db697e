"""Chunkwise (WY / UT-transform) form of the gated delta rule in numpy fp64.

TEST INFRASTRUCTURE ONLY: used by the CPU tests to pin the chunkwise algebra
that the CUDA kernels implement against the token-by-token loop in
``gdn_oracle.c``.  The GPU path is never compared against this file; it is
compared against the token loop.

"Gated Delta Networks: Improving Mamba2 with Delta Rule" (paper review),
sections "Goal" and "Method": the recurrence is kept in a chunkwise-parallel,
matmul-dominated form built on the WY representation and the UT transform.
The review does not print the chunk equations; they are derived here from the
recurrence (every identity below is checked against the token loop by the
tests).

Per chunk of L tokens (rows i = 0..L-1), with S0 the state entering the chunk,
G = within-chunk cumulative sum of the log-gate g, and for the scalar gate
Gam_ij = exp(G_i - G_j):

  unrolled state   S_r = exp(G_r) S0 + sum_{i<=r} exp(G_r - G_i) u_i k_i^T
  pseudo-values    u_i = beta_i (v_i - S_{i-1} a_i k_i)
  => (I + A) U = diag(beta) V - diag(beta exp(G)) K S0^T,
     A = strict_lower(diag(beta) (K K^T .* Gam))
  UT transform     T = (I + A)^{-1}            (unit lower triangular)
  WY factors       W = T diag(beta exp(G)) K,   U~ = T diag(beta) V
                   U = U~ - W S0^T
  output           O = (Q .* exp(G)) S0^T + (lower(Q K^T .* Gam)) U
  next state       S_L = exp(G_last) S0 + U^T (K .* exp(G_last - G))

The channel gate replaces every exp(G_i - G_j) weight of a key/query product
by a per-channel weight inside the contraction:
  A_ij = beta_i sum_c k_ic k_jc exp(G_ic - G_jc),  P_ij = sum_c q_ic k_jc exp(G_ic - G_jc),
  W = T diag(beta) (K .* exp(G)),  S_L = S0 Diag(exp(G_last)) + U^T (K .* exp(G_last - G)).
"""
from __future__ import annotations

import numpy as np


def _pair_decay(G):
    """exp(G_i - G_j) on and below the diagonal, 0 above.  G [L] or [L,dk];
    returns [L,L] or [L,L,dk]."""
    L = G.shape[0]
    mask = np.tril(np.ones((L, L), dtype=bool))
    if G.ndim == 1:
        e = np.where(mask, G[:, None] - G[None, :], -np.inf)
    else:
        e = np.where(mask[:, :, None], G[:, None, :] - G[None, :, :], -np.inf)
    return np.exp(e)


def chunk_forward_bh(q, k, v, g, beta, S0, C, scale=1.0):
    """One (b,h) stream.  q,k [T,dk], v [T,dv], g [T] or [T,dk], beta [T],
    S0 [dv,dk].  Returns (o [T,dv], S_T, per-chunk dict list)."""
    T, dk = q.shape
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    chunks = []
    for n0 in range(0, T, C):
        n1 = min(T, n0 + C)
        Q, K, V, b = scale * q[n0:n1], k[n0:n1], v[n0:n1], beta[n0:n1]
        G = np.cumsum(g[n0:n1], axis=0)
        L = n1 - n0
        D = _pair_decay(G)
        eG = np.exp(G)
        if G.ndim == 1:
            A = np.tril(b[:, None] * (K @ K.T) * D, -1)
            P = (Q @ K.T) * D
            Kg = (b * eG)[:, None] * K
            Qg = eG[:, None] * Q
            Kt = np.exp(G[-1] - G)[:, None] * K
            decay = lambda X: np.exp(G[-1]) * X
        else:
            A = np.tril(b[:, None] * np.einsum("ic,jc,ijc->ij", K, K, D), -1)
            P = np.einsum("ic,jc,ijc->ij", Q, K, D)
            Kg = b[:, None] * K * eG
            Qg = Q * eG
            Kt = K * np.exp(G[-1][None, :] - G)
            decay = lambda X: X * np.exp(G[-1])[None, :]
        Tm = np.linalg.inv(np.eye(L) + A)
        W = Tm @ Kg
        Ut = Tm @ (b[:, None] * V)
        U = Ut - W @ S.T
        O = Qg @ S.T + P @ U
        o[n0:n1] = O
        chunks.append(dict(S0=S.copy(), G=G, A=A, T=Tm, W=W, Ut=Ut, U=U, P=P,
                           Kg=Kg, Qg=Qg, Kt=Kt))
        S = decay(S) + U.T @ Kt
    return o, S, chunks


def chunk_forward(q, k, v, g, beta, h0=None, C=64, scale=1.0):
    """Batched wrapper with the library layouts: q,k [B,T,H,dk] ...
    Returns (o [B,T,H,dv], hT [B,H,dv,dk])."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S0 = h0[b, h] if h0 is not None else np.zeros((dv, dk))
            gg = g[b, :, h] if g.ndim == 3 else g[b, :, h, :]
            ob, Sb, _ = chunk_forward_bh(q[b, :, h], k[b, :, h], v[b, :, h], gg,
                                         beta[b, :, h], S0, C, scale)
            o[b, :, h] = ob
            hT[b, h] = Sb
    return o, hT


def chunk_backward_bh(q, k, v, g, beta, S0, dO, dST, C, scale=1.0):
    """Reverse-mode through the chunk equations above (one (b,h) stream).
    Returns dq, dk, dv, dg, dbeta, dS0."""
    T, dk = q.shape
    dv = v.shape[1]
    _, _, chunks = chunk_forward_bh(q, k, v, g, beta, S0, C, scale)
    dq = np.zeros_like(q); dkk = np.zeros_like(k); dvv = np.zeros_like(v)
    dg = np.zeros_like(g); db = np.zeros_like(beta)
    dS = dST.copy()
    channel = g.ndim == 2
    for ci in range(len(chunks) - 1, -1, -1):
        n0 = ci * C
        c = chunks[ci]
        n1 = n0 + c["U"].shape[0]
        Q, K, V, b = scale * q[n0:n1], k[n0:n1], v[n0:n1], beta[n0:n1]
        G, Tm, W, U, P, S0c = c["G"], c["T"], c["W"], c["U"], c["P"], c["S0"]
        Kt, Qg, Kg = c["Kt"], c["Qg"], c["Kg"]
        dOc = dO[n0:n1]
        eG = np.exp(G)
        D = _pair_decay(G)
        dG = np.zeros_like(G)
        # O = Qg S0^T + P U ; S_L = decay(S0) + U^T Kt ; U = Ut - W S0^T
        dU = P.T @ dOc + Kt @ dS.T
        dP = np.tril(dOc @ U.T)
        dQg = dOc @ S0c
        dKt = U @ dS
        dW = -dU @ S0c
        if channel:
            dS0 = dS * np.exp(G[-1])[None, :] + dOc.T @ Qg - dU.T @ W
            dG[-1] += np.sum(dS * S0c, axis=0) * np.exp(G[-1])
        else:
            dS0 = np.exp(G[-1]) * dS + dOc.T @ Qg - dU.T @ W
            dG[-1] += np.exp(G[-1]) * np.sum(dS * S0c)
        # W = T Kg ; Ut = T (beta V)
        dT = dW @ Kg.T + dU @ (b[:, None] * V).T
        dKg = Tm.T @ dW
        dVb = Tm.T @ dU
        dvv[n0:n1] = b[:, None] * dVb
        db[n0:n1] += np.sum(dVb * V, axis=1)
        # T = (I + A)^{-1}
        dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
        dKc = np.zeros_like(K)
        dQc = np.zeros_like(Q)
        if not channel:
            # Kg = diag(beta e^G) K ; Qg = diag(e^G) Q ; Kt = diag(e^{G_L - G}) K
            dKc += (b * eG)[:, None] * dKg
            hk = np.sum(dKg * K, axis=1)
            db[n0:n1] += eG * hk
            dG += b * eG * hk
            dQc += eG[:, None] * dQg
            dG += eG * np.sum(dQg * Q, axis=1)
            et = np.exp(G[-1] - G)
            dKc += et[:, None] * dKt
            hkt = et * np.sum(dKt * K, axis=1)
            dG[-1] += np.sum(hkt)
            dG -= hkt
            # A = strict_lower(diag(beta)(K K^T .* Gam))
            M = K @ K.T
            db[n0:n1] += np.sum(dA * M * D, axis=1)
            dMM = dA * b[:, None] * D
            dKc += dMM @ K + dMM.T @ K
            hA = dA * b[:, None] * M * D
            # P = lower(Q K^T .* Gam)
            dPG = dP * D
            dQc += dPG @ K
            dKc += dPG.T @ Q
            hP = dP * (Q @ K.T) * D
            hh = hA + hP
            dG += np.sum(hh, axis=1) - np.sum(hh, axis=0)
        else:
            dKc += b[:, None] * eG * dKg
            hk = dKg * K * eG               # [L,dk]
            db[n0:n1] += np.sum(hk, axis=1)
            dG += b[:, None] * hk
            dQc += eG * dQg
            dG += eG * dQg * Q
            et = np.exp(G[-1][None, :] - G)
            dKc += et * dKt
            hkt = et * dKt * K
            dG[-1] += np.sum(hkt, axis=0)
            dG -= hkt
            # A_ij = beta_i sum_c K_ic K_jc D_ijc ;  P_ij = sum_c Q_ic K_jc D_ijc
            db[n0:n1] += np.einsum("ij,ic,jc,ijc->i", dA, K, K, D)
            wA = dA * b[:, None]
            dKc += np.einsum("ij,jc,ijc->ic", wA, K, D) + np.einsum("ij,ic,ijc->jc", wA, K, D)
            hA = np.einsum("ij,ic,jc,ijc->ijc", wA, K, K, D)
            dQc += np.einsum("ij,jc,ijc->ic", dP, K, D)
            dKc += np.einsum("ij,ic,ijc->jc", dP, Q, D)
            hP = np.einsum("ij,ic,jc,ijc->ijc", dP, Q, K, D)
            hh = hA + hP
            dG += np.sum(hh, axis=1) - np.sum(hh, axis=0)
        dq[n0:n1] = scale * dQc
        dkk[n0:n1] = dKc
        # G = cumsum(g) within the chunk -> reverse cumsum
        dg[n0:n1] = np.flip(np.cumsum(np.flip(dG, 0), axis=0), 0)
        dS = dS0
    return dq, dkk, dvv, dg, db, dS


def chunk_backward(q, k, v, g, beta, dO, h0=None, dhT=None, C=64, scale=1.0):
    """Batched wrapper; returns dict like ``oracle.bwd``."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dg=np.zeros_like(g), dbeta=np.zeros_like(beta),
               dh0=np.zeros((B, H, dv, dk)))
    for b in range(B):
        for h in range(H):
            S0 = h0[b, h] if h0 is not None else np.zeros((dv, dk))
            dST = dhT[b, h] if dhT is not None else np.zeros((dv, dk))
            gg = g[b, :, h] if g.ndim == 3 else g[b, :, h, :]
            r = chunk_backward_bh(q[b, :, h], k[b, :, h], v[b, :, h], gg,
                                  beta[b, :, h], S0, dO[b, :, h], dST, C, scale)
            out["dq"][b, :, h], out["dk"][b, :, h], out["dv"][b, :, h] = r[0], r[1], r[2]
            if g.ndim == 3:
                out["dg"][b, :, h] = r[3]
            else:
                out["dg"][b, :, h, :] = r[3]
            out["dbeta"][b, :, h] = r[4]
            out["dh0"][b, h] = r[5]
    return out
