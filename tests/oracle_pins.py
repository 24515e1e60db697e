"""Pins for the fp64 oracle: checks against what the review pages and plain
mathematics fix, none of which re-types the oracle's own loop.

Each ``pin_*`` function takes an oracle library handle (``lib=None`` means the
real one) and raises AssertionError on a mismatch.  ``test_oracle_pins.py``
runs them against the oracle; ``test_oracle_mutants.py`` runs them against
copies of the oracle with planted mistakes and expects at least one to fail.

Page citations: "Gated Delta Networks: Improving Mamba2 with Delta Rule"
(paper review) -- section "Method" (the recurrence; the delta rule as one
test-time SGD step with learning rate b_t and the gate as a weight decay),
section "Key idea" (a_t -> 0 erases, a_t -> 1 is the pure delta rule),
section "Background" (the state as an associative key->value memory),
section "Future work" (negative-eigenvalue transitions: b in (0, 2), so that
I - b k k^T may flip the sign along k).
"""
from __future__ import annotations

import json
import os

import numpy as np
import scipy.linalg

import oracle
from oracle import chunkwise

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _unit(rng, shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _inputs(rng, B=1, T=6, H=1, dk=4, dv=3, channel=False, g_shift=0.0, beta_max=1.0):
    q = _unit(rng, (B, T, H, dk))
    k = _unit(rng, (B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    gshape = (B, T, H, dk) if channel else (B, T, H)
    g = -np.log1p(np.exp(rng.standard_normal(gshape) + g_shift))
    beta = beta_max / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    h0 = 0.5 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, g, beta, h0


def _close(a, b, tol, what):
    err = float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) if np.size(a) else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


# --------------------------------------------------------------------------
def pin_golden(lib=None):
    """Hand-worked decimal examples (tests/golden/hand_worked.json)."""
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        q = np.array(c["q"], float)[None, :, None, :]
        k = np.array(c["k"], float)[None, :, None, :]
        v = np.array(c["v"], float)[None, :, None, :]
        a = np.array(c["alpha"], float)
        g = np.log(a)[None, :, None] if not c["channel_gate"] else np.log(a)[None, :, None, :]
        beta = np.array(c["beta"], float)[None, :, None]
        h0 = np.array(c["h0"], float)[None, None]
        o, hT = oracle.fwd(q, k, v, g, beta, h0, lib=lib)
        _close(o[0, :, 0], c["o"], 1e-12, c["name"] + " o")
        _close(hT[0, 0], c["hT"], 1e-12, c["name"] + " hT")


def pin_overwrite(lib=None):
    """a=1, b=1 and orthonormal keys: the state is an exact key->value memory;
    re-writing a key replaces its value and leaves the others alone."""
    rng = np.random.default_rng(1)
    d, T = 6, 6
    Kq, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Kq.T                                    # rows orthonormal
    vals = rng.standard_normal((T + 1, d))
    k = np.concatenate([keys[:T], keys[:1]])[None, :, None, :]
    v = vals[None, :, None, :]
    q = _unit(rng, (1, T + 1, 1, d))
    g = np.zeros((1, T + 1, 1))
    beta = np.ones((1, T + 1, 1))
    h0 = rng.standard_normal((1, 1, d, d))
    for n in range(1, T + 1):
        _, S = oracle.fwd(q[:, :n], k[:, :n], v[:, :n], g[:, :n], beta[:, :n], h0, lib=lib)
        for i in range(n):
            _close(S[0, 0] @ keys[i], vals[i], 1e-12, f"overwrite n={n} key {i}")
    _, S = oracle.fwd(q, k, v, g, beta, h0, lib=lib)
    _close(S[0, 0] @ keys[0], vals[T], 1e-12, "re-written key 0")
    for i in range(1, T):
        _close(S[0, 0] @ keys[i], vals[i], 1e-12, f"untouched key {i}")


def pin_one_token_geometry(lib=None):
    """One token from a random state S0 (scalar gate, unit k):
    S1 x = a S0 x for x orthogonal to k, and S1 k = a(1-b) S0 k + b v."""
    rng = np.random.default_rng(2)
    dk, dv = 5, 4
    for trial in range(5):
        q, k, v, g, beta, h0 = _inputs(rng, T=1, dk=dk, dv=dv)
        _, S1 = oracle.fwd(q, k, v, g, beta, h0, lib=lib)
        a, b = np.exp(g[0, 0, 0]), beta[0, 0, 0]
        kk = k[0, 0, 0]
        x = rng.standard_normal(dk)
        x -= (x @ kk) * kk
        _close(S1[0, 0] @ x, a * (h0[0, 0] @ x), 1e-12, "orthogonal direction")
        _close(S1[0, 0] @ kk, a * (1 - b) * (h0[0, 0] @ kk) + b * v[0, 0, 0], 1e-12,
               "written direction")


def pin_identity_and_decay(lib=None):
    """b=0: no write.  With a=1 the state stays h0 and o_t = h0 q_t; with a
    general gate it decays in closed form: scalar S_t = exp(G_t) h0,
    channel S_t = h0 Diag(exp(G_t)), G_t = g_1 + ... + g_t."""
    rng = np.random.default_rng(3)
    for channel in (False, True):
        q, k, v, g, beta, h0 = _inputs(rng, B=2, T=7, H=2, dk=4, dv=3, channel=channel)
        beta0 = np.zeros_like(beta)
        o, S = oracle.fwd(q, k, v, np.zeros_like(g), beta0, h0, lib=lib)
        _close(S, h0, 1e-14, "identity state")
        _close(o, np.einsum("bhac,bthc->btha", h0, q), 1e-14, "identity output")
        o, S = oracle.fwd(q, k, v, g, beta0, h0, lib=lib)
        G = np.cumsum(g, axis=1)
        if channel:
            ref_o = np.einsum("bhac,bthc->btha", h0, q * np.exp(G))
            ref_S = h0 * np.exp(G[:, -1])[:, :, None, :]
        else:
            ref_o = np.exp(G)[..., None] * np.einsum("bhac,bthc->btha", h0, q)
            ref_S = h0 * np.exp(G[:, -1])[:, :, None, None]
        _close(o, ref_o, 1e-14, f"decay output channel={channel}")
        _close(S, ref_S, 1e-14, f"decay state channel={channel}")


def pin_erase_limit(lib=None):
    """a -> 0 (g = -80): each token wipes the past, S_t = b_t v_t k_t^T and
    o_t = b_t v_t (k_t . q_t)."""
    rng = np.random.default_rng(4)
    for channel in (False, True):
        q, k, v, g, beta, h0 = _inputs(rng, B=1, T=5, H=2, dk=4, dv=3, channel=channel)
        g = np.full_like(g, -80.0)
        o, S = oracle.fwd(q, k, v, g, beta, h0, lib=lib)
        ref_o = beta[..., None] * v * np.sum(k * q, -1)[..., None]
        _close(o, ref_o, 1e-12, "erase output")
        ref_S = np.einsum("bh,bha,bhc->bhac", beta[:, -1], v[:, -1], k[:, -1])
        _close(S, ref_S, 1e-12, "erase state")


def pin_contraction(lib=None):
    """Unit keys, b in (0,2), a <= 1, v = 0: every step is a contraction
    (|1 - b| < 1 along k), so ||S_t||_F never grows."""
    rng = np.random.default_rng(5)
    for channel in (False, True):
        N, H, d = 3, 2, 5
        S = rng.standard_normal((N, H, d, d))
        prev = np.linalg.norm(S, axis=(2, 3))
        for t in range(12):
            q = _unit(rng, (N, H, d)); k = _unit(rng, (N, H, d))
            v = np.zeros((N, H, d))
            g = -np.log1p(np.exp(rng.standard_normal((N, H, d) if channel else (N, H))))
            b = (1 + (t % 2)) / (1 + np.exp(-rng.standard_normal((N, H))))  # (0,1) or (0,2)
            _, S = oracle.step(q, k, v, g, b, S, lib=lib)
            now = np.linalg.norm(S, axis=(2, 3))
            assert np.all(now < prev + 1e-15), "state norm grew"
            prev = now


def pin_sgd_view(lib=None):
    """The update is one SGD step with learning rate b on the loss
    l(S) = 1/2 ||S k - v||^2 taken at the decayed state Sh = S D:
    S_t = Sh - b grad l(Sh).  The gradient is taken by central differences."""
    rng = np.random.default_rng(6)
    for channel in (False, True):
        N, H, dk, dv = 1, 1, 4, 3
        S0 = rng.standard_normal((N, H, dv, dk))
        q = _unit(rng, (N, H, dk)); k = _unit(rng, (N, H, dk))
        v = rng.standard_normal((N, H, dv))
        g = -np.log1p(np.exp(rng.standard_normal((N, H, dk) if channel else (N, H))))
        b = np.array([[0.37]])
        _, S1 = oracle.step(q, k, v, g, b, S0, lib=lib)
        D = np.diag(np.exp(g[0, 0])) if channel else np.exp(g[0, 0]) * np.eye(dk)
        Sh = S0[0, 0] @ D
        kk, vv = k[0, 0], v[0, 0]
        loss = lambda S: 0.5 * np.sum((S @ kk - vv) ** 2)
        grad = np.zeros_like(Sh)
        h = 1e-6
        for idx in np.ndindex(*Sh.shape):
            E = np.zeros_like(Sh); E[idx] = h
            grad[idx] = (loss(Sh + E) - loss(Sh - E)) / (2 * h)
        _close(S1[0, 0], Sh - b[0, 0] * grad, 1e-8, f"sgd view channel={channel}")


def pin_dense_closed_form(lib=None):
    """Whole sequence as one chunk: (I + A) U = diag(b) V - diag(b e^G) K S0^T
    solved with a library unit-lower-triangular solve, then
    O = (Q e^G) S0^T + lower(Q K^T .* decay) U and
    S_T = e^{G_T} S0 + U^T (K e^{G_T - G})."""
    rng = np.random.default_rng(7)
    for channel in (False, True):
        for T in (1, 7, 16):
            q, k, v, g, beta, h0 = _inputs(rng, T=T, dk=5, dv=4, channel=channel)
            o, S = oracle.fwd(q, k, v, g, beta, h0, lib=lib)
            Q, K, V, b = q[0, :, 0], k[0, :, 0], v[0, :, 0], beta[0, :, 0]
            S0 = h0[0, 0]
            G = np.cumsum(g[0, :, 0], axis=0)
            if channel:
                E = np.exp(G[:, None, :] - G[None, :, :]) * np.tril(np.ones((T, T)))[:, :, None]
                KK = np.einsum("ic,jc,ijc->ij", K, K, E)
                QK = np.einsum("ic,jc,ijc->ij", Q, K, E)
                rhs = b[:, None] * V - (b[:, None] * K * np.exp(G)) @ S0.T
                Qg = Q * np.exp(G)
                Kt = K * np.exp(G[-1] - G)
                S_dec = S0 * np.exp(G[-1])
            else:
                E = np.exp(np.minimum(G[:, None] - G[None, :], 0.0)) * np.tril(np.ones((T, T)))
                KK = (K @ K.T) * E
                QK = (Q @ K.T) * E
                rhs = b[:, None] * V - ((b * np.exp(G))[:, None] * K) @ S0.T
                Qg = Q * np.exp(G)[:, None]
                Kt = K * np.exp(G[-1] - G)[:, None]
                S_dec = S0 * np.exp(G[-1])
            A = np.tril(b[:, None] * KK, -1)
            U = scipy.linalg.solve_triangular(np.eye(T) + A, rhs, lower=True,
                                              unit_diagonal=True)
            O = Qg @ S0.T + np.tril(QK) @ U
            _close(o[0, :, 0], O, 1e-12, f"closed form o T={T} channel={channel}")
            _close(S[0, 0], S_dec + U.T @ Kt, 1e-12, f"closed form state T={T}")


def pin_chunkwise(lib=None):
    """Chunkwise WY/UT algebra (numpy) equals the token loop for several
    chunk sizes, ragged tails included, forward and backward."""
    rng = np.random.default_rng(8)
    for channel in (False, True):
        for T, C in ((1, 4), (7, 2), (16, 4), (37, 16), (64, 16)):
            q, k, v, g, beta, h0 = _inputs(rng, B=1, T=T, H=2, dk=5, dv=4,
                                          channel=channel, g_shift=-1.0)
            dO = rng.standard_normal(v.shape)
            dhT = rng.standard_normal(h0.shape)
            o, S = oracle.fwd(q, k, v, g, beta, h0, scale=0.8, lib=lib)
            o2, S2 = chunkwise.chunk_forward(q, k, v, g, beta, h0, C=C, scale=0.8)
            _close(o, o2, 1e-12, f"chunk fwd o T={T} C={C}")
            _close(S, S2, 1e-12, f"chunk fwd state T={T} C={C}")
            r = oracle.bwd(q, k, v, g, beta, dO, h0, dhT, scale=0.8, ckpt=3, lib=lib)
            r2 = chunkwise.chunk_backward(q, k, v, g, beta, dO, h0, dhT, C=C, scale=0.8)
            for n in r:
                _close(r[n], r2[n], 1e-11, f"chunk bwd {n} T={T} C={C}")


def pin_negative_eigenvalue(lib=None):
    """b in (0, 2) (the negative-eigenvalue extension).  With unit k and v = 0
    one token maps S0 to a S0 (I - b k k^T), whose Frobenius norm satisfies
    ||S1||^2 = a^2 (||S0||^2 - b (2 - b) ||S0 k||^2); at b = 2, a = 1 the map
    is the Householder reflection through k's orthogonal complement
    (S1 k = -S0 k, S1 x = S0 x for x orthogonal to k).  The chunkwise algebra
    still equals the token loop with b up to 2."""
    rng = np.random.default_rng(13)
    dk, dv = 5, 4
    for trial in range(4):
        q, k, v, g, beta, h0 = _inputs(rng, T=1, dk=dk, dv=dv, beta_max=2.0)
        v = np.zeros_like(v)
        _, S1 = oracle.fwd(q, k, v, g, beta, h0, lib=lib)
        a, b, kk = np.exp(g[0, 0, 0]), beta[0, 0, 0], k[0, 0, 0]
        want = a * a * (np.sum(h0[0, 0] ** 2) - b * (2 - b) * np.sum((h0[0, 0] @ kk) ** 2))
        _close(np.sum(S1[0, 0] ** 2), want, 1e-12, "norm drop")
        beta2 = np.full_like(beta, 2.0)
        _, R = oracle.fwd(q, k, v, np.zeros_like(g), beta2, h0, lib=lib)
        x = rng.standard_normal(dk)
        x -= (x @ kk) * kk
        _close(R[0, 0] @ kk, -(h0[0, 0] @ kk), 1e-12, "reflected direction")
        _close(R[0, 0] @ x, h0[0, 0] @ x, 1e-12, "fixed complement")
        _close(np.linalg.norm(R[0, 0]), np.linalg.norm(h0[0, 0]), 1e-12, "reflection norm")
    for channel in (False, True):
        q, k, v, g, beta, h0 = _inputs(rng, B=1, T=37, H=2, dk=5, dv=4, channel=channel,
                                      g_shift=-1.0, beta_max=2.0)
        assert beta.max() > 1.0
        dO = rng.standard_normal(v.shape)
        dhT = rng.standard_normal(h0.shape)
        o, S = oracle.fwd(q, k, v, g, beta, h0, lib=lib)
        o2, S2 = chunkwise.chunk_forward(q, k, v, g, beta, h0, C=16)
        _close(o, o2, 1e-11, "chunk fwd o, b in (0,2)")
        _close(S, S2, 1e-11, "chunk fwd state, b in (0,2)")
        r = oracle.bwd(q, k, v, g, beta, dO, h0, dhT, ckpt=3, lib=lib)
        r2 = chunkwise.chunk_backward(q, k, v, g, beta, dO, h0, dhT, C=16)
        for n in r:
            _close(r[n], r2[n], 1e-10, f"chunk bwd {n}, b in (0,2)")


def pin_channel_equals_scalar(lib=None):
    """A channel gate with the same value in every channel is the scalar gate
    (forward, and the scalar dg is the channel sum of the channel dg)."""
    rng = np.random.default_rng(9)
    q, k, v, g, beta, h0 = _inputs(rng, B=2, T=9, H=2, dk=4, dv=3)
    gc = np.repeat(g[..., None], 4, axis=-1)
    dO = rng.standard_normal(v.shape); dhT = rng.standard_normal(h0.shape)
    o1, S1 = oracle.fwd(q, k, v, g, beta, h0, lib=lib)
    o2, S2 = oracle.fwd(q, k, v, gc, beta, h0, lib=lib)
    _close(o1, o2, 1e-13, "channel==scalar o")
    _close(S1, S2, 1e-13, "channel==scalar state")
    r1 = oracle.bwd(q, k, v, g, beta, dO, h0, dhT, lib=lib)
    r2 = oracle.bwd(q, k, v, gc, beta, dO, h0, dhT, lib=lib)
    _close(r1["dg"], r2["dg"].sum(-1), 1e-12, "channel==scalar dg")
    for n in ("dq", "dk", "dv", "dbeta", "dh0"):
        _close(r1[n], r2[n], 1e-12, f"channel==scalar {n}")


def pin_step_and_resume(lib=None):
    """fwd over T tokens == T successive decode steps; fwd(T1+T2) ==
    fwd(T2) started from the state fwd(T1) returns."""
    rng = np.random.default_rng(10)
    for channel in (False, True):
        q, k, v, g, beta, h0 = _inputs(rng, B=2, T=11, H=3, dk=4, dv=5, channel=channel)
        o, S = oracle.fwd(q, k, v, g, beta, h0, scale=1.3, lib=lib)
        st = h0.copy()
        for t in range(q.shape[1]):
            ot, st = oracle.step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], st,
                                 scale=1.3, lib=lib)
            _close(ot, o[:, t], 1e-13, f"step t={t}")
        _close(st, S, 1e-13, "steps final state")
        oa, Sa = oracle.fwd(q[:, :4], k[:, :4], v[:, :4], g[:, :4], beta[:, :4], h0,
                            scale=1.3, lib=lib)
        ob, Sb = oracle.fwd(q[:, 4:], k[:, 4:], v[:, 4:], g[:, 4:], beta[:, 4:], Sa,
                            scale=1.3, lib=lib)
        _close(np.concatenate([oa, ob], 1), o, 1e-13, "resume o")
        _close(Sb, S, 1e-13, "resume state")


def _loss(params, dO, dhT, scale, lib):
    o, S = oracle.fwd(params["q"], params["k"], params["v"], params["g"],
                      params["beta"], params["h0"], scale=scale, lib=lib)
    return float(np.sum(dO * o) + np.sum(dhT * S))


def pin_bwd_finite_differences(lib=None):
    """Backward = central finite differences of L = <dO,o> + <dhT,hT>."""
    rng = np.random.default_rng(11)
    for channel in (False, True):
        q, k, v, g, beta, h0 = _inputs(rng, B=1, T=5, H=1, dk=3, dv=3, channel=channel)
        dO = rng.standard_normal(v.shape); dhT = rng.standard_normal(h0.shape)
        scale = 0.9
        r = oracle.bwd(q, k, v, g, beta, dO, h0, dhT, scale=scale, ckpt=2, lib=lib)
        params = dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0)
        names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0")
        h = 1e-6
        for p, gname in names.items():
            fd = np.zeros_like(params[p])
            for idx in np.ndindex(*params[p].shape):
                for sgn in (1, -1):
                    pp = {n: a.copy() for n, a in params.items()}
                    pp[p][idx] += sgn * h
                    fd[idx] += sgn * _loss(pp, dO, dhT, scale, lib) / (2 * h)
            _close(r[gname], fd, 1e-7, f"FD {gname} channel={channel}")


def pin_euler(lib=None):
    """o and hT are linear in (v, h0), and o is linear in q, so
    <dv,v> + <dh0,h0> = <dO,o> + <dhT,hT> and <dq,q> = <dO,o>."""
    rng = np.random.default_rng(12)
    for channel in (False, True):
        q, k, v, g, beta, h0 = _inputs(rng, B=2, T=13, H=2, dk=6, dv=5, channel=channel)
        dO = rng.standard_normal(v.shape); dhT = rng.standard_normal(h0.shape)
        o, S = oracle.fwd(q, k, v, g, beta, h0, lib=lib)
        r = oracle.bwd(q, k, v, g, beta, dO, h0, dhT, ckpt=4, lib=lib)
        lhs = np.sum(r["dv"] * v) + np.sum(r["dh0"] * h0)
        rhs = np.sum(dO * o) + np.sum(dhT * S)
        assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(rhs)), f"euler v/h0 {lhs} {rhs}"
        lq = np.sum(r["dq"] * q)
        assert abs(lq - np.sum(dO * o)) <= 1e-11 * max(1.0, abs(rhs)), "euler q"


ALL_PINS = [pin_golden, pin_overwrite, pin_one_token_geometry, pin_identity_and_decay,
            pin_erase_limit, pin_contraction, pin_negative_eigenvalue, pin_sgd_view,
            pin_dense_closed_form,
            pin_chunkwise, pin_channel_equals_scalar, pin_step_and_resume,
            pin_bwd_finite_differences, pin_euler]
