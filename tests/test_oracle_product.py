"""Pins for the fp64 DeltaProduct oracle (oracle/product.py), each against
something other than the oracle itself: the gated-delta oracle (a separate
C implementation), explicit Householder products, reflections, finite
differences.  Page citation: "DeltaProduct: Improving State-Tracking in Linear
RNNs via Householder Products" (title on the pages) and the "Gated Delta
Networks" review, section "Future work" (products of Householder matrices)."""
import numpy as np

import oracle
from oracle import product


def _unit(rng, shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _inputs(rng, B=2, T=5, n=2, H=2, dk=4, dv=3, channel=False, beta_max=1.0):
    q = _unit(rng, (B, T, H, dk))
    k = _unit(rng, (B, T, n, H, dk))
    v = rng.standard_normal((B, T, n, H, dv))
    g = -np.log1p(np.exp(rng.standard_normal((B, T, H, dk) if channel else (B, T, H))))
    beta = beta_max / (1 + np.exp(-rng.standard_normal((B, T, n, H))))
    h0 = 0.5 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, g, beta, h0


def test_one_step_per_token_is_the_gated_delta_rule():
    rng = np.random.default_rng(21)
    for channel in (False, True):
        q, k, v, g, beta, h0 = _inputs(rng, n=1, channel=channel)
        o, S = product.forward(q, k, v, g, beta, h0, scale=0.7)
        o2, S2 = oracle.fwd(q, k[:, :, 0], v[:, :, 0], g, beta[:, :, 0], h0, scale=0.7)
        assert np.abs(o - o2).max() < 1e-12 and np.abs(S - S2).max() < 1e-12
        dO = rng.standard_normal(o.shape)
        dhT = rng.standard_normal(S.shape)
        r = product.backward(q, k, v, g, beta, dO, h0, dhT, scale=0.7)
        r2 = oracle.bwd(q, k[:, :, 0], v[:, :, 0], g, beta[:, :, 0], dO, h0, dhT, scale=0.7)
        assert np.abs(r["dq"] - r2["dq"]).max() < 1e-11
        assert np.abs(r["dk"][:, :, 0] - r2["dk"]).max() < 1e-11
        assert np.abs(r["dv"][:, :, 0] - r2["dv"]).max() < 1e-11
        assert np.abs(r["dbeta"][:, :, 0] - r2["dbeta"]).max() < 1e-11
        assert np.abs(r["dg"] - r2["dg"]).max() < 1e-11
        assert np.abs(r["dh0"] - r2["dh0"]).max() < 1e-11


def test_transition_is_the_ordered_householder_product():
    """a = 1, v = 0: the state is h0 times prod_t prod_j (I - b_tj k_tj k_tj^T),
    in that order."""
    rng = np.random.default_rng(22)
    q, k, v, g, beta, h0 = _inputs(rng, B=1, T=4, n=3, H=1, dk=5, dv=3, beta_max=2.0)
    _, S = product.forward(q, k, np.zeros_like(v), np.zeros_like(g), beta, h0)
    M = np.eye(5)
    for t in range(4):
        for j in range(3):
            kk = k[0, t, j, 0]
            M = M @ (np.eye(5) - beta[0, t, j, 0] * np.outer(kk, kk))
    assert np.abs(S[0, 0] - h0[0, 0] @ M).max() < 1e-12


def test_reflections_keep_the_norm():
    """b = 2, unit keys, a = 1, v = 0: every sub-step is a reflection."""
    rng = np.random.default_rng(23)
    q, k, v, g, beta, h0 = _inputs(rng, B=1, T=6, n=3, H=2)
    _, S = product.forward(q, k, np.zeros_like(v), np.zeros_like(g), np.full_like(beta, 2.0), h0)
    assert np.abs(np.linalg.norm(S, axis=(2, 3)) - np.linalg.norm(h0, axis=(2, 3))).max() < 1e-12


def test_equals_the_gated_delta_rule_on_interleaved_sub_tokens():
    """The n sub-steps of token t are the gated delta rule on the sub-token
    sequence (t, 1) .. (t, n), with g_t on the first sub-token, 0 on the rest,
    and o_t read at the last (zero q elsewhere)."""
    rng = np.random.default_rng(24)
    for channel in (False, True):
        B, T, n, H, dk, dv = 2, 7, 3, 2, 4, 3
        q, k, v, g, beta, h0 = _inputs(rng, B, T, n, H, dk, dv, channel=channel, beta_max=2.0)
        o, S = product.forward(q, k, v, g, beta, h0)
        qx = np.zeros((B, T, n, H, dk)); qx[:, :, -1] = q
        gx = np.zeros((B, T, n) + g.shape[2:]); gx[:, :, 0] = g
        o2, S2 = oracle.fwd(qx.reshape(B, T * n, H, dk), k.reshape(B, T * n, H, dk),
                            v.reshape(B, T * n, H, dv), gx.reshape((B, T * n) + g.shape[2:]),
                            beta.reshape(B, T * n, H), h0)
        assert np.abs(o - o2.reshape(B, T, n, H, dv)[:, :, -1]).max() < 1e-12
        assert np.abs(S - S2).max() < 1e-12


def test_gradients_match_finite_differences():
    rng = np.random.default_rng(25)
    q, k, v, g, beta, h0 = _inputs(rng, B=1, T=3, n=2, H=1, dk=3, dv=2, channel=True)
    dO = rng.standard_normal((1, 3, 1, 2))
    dhT = rng.standard_normal((1, 1, 2, 3))
    r = product.backward(q, k, v, g, beta, dO, h0, dhT)

    def loss(**over):
        a = dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0)
        a.update(over)
        o, S = product.forward(a["q"], a["k"], a["v"], a["g"], a["beta"], a["h0"])
        return float((o * dO).sum() + (S * dhT).sum())

    h = 1e-6
    for name, x in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta), ("h0", h0)):
        d = rng.standard_normal(x.shape)
        fd = (loss(**{name: x + h * d}) - loss(**{name: x - h * d})) / (2 * h)
        assert abs(fd - float((r["d" + name] * d).sum())) < 1e-7 * max(1.0, abs(fd)), name
