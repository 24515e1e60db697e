"""Pins for the draft-tree oracle (oracle/tree.py), each against something
other than the oracle itself: the C token-loop oracle on chains, stars and the
root paths of random trees, plus two structural invariants (only descendants
see a node's token; relabelling the nodes in another topological order
relabels the outputs).  Page citation: "TreeWY: Speculative Verification for
Gated DeltaNet Hybrids" (the "Linked reviews" entry of the "Gated Delta Networks"
review page) and the gated delta rule of the "Gated Delta Networks" review,
section "Method"."""
import numpy as np

import oracle
from oracle import tree


def _unit(rng, shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _inputs(rng, N=2, M=7, H=2, dk=5, dv=3, channel=False):
    q = _unit(rng, (N, M, H, dk))
    k = _unit(rng, (N, M, H, dk))
    v = rng.standard_normal((N, M, H, dv))
    g = -np.log1p(np.exp(rng.standard_normal((N, M, H) + ((dk,) if channel else ()))))
    beta = 1 / (1 + np.exp(-rng.standard_normal((N, M, H))))
    S0 = 0.5 * rng.standard_normal((N, H, dv, dk))
    return q, k, v, g, beta, S0


def _random_parents(rng, N, M):
    return np.array([[rng.integers(-1, i) for i in range(M)] for _ in range(N)])


def test_chain_is_the_token_loop(channel=False):
    """parent[i] = i - 1: node i reads out token i of one sequence; committing
    node j gives the state after its first j + 1 tokens (scalar gate, and the
    channel gate against the C oracle's per-key decay)."""
    rng = np.random.default_rng(31)
    q, k, v, g, beta, S0 = _inputs(rng, channel=channel)
    N, M = q.shape[:2]
    par = np.tile(np.arange(M) - 1, (N, 1))
    o = tree.verify(par, q, k, v, g, beta, S0, scale=0.8)
    o2, _ = oracle.fwd(q, k, v, g, beta, S0, scale=0.8)
    assert np.abs(o - o2).max() < 1e-12
    for j in (0, 3, M - 1):
        S = tree.commit(par, [j] * N, k, v, g, beta, S0)
        _, S2 = oracle.fwd(q[:, :j + 1], k[:, :j + 1], v[:, :j + 1], g[:, :j + 1],
                           beta[:, :j + 1], S0)
        assert np.abs(S - S2).max() < 1e-12


def test_star_is_one_decode_step_per_node(channel=False):
    """Every parent -1: each node is one decode step from S0."""
    rng = np.random.default_rng(32)
    q, k, v, g, beta, S0 = _inputs(rng, N=1, M=6, channel=channel)
    par = -np.ones((1, 6), dtype=int)
    o = tree.verify(par, q, k, v, g, beta, S0, scale=1.3)
    for i in range(6):
        oi, Si = oracle.step(q[:, i], k[:, i], v[:, i], g[:, i], beta[:, i], S0, scale=1.3)
        assert np.abs(o[:, i] - oi).max() < 1e-12
        S = tree.commit(par, [i], k, v, g, beta, S0)
        assert np.abs(S - Si).max() < 1e-12


def test_chain_is_the_token_loop_channel_gate():
    test_chain_is_the_token_loop(channel=True)


def test_star_is_one_decode_step_per_node_channel_gate():
    test_star_is_one_decode_step_per_node(channel=True)


def test_random_trees_follow_their_root_paths():
    """Node i of a random tree equals the C oracle run over the tokens of its
    root path (last read-out); commit equals that run's final state."""
    rng = np.random.default_rng(33)
    N, M = 3, 9
    q, k, v, g, beta, S0 = _inputs(rng, N=N, M=M)
    par = _random_parents(rng, N, M)
    o = tree.verify(par, q, k, v, g, beta, S0)
    acc = [int(rng.integers(-1, M)) for _ in range(N)]
    S = tree.commit(par, acc, k, v, g, beta, S0)
    for n in range(N):
        for i in range(M):
            p = tree.root_path(par[n], i)
            assert p[-1] == i and all(par[n][p[j]] == (p[j - 1] if j else -1)
                                      for j in range(len(p)))
            oi, Si = oracle.fwd(*(x[n:n + 1, p] for x in (q, k, v, g, beta)), S0[n:n + 1])
            assert np.abs(o[n, i] - oi[0, -1]).max() < 1e-12
            if i == acc[n]:
                assert np.abs(S[n] - Si[0]).max() < 1e-12
        if acc[n] < 0:
            assert np.array_equal(S[n], S0[n])


def test_only_descendants_see_a_node():
    rng = np.random.default_rng(34)
    N, M = 1, 10
    q, k, v, g, beta, S0 = _inputs(rng, N=N, M=M)
    par = _random_parents(rng, N, M)
    o = tree.verify(par, q, k, v, g, beta, S0)
    j = 2
    v2 = v.copy()
    v2[0, j] += 1.0
    o2 = tree.verify(par, q, k, v2, g, beta, S0)
    for i in range(M):
        below = j in tree.root_path(par[0], i)
        changed = np.abs(o2[0, i] - o[0, i]).max() > 1e-9
        assert changed == below, (i, below)


def test_relabelling_relabels_the_outputs():
    """Any topological renumbering of the same tree gives the same per-node
    outputs under the new numbers."""
    rng = np.random.default_rng(35)
    M = 8
    q, k, v, g, beta, S0 = _inputs(rng, N=1, M=M)
    par = _random_parents(rng, 1, M)[0]
    # a topological order other than the identity: children before later
    # siblings' subtrees, by depth-first search with reversed child lists
    kids = {i: [c for c in range(M) if par[c] == i] for i in range(-1, M)}
    order, stack = [], list(kids[-1])
    while stack:
        x = stack.pop()
        order.append(x)
        stack.extend(kids[x])
    new_of = {old: new for new, old in enumerate(order)}
    par2 = np.array([[new_of[par[old]] if par[old] >= 0 else -1 for old in order]])
    sel = lambda x: x[:, order]  # noqa: E731
    o = tree.verify(par[None], q, k, v, g, beta, S0)
    o2 = tree.verify(par2, sel(q), sel(k), sel(v), sel(g), sel(beta), S0)
    assert np.abs(o2 - o[:, order]).max() < 1e-12
