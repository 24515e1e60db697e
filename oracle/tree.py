"""fp64 CPU oracle for draft-tree verification and commit -- TEST
INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
may import this module; the CUDA library never uses it.

Source: "TreeWY: Speculative Verification for Gated DeltaNet Hybrids" (the
"Linked reviews" entry of the "Gated Delta Networks: Improving Mamba2 with
Delta Rule" review page).  The page gives the goal, not the
equations: score every node of a speculative draft tree against the committed
recurrent state without keeping one state snapshot per draft position, and on
commit rebuild only the state of the accepted node.  The reading taken here:

* A draft tree of M nodes hangs below the committed state S0 of each
  (sequence, head).  Node i carries one token (q_i, k_i, v_i, g_i, beta_i) and
  a parent index parent[i] in [-1, i); -1 means the node follows S0 directly.
  Parents come before their children, so the node order is topological.
* The output of node i is the gated delta rule ("Gated Delta Networks:
  Improving Mamba2 with Delta Rule", section "Method") run from S0 over the
  tokens of the root path of i, in path order, read out at i:
      S <- S a_t (I - b_t k_t k_t^T) + b_t v_t k_t^T  for t on the path,
      o_i = S (scale q_i).
* Commit with accepted node a (or -1: nothing accepted) replaces S0 by the
  state after the root path of a (S0 itself for -1).

Both functions below are those definitions written out: a token loop along
each node's path, in float64 numpy.  The tree-structured WY form is the CUDA
side's business; the pins compare this oracle with the C token-loop oracle on
chains, stars and the root paths of random trees.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().double().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def root_path(parent, i):
    """Node indices from the first node below S0 down to node i."""
    path = []
    j = int(i)
    while j >= 0:
        path.append(j)
        j = int(parent[j])
    return path[::-1]


def _run_path(S, path, k, v, g, beta):
    """Token loop of the gated delta rule over the nodes of `path`, one
    (sequence, head) pair: S [dv, dk]; k [M, dk]; v [M, dv]; beta [M]; g [M]
    (scalar gate) or [M, dk] (channel gate: the decay Diag(e^{g_t}) acts on the
    key index, i.e. scales the columns of S)."""
    S = S.copy()
    for t in path:
        S = S * np.exp(g[t])
        u = beta[t] * (v[t] - S @ k[t])
        S = S + np.outer(u, k[t])
    return S


def verify(parent, q, k, v, g, beta, state, scale=1.0):
    """parent [N, M] ints; q, k [N, M, H, dk]; v [N, M, H, dv]; g [N, M, H]
    or [N, M, H, dk]; beta [N, M, H]; state [N, H, dv, dk].  Returns o [N, M, H, dv] (float64): the
    read-out of every node after the tokens of its root path."""
    parent = np.asarray(parent)
    q, k, v, g, beta, state = map(_f64, (q, k, v, g, beta, state))
    N, M, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((N, M, H, dv))
    for n in range(N):
        for h in range(H):
            for i in range(M):
                S = _run_path(state[n, h], root_path(parent[n], i), k[n, :, h], v[n, :, h],
                              g[n, :, h], beta[n, :, h])
                o[n, i, h] = scale * (S @ q[n, i, h])
    return o


def commit(parent, accepted, k, v, g, beta, state):
    """The state after the root path of node accepted[n] (unchanged for -1),
    for every (n, h).  Returns a new float64 array [N, H, dv, dk]."""
    parent = np.asarray(parent)
    k, v, g, beta, state = map(_f64, (k, v, g, beta, state))
    out = state.copy()
    N, M, H, _ = k.shape
    for n in range(N):
        a = int(accepted[n])
        if a < 0:
            continue
        path = root_path(parent[n], a)
        for h in range(H):
            out[n, h] = _run_path(state[n, h], path, k[n, :, h], v[n, :, h], g[n, :, h],
                                  beta[n, :, h])
    return out
