"""fp64 CPU oracle for the gated DeltaProduct -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` may import this module; the CUDA library never uses it.

Source: "DeltaProduct: Improving State-Tracking in Linear RNNs via
Householder Products" (listed by title among the related papers of the
"Linear Attention Architectures: Mechanisms, Trade-offs, and Cross-Layer
Routing" summary page) and the "Gated Delta Networks: Improving Mamba2 with
Delta Rule" review, section "Future work",
which names products of Householder matrices as an extension of the gated
delta rule.  The pages give no equation; the reading taken here: each token t
carries n keys, values and betas, applies its gate once, then performs n
delta-rule steps in order j = 1..n, and is read out after the last:

    S <- S . D_t                                  (D_t = a_t, or Diag(a_t))
    for j = 1..n:  S <- S (I - b_tj k_tj k_tj^T) + b_tj v_tj k_tj^T
    o_t = S (scale q_t)

so the state transition of a token is a_t times a product of n generalised
Householder matrices.  The loop below is that definition, in float64 PyTorch
on the CPU; gradients come from PyTorch's autograd through the same loop
(small cases only).
"""
from __future__ import annotations

import numpy as np
import torch


def _t(x):
    if isinstance(x, torch.Tensor):
        return x if x.dtype == torch.float64 else x.double()
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def forward(q, k, v, g, beta, h0=None, scale=1.0, return_graph=False):
    """q [B,T,H,dk]; k [B,T,n,H,dk]; v [B,T,n,H,dv]; g [B,T,H] or [B,T,H,dk];
    beta [B,T,n,H]; h0 [B,H,dv,dk] or None.  Returns (o [B,T,H,dv], hT)."""
    q, k, v, g, beta = (_t(x) for x in (q, k, v, g, beta))
    B, T, n, H, dk = k.shape
    dv = v.shape[-1]
    S = _t(h0).clone() if h0 is not None else torch.zeros(B, H, dv, dk, dtype=torch.float64)
    channel = g.dim() == 4
    outs = []
    for t in range(T):
        a = torch.exp(g[:, t])
        S = S * (a[:, :, None, :] if channel else a[:, :, None, None])
        for j in range(n):
            kk, vv, bb = k[:, t, j], v[:, t, j], beta[:, t, j]
            p = torch.einsum("bhac,bhc->bha", S, kk)
            u = bb[..., None] * (vv - p)
            S = S + torch.einsum("bha,bhc->bhac", u, kk)
        outs.append(scale * torch.einsum("bhac,bhc->bha", S, q[:, t]))
    o = torch.stack(outs, 1)
    if return_graph:
        return o, S
    return o.numpy(), S.numpy()


def backward(q, k, v, g, beta, dO, h0=None, dhT=None, scale=1.0):
    """Gradients of <dO, o> + <dhT, hT> with respect to every input
    (dq, dk, dv, dg, dbeta and, when h0 is given, dh0), as numpy arrays."""
    leaves = {n: _t(x).requires_grad_(True) for n, x in
              (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta))}
    if h0 is not None:
        leaves["h0"] = _t(h0).requires_grad_(True)
    o, S = forward(leaves["q"], leaves["k"], leaves["v"], leaves["g"], leaves["beta"],
                   leaves.get("h0"), scale, return_graph=True)
    loss = (o * _t(dO)).sum()
    if dhT is not None:
        loss = loss + (S * _t(dhT)).sum()
    loss.backward()
    return {"d" + n: x.grad.numpy() for n, x in leaves.items()}
