"""fp64 CPU oracle for the q/k/v prologue of the layer -- TEST INFRASTRUCTURE
ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
may import this module; the CUDA library never uses it.

Source: "Gated Delta Networks: Improving Mamba2 with Delta Rule" (paper
review), section "Method": in the block design q and k pass through a linear
projection, a short convolution and SiLU, then L2 normalisation; v takes the
same path without the L2 norm.  The projection is an ordinary GEMM outside
this path.  Readings where the page is silent:

* "short convolution" is causal and depthwise (one filter of K taps per
  channel, no bias), over the tokens of each sequence, with zeros before the
  first token:  z_t[c] = sum_{j<K} w[c, j] x_{t-j}[c];
* SiLU(z) = z * sigmoid(z), elementwise;
* the L2 norm runs over the d channels of one head, with eps = 1e-6 under the
  square root:  y = s / sqrt(sum_c s_c^2 + eps).

The function below is that definition in float64 PyTorch on the CPU, with an
explicit loop over the taps; gradients come from autograd through it.
"""
from __future__ import annotations

import numpy as np
import torch

EPS = 1e-6


def _t(x):
    if isinstance(x, torch.Tensor):
        return x if x.dtype == torch.float64 else x.detach().double()
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def forward(x, w, norm, return_graph=False):
    """x [B, T, H, d]; w [H, d, K]; norm: L2-normalise each head's d channels.
    Returns y [B, T, H, d]."""
    x, w = _t(x), _t(w)
    B, T, H, d = x.shape
    K = w.shape[-1]
    z = torch.zeros_like(x)
    for j in range(K):  # tap j reads the token j steps back
        if j < T:
            z[:, j:] = z[:, j:] + w[:, :, j] * x[:, :T - j]
    s = z * torch.sigmoid(z)
    y = s / torch.sqrt((s * s).sum(-1, keepdim=True) + EPS) if norm else s
    return y if return_graph else y.numpy()


def backward(x, w, dy, norm):
    """Gradients of <dy, y> with respect to x and w, as numpy arrays."""
    xl = _t(x).clone().requires_grad_(True)
    wl = _t(w).clone().requires_grad_(True)
    y = forward(xl, wl, norm, return_graph=True)
    (y * _t(dy)).sum().backward()
    return {"dx": xl.grad.numpy(), "dw": wl.grad.numpy()}
