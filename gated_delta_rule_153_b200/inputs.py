"""Seeded synthetic inputs for the gated delta-rule layer.

This module only draws random numbers and shapes them; it holds none of the
layer's arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle
consume the same host tensors it returns, so the oracle sees the exact
bf16-rounded values the GPU sees (upcast to fp64).

Distributions follow the workloads the layer is described on (350M..3B-scale
layers of a Gated DeltaNet / Kimi-Delta-Attention stack):

* q, k ~ N(0,1), L2-normalised per token (fp32, eps 1e-6 under the root),
  then cast to the compute dtype -- the block design normalises q and k;
* v ~ N(0,1), not normalised;
* beta = sigmoid(N(0,1));
* log-gate g = -softplus(N(0,1) + shift): shift 0 for the small and the
  long-context workloads, 2 for the 350M-scale and the channel-gate ones,
  and -6 for the "slow gate" cases that keep the inter-chunk state alive;
* optional initial state ~ N(0, std^2) in fp32; dO ~ N(0,1).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


@dataclass(frozen=True)
class ChunkConfig:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: str = "bf16"          # "bf16" or "f32" for q, k, v, o, dO
    gate: str = "scalar"         # "scalar" or "channel"
    g_shift: float = 0.0
    h0_std: Optional[float] = None
    backward: bool = True
    dhT_std: Optional[float] = None
    seed: int = 1000
    beta_max: float = 1.0        # beta = beta_max * sigmoid(N(0,1)); 2 allows I - beta k k^T
                                 # a negative eigenvalue along k


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    N: int
    H: int
    dk: int
    dv: int
    steps: int
    dtype: str = "bf16"
    gate: str = "scalar"
    g_shift: float = 0.0
    state_std: float = 0.02
    seed: int = 1003
    beta_max: float = 1.0


# The five workloads.  Index 0 is the small case the oracle finishes in a
# blink; "same distributions as the small case" is read for the long-context
# and decode workloads (g shift 0).
TINY = ChunkConfig("tiny B1 H1 T64 d16 C16 f32", 1, 64, 1, 16, 16, 16, "f32",
                   "scalar", 0.0, None, False, None, 1000)
L350M = ChunkConfig("350M-layer B8 H8 T2048 d128 C64 bf16", 8, 2048, 8, 128, 128,
                    64, "bf16", "scalar", 2.0, None, True, None, 1001)
LONG = ChunkConfig("long-context B1 H16 T8192 d128 C64 bf16", 1, 8192, 16, 128,
                   128, 64, "bf16", "scalar", 0.0, 0.02, True, 1.0, 1002)
DECODE = DecodeConfig("decode N256 H16 d128 x1000 steps", 256, 16, 128, 128,
                      1000, "bf16", "scalar", 0.0, 0.02, 1003)
KDA = ChunkConfig("kda B2 H32 T4096 d128 C64 bf16 channel-gate", 2, 4096, 32, 128,
                  128, 64, "bf16", "channel", 2.0, None, True, None, 1004)


def _gen(seed: int, idx: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 97 + idx)
    return g


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x * torch.rsqrt((x * x).sum(-1, keepdim=True) + 1e-6)


def make_chunk_inputs(cfg: ChunkConfig, **over) -> dict:
    """Host (CPU) tensors for one chunkwise fwd/bwd call.

    Keyword overrides replace fields of ``cfg`` (e.g. T=100, g_shift=-6).
    Returns q, k, v, dO in the config dtype; g, beta, h0, dhT in fp32."""
    if over:
        cfg = ChunkConfig(**{**cfg.__dict__, **over})
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv
    dt = _DT[cfg.dtype]
    s = cfg.seed
    q = _l2norm(torch.randn(B, T, H, dk, generator=_gen(s, 0))).to(dt)
    k = _l2norm(torch.randn(B, T, H, dk, generator=_gen(s, 1))).to(dt)
    v = torch.randn(B, T, H, dv, generator=_gen(s, 2)).to(dt)
    gshape = (B, T, H, dk) if cfg.gate == "channel" else (B, T, H)
    g = -torch.nn.functional.softplus(
        torch.randn(*gshape, generator=_gen(s, 3)) + cfg.g_shift)
    beta = cfg.beta_max * torch.sigmoid(torch.randn(B, T, H, generator=_gen(s, 4)))
    h0 = None
    if cfg.h0_std is not None:
        h0 = torch.randn(B, H, dv, dk, generator=_gen(s, 5)) * cfg.h0_std
    dO = torch.randn(B, T, H, dv, generator=_gen(s, 6)).to(dt)
    dhT = None
    if cfg.dhT_std is not None:
        dhT = torch.randn(B, H, dv, dk, generator=_gen(s, 7)) * cfg.dhT_std
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
                g=g.contiguous(), beta=beta.contiguous(), h0=h0, dO=dO.contiguous(),
                dhT=dhT, cfg=cfg)


def make_decode_inputs(cfg: DecodeConfig, steps: Optional[int] = None, **over) -> dict:
    """Host tensors for ``steps`` successive single-token updates.
    q, k [steps,N,H,dk], v [steps,N,H,dv] in the config dtype;
    g [steps,N,H] (or [...,dk]), beta [steps,N,H], state0 [N,H,dv,dk] fp32."""
    if over:
        cfg = DecodeConfig(**{**cfg.__dict__, **over})
    S = cfg.steps if steps is None else steps
    N, H, dk, dv = cfg.N, cfg.H, cfg.dk, cfg.dv
    dt = _DT[cfg.dtype]
    s = cfg.seed
    gens = [_gen(s, i) for i in range(6)]
    gshape = (N, H, dk) if cfg.gate == "channel" else (N, H)
    q = torch.empty(S, N, H, dk, dtype=dt)
    k = torch.empty(S, N, H, dk, dtype=dt)
    v = torch.empty(S, N, H, dv, dtype=dt)
    g = torch.empty(S, *gshape)
    beta = torch.empty(S, N, H)
    blk = 25  # steps drawn per block, to bound host memory at full size
    for t0 in range(0, S, blk):
        n = min(blk, S - t0)
        q[t0:t0 + n] = _l2norm(torch.randn(n, N, H, dk, generator=gens[0])).to(dt)
        k[t0:t0 + n] = _l2norm(torch.randn(n, N, H, dk, generator=gens[1])).to(dt)
        v[t0:t0 + n] = torch.randn(n, N, H, dv, generator=gens[2]).to(dt)
        g[t0:t0 + n] = -torch.nn.functional.softplus(
            torch.randn(n, *gshape, generator=gens[3]) + cfg.g_shift)
        beta[t0:t0 + n] = cfg.beta_max * torch.sigmoid(torch.randn(n, N, H, generator=gens[4]))
    state0 = torch.randn(N, H, dv, dk, generator=gens[5]) * cfg.state_std
    return dict(q=q, k=k, v=v, g=g.contiguous(), beta=beta.contiguous(),
                state0=state0, cfg=cfg)


def make_product_inputs(cfg: ChunkConfig, n: int, **over) -> dict:
    """Host tensors for the gated DeltaProduct with n steps per token:
    k, v [B,T,n,H,d] and beta [B,T,n,H] are the n*T-token draw of
    ``make_chunk_inputs`` viewed per token; q, g, h0, dO, dhT come from the
    T-token draw."""
    tok = make_chunk_inputs(cfg, **over)
    c = tok["cfg"]
    sub = make_chunk_inputs(c, T=c.T * n, seed=c.seed + 500)
    B, T, H = c.B, c.T, c.H
    return dict(q=tok["q"], g=tok["g"], h0=tok["h0"], dO=tok["dO"], dhT=tok["dhT"],
                k=sub["k"].reshape(B, T, n, H, c.dk).contiguous(),
                v=sub["v"].reshape(B, T, n, H, c.dv).contiguous(),
                beta=sub["beta"].reshape(B, T, n, H).contiguous(), n=n, cfg=c)


def make_varlen_inputs(cfg: ChunkConfig, lens, **over) -> dict:
    """Host tensors for a packed batch of len(lens) sequences of the given
    token counts: q, k, v, g, beta, dO [1, sum(lens), H, ...] drawn as one
    row, h0 / dhT [len(lens), H, dv, dk] (when the config draws them) and
    cu_seqlens [len(lens) + 1] int32 (0, then the running sums)."""
    lens = [int(n) for n in lens]
    tok = make_chunk_inputs(cfg, B=1, T=max(1, sum(lens)), **over)
    c = tok["cfg"]
    states = make_chunk_inputs(c, B=len(lens), T=1, seed=c.seed + 700)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(torch.int32)
    return dict(tok, h0=states["h0"], dhT=states["dhT"], cu_seqlens=cu, lens=lens)


def tree_parents(N: int, M: int, shape: str = "random", seed: int = 0) -> torch.Tensor:
    """Parent indices [N, M] int32 of draft trees (parent[i] in [-1, i)):
    "random" draws each parent uniformly from -1 .. i-1, "chain" is
    i - 1, "star" is -1 everywhere, "kary4" is the complete 4-ary tree in
    breadth-first order below a root node 0."""
    if shape == "chain":
        p = torch.arange(M) - 1
        return p.repeat(N, 1).to(torch.int32).contiguous()
    if shape == "star":
        return torch.full((N, M), -1, dtype=torch.int32)
    if shape == "kary4":
        p = torch.tensor([-1] + [(i - 1) // 4 for i in range(1, M)])
        return p.repeat(N, 1).to(torch.int32).contiguous()
    gen = _gen(seed, 11)
    u = torch.rand(N, M, generator=gen)
    idx = torch.arange(M)
    return (torch.floor(u * (idx + 1)).to(torch.int64) - 1).to(torch.int32).contiguous()


def make_tree_inputs(N: int, M: int, H: int, shape: str = "random", seed: int = 1200,
                     g_shift: float = 0.0, beta_max: float = 1.0,
                     state_std: float = 0.02, gate: str = "scalar") -> dict:
    """Host tensors for draft-tree verification: q, k [N,M,H,128] and v
    [N,M,H,128] bf16 (q, k L2-normalised), g [N,M,H] (or [N,M,H,128] for the
    channel gate) and beta [N,M,H] fp32 drawn as in make_chunk_inputs, state
    [N,H,128,128] fp32, parent [N,M] int32 and accepted [N] int32 (uniform
    over -1 .. M-1)."""
    cfg = ChunkConfig("tree", N, M, H, 128, 128, 64, "bf16", gate, g_shift, None,
                      False, None, seed, beta_max)
    tok = make_chunk_inputs(cfg)
    state = torch.randn(N, H, 128, 128, generator=_gen(seed, 12)) * state_std
    accepted = (torch.floor(torch.rand(N, generator=_gen(seed, 13)) * (M + 1)) - 1)
    return dict(q=tok["q"], k=tok["k"], v=tok["v"], g=tok["g"], beta=tok["beta"],
                state=state, parent=tree_parents(N, M, shape, seed),
                accepted=accepted.to(torch.int32), N=N, M=M, H=H)


def make_prologue_inputs(B: int, T: int, H: int, d: int = 128, K: int = 4,
                         dtype: str = "bf16", seed: int = 1400) -> dict:
    """Host tensors for the short-conv prologue: projected activations x and
    an upstream gradient dy [B,T,H,d] in ``dtype`` (N(0,1)), filters w
    [H,d,K] fp32 (N(0, 1/K))."""
    dt = _DT[dtype]
    x = torch.randn(B, T, H, d, generator=_gen(seed, 20)).to(dt)
    w = torch.randn(H, d, K, generator=_gen(seed, 21)) / K ** 0.5
    dy = torch.randn(B, T, H, d, generator=_gen(seed, 22)).to(dt)
    return dict(x=x.contiguous(), w=w.contiguous(), dy=dy.contiguous(), dtype=dtype)
