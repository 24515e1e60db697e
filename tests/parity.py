"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding and the fp64 oracle on the same host tensors, and compare them with
the metric the tolerances are stated in: max|gpu - ref| / max|ref| per tensor.

Tolerances: 1e-4 when q/k/v are fp32, 2e-2 when they are bf16 (outputs stored
in bf16 are compared as stored)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import gated_delta_rule_153_b200 as gdn

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(gpu, ref) -> float:
    g = gpu.detach().double().cpu().numpy() if torch.is_tensor(gpu) else np.asarray(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "non-finite values in GPU output"
    den = float(np.max(np.abs(r)))
    num = float(np.max(np.abs(g - r)))
    return num / den if den > 0 else num


def to_dev(x, dev):
    return None if x is None else x.to(dev).contiguous()


def gpu_fwd(inp, dev, chunk=None, poison=True, h0=True):
    cfg = inp["cfg"]
    q, k, v, g, beta = (to_dev(inp[n], dev) for n in ("q", "k", "v", "g", "beta"))
    h0t = to_dev(inp["h0"], dev) if h0 else None
    o = torch.full_like(v, float("nan")) if poison else None
    hT = torch.full((cfg.B, cfg.H, cfg.dv, cfg.dk), float("nan"), device=dev) if poison else None
    o, hT = gdn.gdn_chunk_fwd(q, k, v, g, beta, h0t, chunk=chunk or cfg.chunk, o=o, hT=hT)
    torch.cuda.synchronize()
    return o, hT


def gpu_bwd(inp, dev, chunk=None, h0=True):
    cfg = inp["cfg"]
    q, k, v, g, beta, dO = (to_dev(inp[n], dev) for n in ("q", "k", "v", "g", "beta", "dO"))
    h0t = to_dev(inp["h0"], dev) if h0 else None
    dhT = to_dev(inp["dhT"], dev)
    r = gdn.gdn_chunk_bwd(q, k, v, g, beta, dO, h0t, dhT, chunk=chunk or cfg.chunk)
    torch.cuda.synchronize()
    return r


def oracle_fwd(inp, h0=True):
    return oracle.fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                      inp["h0"] if h0 else None)


def oracle_bwd(inp, h0=True):
    return oracle.bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["dO"],
                      inp["h0"] if h0 else None, inp["dhT"])


def check_fwd(inp, dev, chunk=None, tol=None, h0=True):
    cfg = inp["cfg"]
    tol = tol or TOL[cfg.dtype]
    o, hT = gpu_fwd(inp, dev, chunk, h0=h0)
    o_ref, hT_ref = oracle_fwd(inp, h0)
    eo, eh = rel_err(o, o_ref), rel_err(hT, hT_ref)
    assert eo <= tol, f"o rel err {eo:.3e} > {tol}"
    assert eh <= tol, f"hT rel err {eh:.3e} > {tol}"
    return eo, eh


def check_bwd(inp, dev, chunk=None, tol=None, h0=True):
    cfg = inp["cfg"]
    tol = tol or TOL[cfg.dtype]
    r = gpu_bwd(inp, dev, chunk, h0=h0)
    ref = oracle_bwd(inp, h0)
    errs = {}
    for n in ("dq", "dk", "dv", "dg", "dbeta") + (("dh0",) if (h0 and inp["h0"] is not None) else ()):
        errs[n] = rel_err(r[n], ref[n])
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, f"bwd rel errs over {tol}: {bad} (all: {errs})"
    return errs
