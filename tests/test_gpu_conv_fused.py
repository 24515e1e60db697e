"""GPU parity of the training pair with the q/k/v prologue fused into the chunk
preparation (gdn_chunk_fwd_save_conv / gdn_chunk_bwd_saved_conv) against the
fp64 oracle: the oracle prologue on the raw projections, then the oracle
chunk forward and backward, and the prologue's backward on the resulting
q, k, v gradients.  Also: the fused pair against the same computation run as
separate GPU passes, and the paths that keep the prologue as its own pass."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_153_b200 as gdn
from gated_delta_rule_153_b200.inputs import KDA, L350M, make_chunk_inputs, make_prologue_inputs
from oracle import prologue as pro_oracle
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu


def _inputs(cfg, K=4, seed=7, **over):
    inp = make_chunk_inputs(cfg, seed=seed, **over)
    c = inp["cfg"]
    pro = {n: make_prologue_inputs(c.B, c.T, c.H, c.dk, K, c.dtype, seed=seed + 10 * i)
           for i, n in enumerate(("q", "k", "v"))}
    inp["x"] = {n: pro[n]["x"] for n in pro}
    inp["w"] = {n: pro[n]["w"] for n in pro}
    return inp


def _oracle(inp):
    """fp64 reference: prologue, chunk forward and backward, prologue backward."""
    x, w = inp["x"], inp["w"]
    f = {n: pro_oracle.forward(x[n], w[n], n != "v") for n in ("q", "k", "v")}
    t = {n: torch.from_numpy(f[n]) for n in f}
    o, hT = oracle.fwd(t["q"], t["k"], t["v"], inp["g"], inp["beta"], inp["h0"])
    r = oracle.bwd(t["q"], t["k"], t["v"], inp["g"], inp["beta"], inp["dO"], inp["h0"], inp["dhT"])
    out = {"o": o, "hT": hT, "dg": r["dg"], "dbeta": r["dbeta"]}
    if inp["h0"] is not None:
        out["dh0"] = r["dh0"]
    for n in ("q", "k", "v"):
        gb = pro_oracle.backward(x[n], w[n], r["d" + n], n != "v")
        out["dx" + n], out["dw" + n] = gb["dx"], gb["dw"]
    return out


def _fused(inp, dev):
    d = lambda t: None if t is None else t.to(dev).contiguous()
    x = {n: d(inp["x"][n]) for n in ("q", "k", "v")}
    w = {n: d(inp["w"][n]) for n in ("q", "k", "v")}
    g, beta, h0, dO, dhT = (d(inp[n]) for n in ("g", "beta", "h0", "dO", "dhT"))
    o, hT, ws = gdn.gdn_chunk_fwd_save_conv(x["q"], x["k"], x["v"], w["q"], w["k"], w["v"], g, beta, h0)
    r = gdn.gdn_chunk_bwd_saved_conv(x["q"], x["k"], x["v"], w["q"], w["k"], w["v"], g, beta, dO, ws,
                                     h0, dhT)
    torch.cuda.synchronize()
    out = {"o": o, "hT": hT, "dg": r["dg"], "dbeta": r["dbeta"]}
    if h0 is not None:
        out["dh0"] = r["dh0"]
    for n in ("q", "k", "v"):
        out["dx" + n], out["dw" + n] = r["dx" + n], r["dw" + n]
    return out


def _check(got, ref, tol):
    errs = {n: rel_err(got[n], ref[n]) for n in ref}
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, f"rel errs over {tol}: {bad} (all {errs})"


@pytest.mark.parametrize("cfg,over,K", [
    (L350M, dict(B=2, H=16, T=200, h0_std=0.1, dhT_std=0.3), 4),   # whole-head walks, tails
    (L350M, dict(B=1, H=3, T=129, h0_std=0.1, dhT_std=0.3), 3),    # 16-row walks
    (L350M, dict(B=3, H=16, T=64, dhT_std=0.3), 1),                # one chunk per sequence
    (L350M, dict(B=2, H=4, T=1000, g_shift=-3.0, dhT_std=0.3), 2),  # chains cut into runs
    (KDA, dict(B=2, H=16, T=130, h0_std=0.1, dhT_std=0.3), 4),     # prologue as its own pass
])
def test_fused_pair_matches_oracle(dev, cfg, over, K):
    inp = _inputs(cfg, K=K, **over)
    _check(_fused(inp, dev), _oracle(inp), TOL[inp["cfg"].dtype])


def test_fused_pair_at_350m_shape(dev):
    inp = _inputs(L350M, K=4)
    _check(_fused(inp, dev), _oracle(inp), TOL[inp["cfg"].dtype])


def test_fused_pair_matches_separate_passes(dev):
    """The fused preparation against the prologue run as its own GPU pass
    (same filter arithmetic, so the results agree to bf16 rounding)."""
    inp = _inputs(L350M, K=4, B=2, H=16, T=300, h0_std=0.1, dhT_std=0.3)
    got = _fused(inp, dev)
    d = lambda t: None if t is None else t.to(dev).contiguous()
    f = {n: gdn.gdn_short_conv_fwd(d(inp["x"][n]), d(inp["w"][n]), l2norm=n != "v") for n in ("q", "k", "v")}
    g, beta, h0, dO, dhT = (d(inp[n]) for n in ("g", "beta", "h0", "dO", "dhT"))
    o, hT, ws = gdn.gdn_chunk_fwd_save(f["q"], f["k"], f["v"], g, beta, h0)
    r = gdn.gdn_chunk_bwd_saved(f["q"], f["k"], f["v"], g, beta, dO, ws, h0, dhT)
    torch.cuda.synchronize()
    assert rel_err(got["o"], o.double().cpu().numpy()) < 2e-2
    assert rel_err(got["hT"], hT.double().cpu().numpy()) < 1e-2
    for n in ("q", "k", "v"):
        dx, dw = gdn.gdn_short_conv_bwd(d(inp["x"][n]), d(inp["w"][n]), r["d" + n], l2norm=n != "v")
        assert rel_err(got["dx" + n], dx.double().cpu().numpy()) < 2e-2, n
        assert rel_err(got["dw" + n], dw.double().cpu().numpy()) < 2e-2, n


def test_fused_workspace_checks(dev):
    inp = _inputs(L350M, K=4, B=1, H=2, T=64)
    d = lambda t: t.to(dev).contiguous()
    x = {n: d(inp["x"][n]) for n in ("q", "k", "v")}
    w = {n: d(inp["w"][n]) for n in ("q", "k", "v")}
    small = torch.empty(256, dtype=torch.uint8, device=dev)
    with pytest.raises(ValueError):
        gdn.gdn_chunk_fwd_save_conv(x["q"], x["k"], x["v"], w["q"], w["k"], w["v"], d(inp["g"]),
                                    d(inp["beta"]), workspace=small)
