"""GPU parity of the gated DeltaProduct (gdn_product_fwd / gdn_product_bwd)
against its fp64 oracle (oracle/product.py), over both gates, the tensor-core
path (16-row and whole-head walks) and the fp32 SIMT path, with ragged
sub-token counts."""
import numpy as np
import pytest
import torch

import gated_delta_rule_153_b200 as gdn
from gated_delta_rule_153_b200.inputs import KDA, L350M, TINY, make_product_inputs
from oracle import product
from tests.parity import rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,n,over", [
    (L350M, 3, dict(B=2, H=2, T=50, h0_std=0.1, dhT_std=0.3)),            # 150 sub-tokens
    (L350M, 2, dict(B=3, H=16, T=48, h0_std=0.1, dhT_std=0.3)),           # whole-head walks
    (KDA, 2, dict(B=1, H=2, T=40, h0_std=0.1, dhT_std=0.3, beta_max=2.0)),
    (TINY, 2, dict(B=2, H=3, T=33, dk=32, dv=16, chunk=16, h0_std=0.3, dhT_std=0.5)),  # SIMT fp32
])
def test_product_matches_oracle(dev, cfg, n, over):
    inp = make_product_inputs(cfg, n, **over)
    c = inp["cfg"]
    tol = 1e-4 if c.dtype == "f32" else 2e-2
    d = {k: (inp[k].to(dev) if torch.is_tensor(inp[k]) else None)
         for k in ("q", "k", "v", "g", "beta", "h0", "dO", "dhT")}
    o, hT = gdn.gdn_product_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], chunk=c.chunk)
    r = gdn.gdn_product_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], d["h0"], d["dhT"],
                            chunk=c.chunk)
    torch.cuda.synchronize()
    f = lambda x: None if x is None else x.double().numpy()
    q, k, v, g, beta, h0 = (f(inp[k]) for k in ("q", "k", "v", "g", "beta", "h0"))
    o_ref, hT_ref = product.forward(q, k, v, g, beta, h0)
    ref = product.backward(q, k, v, g, beta, f(inp["dO"]), h0, f(inp["dhT"]))
    errs = {"o": rel_err(o, o_ref), "hT": rel_err(hT, hT_ref)}
    errs.update({k: rel_err(r[k], ref[k]) for k in ("dq", "dk", "dv", "dg", "dbeta", "dh0")})
    bad = {k: e for k, e in errs.items() if not e <= tol}
    assert not bad, f"rel errs over {tol}: {bad} (all: {errs})"


def test_one_step_product_is_the_chunk_call(dev):
    inp = make_product_inputs(L350M, 1, B=1, H=2, T=100, h0_std=0.1)
    d = {k: inp[k].to(dev) for k in ("q", "k", "v", "g", "beta", "h0")}
    o1, h1 = gdn.gdn_product_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    o2, h2 = gdn.gdn_chunk_fwd(d["q"], d["k"][:, :, 0].contiguous(), d["v"][:, :, 0].contiguous(),
                               d["g"], d["beta"][:, :, 0].contiguous(), d["h0"])
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
