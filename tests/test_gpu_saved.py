"""GPU checks of the training-step pair gdn_chunk_fwd_save / gdn_chunk_bwd_saved.

The saving forward runs the forward's kernels and keeps the chunk products
and chunk-start states; the backward reads them instead of recomputing them.
Both sides compute those quantities with the same kernels in the same order,
so every output must equal the stateless gdn_chunk_fwd / gdn_chunk_bwd pair
bit for bit; one case is also checked against the fp64 oracle."""
import pytest
import torch

import gated_delta_rule_153_b200 as gdn
from gated_delta_rule_153_b200.inputs import KDA, L350M, LONG, TINY, make_chunk_inputs
from tests.parity import TOL, oracle_bwd, oracle_fwd, rel_err, to_dev

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dh0")


def _pair(inp, dev, h0=True):
    cfg = inp["cfg"]
    q, k, v, g, beta, dO = (to_dev(inp[n], dev) for n in ("q", "k", "v", "g", "beta", "dO"))
    h0t = to_dev(inp["h0"], dev) if h0 and inp["h0"] is not None else None
    dhT = to_dev(inp["dhT"], dev)
    o1, hT1 = gdn.gdn_chunk_fwd(q, k, v, g, beta, h0t, chunk=cfg.chunk)
    r1 = gdn.gdn_chunk_bwd(q, k, v, g, beta, dO, h0t, dhT, chunk=cfg.chunk)
    o2, hT2, ws = gdn.gdn_chunk_fwd_save(q, k, v, g, beta, h0t, chunk=cfg.chunk)
    r2 = gdn.gdn_chunk_bwd_saved(q, k, v, g, beta, dO, ws, h0t, dhT, chunk=cfg.chunk)
    torch.cuda.synchronize()
    return (o1, hT1, r1), (o2, hT2, r2)


def _assert_equal(a, b):
    (o1, hT1, r1), (o2, hT2, r2) = a, b
    assert torch.equal(o1, o2), "o"
    assert torch.equal(hT1, hT2), "hT"
    for n in NAMES:
        if r1[n] is None:
            assert r2[n] is None
            continue
        assert torch.equal(r1[n], r2[n]), n


@pytest.mark.parametrize("cfg,over", [
    (L350M, dict(B=3, H=16, T=200, h0_std=0.1, dhT_std=0.3)),        # whole-head walks, tails
    (L350M, dict(B=1, H=3, T=129, h0_std=0.1, dhT_std=0.3)),         # 16-row walks
    (KDA, dict(B=3, H=16, T=130, h0_std=0.1, dhT_std=0.3)),          # channel gate
    (KDA, dict(B=1, H=3, T=100, h0_std=0.1, dhT_std=0.3)),           # channel gate, 16-row
    (L350M, dict(B=1, H=4, T=64 * 40, g_shift=-4.0, dhT_std=0.3)),   # chains cut into runs
    (LONG, dict(H=2, T=64 * 130 - 9, g_shift=-6.0, h0_std=0.1)),     # runs, ragged tail
    (TINY, dict(B=2, H=3, T=77)),                                    # general-shape path
])
def test_saved_pair_equals_stateless_pair(dev, cfg, over):
    inp = make_chunk_inputs(cfg, **over)
    a, b = _pair(inp, dev)
    _assert_equal(a, b)


def test_saved_pair_without_h0(dev):
    inp = make_chunk_inputs(L350M, B=2, H=16, T=150, dhT_std=0.3)
    a, b = _pair(inp, dev, h0=False)
    _assert_equal(a, b)


def test_saved_pair_against_oracle(dev):
    inp = make_chunk_inputs(KDA, B=2, H=16, T=200, h0_std=0.1, dhT_std=0.3)
    _, (o, hT, r) = _pair(inp, dev)
    o_ref, hT_ref = oracle_fwd(inp)
    ref = oracle_bwd(inp)
    tol = TOL[inp["cfg"].dtype]
    assert rel_err(o, o_ref) < tol and rel_err(hT, hT_ref) < tol
    for n in NAMES:
        assert rel_err(r[n], ref[n]) < tol, n


def test_saved_workspace_checks(dev):
    inp = make_chunk_inputs(L350M, B=1, H=2, T=64)
    q, k, v, g, beta, dO = (to_dev(inp[n], dev) for n in ("q", "k", "v", "g", "beta", "dO"))
    small = torch.empty(256, dtype=torch.uint8, device=dev)
    with pytest.raises(ValueError):
        gdn.gdn_chunk_fwd_save(q, k, v, g, beta, workspace=small)
    with pytest.raises(ValueError):
        gdn.gdn_chunk_bwd_saved(q, k, v, g, beta, dO, small)
