"""GPU parity of gdn_recurrent_step against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_153_b200 as gdn
from gated_delta_rule_153_b200.inputs import DECODE, L350M, make_chunk_inputs, make_decode_inputs
from tests.parity import rel_err

pytestmark = pytest.mark.gpu


def _run_steps(inp, dev, steps):
    st = inp["state0"].to(dev).contiguous()
    outs = []
    for t in range(steps):
        o = gdn.gdn_recurrent_step(inp["q"][t].to(dev), inp["k"][t].to(dev),
                                   inp["v"][t].to(dev), inp["g"][t].to(dev),
                                   inp["beta"][t].to(dev), st)
        outs.append(o)
    torch.cuda.synchronize()
    return torch.stack(outs), st


@pytest.mark.parametrize("dtype,gate,dk,dv", [
    ("f32", "scalar", 16, 32), ("f32", "channel", 64, 16), ("bf16", "scalar", 128, 128),
    ("bf16", "channel", 128, 64), ("f32", "scalar", 32, 128),
])
def test_decode_small(dev, dtype, gate, dk, dv):
    inp = make_decode_inputs(DECODE, steps=20, N=3, H=5, dk=dk, dv=dv, dtype=dtype, gate=gate)
    o, st = _run_steps(inp, dev, 20)
    s_ref = inp["state0"].double().numpy()
    tol = 1e-4 if dtype == "f32" else 2e-2
    for t in range(20):
        o_ref, s_ref = oracle.step(inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t],
                                   inp["beta"][t], s_ref)
        assert rel_err(o[t], o_ref) <= tol, t
    assert rel_err(st, s_ref) <= tol


def test_decode_full_config_1000_steps(dev):
    """256 sequences x 16 heads, 1000 steps; every output and the final
    states of a sample of (sequence, head) pairs against the oracle, and all
    final states checked finite.  The sample holds the first and the last
    pair, one pair from every block of 16 sequences (so an indexing fault
    confined to high sequence numbers cannot slip through), one pair of every
    head, and 48 seeded random pairs."""
    inp = make_decode_inputs(DECODE)
    S = DECODE.steps
    o, st = _run_steps(inp, dev, S)
    rng = np.random.default_rng(0)
    NH = DECODE.N * DECODE.H
    blocks = [16 * blk + int(rng.integers(16)) for blk in range(DECODE.N // 16)]
    per_block = [n * DECODE.H + int(rng.integers(DECODE.H)) for n in blocks]
    per_head = [int(rng.integers(DECODE.N)) * DECODE.H + h for h in range(DECODE.H)]
    pairs = np.unique(np.concatenate([[0, NH - 1], per_block, per_head,
                                      rng.choice(NH, size=48, replace=False)]))
    n_idx, h_idx = pairs // DECODE.H, pairs % DECODE.H
    sel = lambda x: x[:, n_idx, h_idx][:, :, None]   # [S, P, 1, ...] as N=P, H=1
    q, k, v, g, b = (sel(inp[n]) for n in ("q", "k", "v", "g", "beta"))
    s_ref = inp["state0"][n_idx, h_idx][:, None].double().numpy()
    o_ref = np.zeros((S, len(pairs), 1, DECODE.dv))
    for t in range(S):
        o_ref[t], s_ref = oracle.step(q[t], k[t], v[t], g[t], b[t], s_ref)
    o_gpu = o[:, n_idx, h_idx][:, :, None]
    assert rel_err(o_gpu, o_ref) <= 2e-2
    assert rel_err(st[n_idx, h_idx][:, None], s_ref) <= 2e-2
    assert torch.isfinite(st).all()


def test_decode_matches_chunk_fwd(dev):
    """T successive decode steps == the chunkwise forward over T tokens."""
    inp = make_chunk_inputs(L350M, B=4, H=3, T=50, g_shift=-2.0, h0_std=0.2, dtype="f32")
    q, k, v, g, b = (inp[n].to(dev) for n in ("q", "k", "v", "g", "beta"))
    h0 = inp["h0"].to(dev)
    o_chunk, hT = gdn.gdn_chunk_fwd(q, k, v, g, b, h0, chunk=16)
    st = h0.clone()
    outs = [gdn.gdn_recurrent_step(q[:, t].contiguous(), k[:, t].contiguous(),
                                   v[:, t].contiguous(), g[:, t].contiguous(),
                                   b[:, t].contiguous(), st) for t in range(50)]
    o_dec = torch.stack(outs, 1)
    torch.cuda.synchronize()
    assert rel_err(o_dec, o_chunk.double().cpu().numpy()) < 1e-4
    assert rel_err(st, hT.double().cpu().numpy()) < 1e-4


@pytest.mark.parametrize("dtype,gate", [("f32", "scalar"), ("bf16", "channel")])
def test_decode_negative_eigenvalue(dev, dtype, gate):
    """beta in (0, 2): I - beta k k^T may flip the sign along k."""
    inp = make_decode_inputs(DECODE, steps=20, N=3, H=5, dk=128, dv=128, dtype=dtype, gate=gate,
                             beta_max=2.0)
    assert float(inp["beta"].max()) > 1.0
    o, st = _run_steps(inp, dev, 20)
    s_ref = inp["state0"].double().numpy()
    tol = 1e-4 if dtype == "f32" else 2e-2
    for t in range(20):
        o_ref, s_ref = oracle.step(inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t],
                                   inp["beta"][t], s_ref)
        assert rel_err(o[t], o_ref) <= tol, t
    assert rel_err(st, s_ref) <= tol
