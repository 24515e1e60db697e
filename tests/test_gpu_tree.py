"""GPU parity of draft-tree verification and commit (gdn_tree_verify /
gdn_tree_commit) against the fp64 tree oracle, plus agreement with the
chunkwise forward on chains and with the decode step on stars."""
import numpy as np
import pytest
import torch

import gated_delta_rule_153_b200 as gdn
from gated_delta_rule_153_b200.inputs import make_tree_inputs
from oracle import tree as tree_oracle
from tests.parity import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _dev(inp, dev):
    return {n: to_dev(inp[n], dev) for n in
            ("q", "k", "v", "g", "beta", "state", "parent", "accepted")}


def _verify(d, scale=1.0, status=None):
    o = gdn.gdn_tree_verify(d["parent"], d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                            scale=scale, status=status)
    torch.cuda.synchronize()
    return o


@pytest.mark.parametrize("M", [1, 5, 16, 17, 33, 48, 64])
@pytest.mark.parametrize("shape", ["random", "kary4"])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_verify_matches_oracle(dev, M, shape, gate):
    inp = make_tree_inputs(3, M, 4, shape=shape, seed=1200 + M, g_shift=-1.0, state_std=0.05,
                           gate=gate)
    o = _verify(_dev(inp, dev), scale=0.9)
    ref = tree_oracle.verify(inp["parent"].numpy(), inp["q"], inp["k"], inp["v"], inp["g"],
                             inp["beta"], inp["state"], scale=0.9)
    e = rel_err(o, ref)
    assert e <= TOL["bf16"], f"o rel err {e:.3e}"


@pytest.mark.parametrize("M", [1, 7, 64])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_commit_matches_oracle(dev, M, gate):
    """fp32 recurrent form along the accepted path: held to the fp32 bar."""
    inp = make_tree_inputs(6, M, 3, seed=1300 + M, g_shift=-1.0, state_std=0.05, gate=gate)
    inp["accepted"][0] = -1
    inp["accepted"][1] = M - 1
    d = _dev(inp, dev)
    before = d["state"].clone()
    gdn.gdn_tree_commit(d["parent"], d["accepted"], d["k"], d["v"], d["g"], d["beta"],
                        d["state"])
    torch.cuda.synchronize()
    ref = tree_oracle.commit(inp["parent"].numpy(), inp["accepted"].numpy(), inp["k"],
                             inp["v"], inp["g"], inp["beta"], inp["state"])
    e = rel_err(d["state"], ref)
    assert e <= TOL["f32"], f"state rel err {e:.3e}"
    assert torch.equal(d["state"][0], before[0])  # nothing accepted: untouched


def test_chain_equals_chunkwise_forward(dev):
    """A 64-node chain is one 64-token chunk: the tree outputs and the
    committed state agree with gdn_chunk_fwd from the same state."""
    inp = make_tree_inputs(4, 64, 8, shape="chain", seed=21, g_shift=-2.0, state_std=0.05)
    inp["accepted"][:] = 63
    d = _dev(inp, dev)
    o = _verify(d)
    o2, hT = gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"])
    torch.cuda.synchronize()
    assert rel_err(o, o2.double().cpu().numpy()) <= TOL["bf16"]
    gdn.gdn_tree_commit(d["parent"], d["accepted"], d["k"], d["v"], d["g"], d["beta"],
                        d["state"])
    torch.cuda.synchronize()
    assert rel_err(d["state"], hT.double().cpu().numpy()) <= TOL["bf16"]


def test_star_equals_decode_steps(dev):
    """Parents all -1: node i is one decode step from the committed state."""
    inp = make_tree_inputs(2, 12, 4, shape="star", seed=22, state_std=0.05)
    d = _dev(inp, dev)
    o = _verify(d, scale=1.1)
    for i in range(12):
        st = d["state"].clone()
        oi = gdn.gdn_recurrent_step(d["q"][:, i].contiguous(), d["k"][:, i].contiguous(),
                                    d["v"][:, i].contiguous(), d["g"][:, i].contiguous(),
                                    d["beta"][:, i].contiguous(), st, scale=1.1)
        torch.cuda.synchronize()
        assert rel_err(o[:, i], oi.double().cpu().numpy()) <= TOL["bf16"], i


def test_verify_leaves_state_and_is_deterministic(dev):
    inp = make_tree_inputs(2, 40, 4, seed=23)
    d = _dev(inp, dev)
    before = d["state"].clone()
    o1 = _verify(d)
    o2 = _verify(d)
    assert torch.equal(d["state"], before)
    assert torch.equal(o1, o2)


def test_invalid_tree_indices_are_reported(dev):
    """A parent that is not earlier in the order reads as -1, an accepted index
    out of range as -1; both raise the status word to GDN_ERR_INVALID_ARG."""
    inp = make_tree_inputs(2, 10, 2, seed=24, state_std=0.05)
    inp["parent"][1, 4] = 7  # not before node 4
    d = _dev(inp, dev)
    status = torch.zeros(64, dtype=torch.int32, device=dev)
    o = _verify(d, status=status)
    fixed = inp["parent"].clone()
    fixed[1, 4] = -1
    ref = tree_oracle.verify(fixed.numpy(), inp["q"], inp["k"], inp["v"], inp["g"],
                             inp["beta"], inp["state"])
    assert rel_err(o, ref) <= TOL["bf16"]
    assert gdn.gdn_query_device_status(status) == gdn.GDN_ERR_INVALID_ARG
    assert gdn.gdn_query_device_status(status) == gdn.GDN_OK
    acc = torch.tensor([10, -1], dtype=torch.int32, device=dev)
    before = d["state"].clone()
    d["parent"][1, 4] = -1
    gdn.gdn_tree_commit(d["parent"], acc, d["k"], d["v"], d["g"], d["beta"], d["state"],
                        status=status)
    assert gdn.gdn_query_device_status(status) == gdn.GDN_ERR_INVALID_ARG
    assert torch.equal(d["state"], before)


def test_channel_gate_chain_equals_chunkwise_forward(dev):
    """Channel gate: a 64-node chain agrees with gdn_chunk_fwd from the same
    state, the decays acting per key."""
    inp = make_tree_inputs(2, 64, 4, shape="chain", seed=23, g_shift=-2.0, state_std=0.05,
                           gate="channel")
    d = _dev(inp, dev)
    o = _verify(d)
    q, k, v, g, beta = (d[n].contiguous() for n in ("q", "k", "v", "g", "beta"))
    o2, _ = gdn.gdn_chunk_fwd(q, k, v, g, beta, d["state"])
    torch.cuda.synchronize()
    assert rel_err(o, o2.double().cpu().numpy()) < 2e-2
