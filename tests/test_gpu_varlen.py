"""GPU parity of the packed variable-length calls (gdn_chunk_fwd_varlen /
gdn_chunk_bwd_varlen) against the fp64 oracle run on each sequence alone:
every sequence of a packed batch is its own instance of the recurrence, so
its outputs and gradients must match the oracle on that sequence, with its
own initial state, whatever sits next to it in memory."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_153_b200 as gdn
from gated_delta_rule_153_b200.inputs import KDA, L350M, make_varlen_inputs
from tests.parity import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu

# Lengths 0 and 1, a chunk and a chunk plus one, ragged tails, two empty
# sequences (one first, one inside the batch).
LENS = [0, 1, 65, 64, 130, 7, 300, 0, 200, 63]


def _seq(x, a, b):
    return x[:, a:b]


def oracle_varlen(inp, want_bwd):
    """Per-sequence oracle results, concatenated back into the packed layout."""
    cu = inp["cu_seqlens"].tolist()
    H, dk, dv = inp["cfg"].H, inp["cfg"].dk, inp["cfg"].dv
    h0, dhT = inp["h0"], inp["dhT"]
    os, hTs = [], []
    grads = {n: [] for n in ("dq", "dk", "dv", "dg", "dbeta")}
    dh0s = []
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        h0s = None if h0 is None else h0[s:s + 1]
        dhs = None if dhT is None else dhT[s:s + 1]
        if a == b:  # empty: the state passes through
            hTs.append(np.zeros((1, H, dv, dk)) if h0s is None else h0s.double().numpy())
            dh0s.append(np.zeros((1, H, dv, dk)) if dhs is None else dhs.double().numpy())
            continue
        args = [_seq(inp[n], a, b) for n in ("q", "k", "v", "g", "beta")]
        o, hT = oracle.fwd(*args, h0s)
        os.append(o)
        hTs.append(hT)
        if want_bwd:
            r = oracle.bwd(*args, _seq(inp["dO"], a, b), h0s, dhs)
            for n in grads:
                grads[n].append(r[n])
            dh0s.append(r["dh0"])
    out = dict(o=np.concatenate(os, 1), hT=np.concatenate(hTs, 0))
    if want_bwd:
        out.update({n: np.concatenate(x, 1) for n, x in grads.items()})
        out["dh0"] = np.concatenate(dh0s, 0)
    return out


def gpu_varlen(inp, dev, want_bwd, h0=True):
    q, k, v, g, beta, dO, cu = (to_dev(inp[n], dev) for n in
                                ("q", "k", "v", "g", "beta", "dO", "cu_seqlens"))
    h0t = to_dev(inp["h0"], dev) if h0 else None
    dhT = to_dev(inp["dhT"], dev)
    o, hT = gdn.gdn_chunk_fwd_varlen(q, k, v, g, beta, cu, h0t)
    out = dict(o=o, hT=hT)
    if want_bwd:
        out.update(gdn.gdn_chunk_bwd_varlen(q, k, v, g, beta, cu, dO, h0t, dhT))
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("cfg,H", [(L350M, 2), (L350M, 4), (KDA, 2), (KDA, 4)])
def test_varlen_matches_per_sequence_oracle(dev, cfg, H):
    """H = 2: 20 chains, the 16-row walks; H = 4: 40 chains, the whole-head walks."""
    inp = make_varlen_inputs(cfg, LENS, H=H, g_shift=-1.0, h0_std=0.1, dhT_std=0.3,
                             seed=40 + H)
    got = gpu_varlen(inp, dev, True)
    ref = oracle_varlen(inp, True)
    tol = TOL["bf16"]
    errs = {n: rel_err(got[n], ref[n]) for n in ref}
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, f"rel errs over {tol}: {bad} (all: {errs})"


def test_varlen_without_initial_state(dev):
    inp = make_varlen_inputs(L350M, [129, 0, 3, 64], H=4, h0_std=None, dhT_std=0.3, seed=9)
    got = gpu_varlen(inp, dev, True, h0=True)
    ref = oracle_varlen(inp, True)
    for n in ("o", "hT", "dq", "dk", "dv", "dg", "dbeta"):
        assert rel_err(got[n], ref[n]) <= TOL["bf16"], n
    assert got["dh0"] is None


@pytest.mark.parametrize("cfg", [L350M, KDA])
def test_equal_lengths_match_batched_call(dev, cfg):
    """B sequences of T tokens packed with cu = 0, T, 2T, ... run the same
    per-chunk arithmetic as the batched call: the results agree bit for bit."""
    B, T, H = 3, 200, 16
    inp = make_varlen_inputs(cfg, [T] * B, H=H, h0_std=0.1, dhT_std=0.3, seed=3)
    got = gpu_varlen(inp, dev, True)
    bat = {n: to_dev(inp[n], dev).reshape(B, T, *inp[n].shape[2:])
           for n in ("q", "k", "v", "g", "beta", "dO")}
    h0, dhT = to_dev(inp["h0"], dev), to_dev(inp["dhT"], dev)
    o, hT = gdn.gdn_chunk_fwd(bat["q"], bat["k"], bat["v"], bat["g"], bat["beta"], h0)
    r = gdn.gdn_chunk_bwd(bat["q"], bat["k"], bat["v"], bat["g"], bat["beta"], bat["dO"],
                          h0, dhT)
    torch.cuda.synchronize()
    assert torch.equal(got["o"].reshape(o.shape), o)
    assert torch.equal(got["hT"], hT)
    for n in ("dq", "dk", "dv", "dg", "dbeta"):
        assert torch.equal(got[n].reshape(r[n].shape), r[n]), n
    assert torch.equal(got["dh0"], r["dh0"])


def test_invalid_offsets_reported(dev):
    """Offsets that decrease: the call returns, no chunk runs, and the status
    query on its workspace reports GDN_ERR_INVALID_ARG (then GDN_OK once read)."""
    inp = make_varlen_inputs(L350M, [40, 30, 50], H=2, h0_std=0.1, seed=5)
    cu = to_dev(torch.tensor([0, 40, 20, 120], dtype=torch.int32), dev)
    q, k, v, g, beta = (to_dev(inp[n], dev) for n in ("q", "k", "v", "g", "beta"))
    h0 = to_dev(inp["h0"], dev)
    d = gdn.make_dims(q, v, g)
    ws = torch.empty(gdn.lib().gdn_chunk_fwd_varlen_workspace(__import__("ctypes").byref(d), 3),
                     dtype=torch.uint8, device=dev)
    gdn.gdn_chunk_fwd_varlen(q, k, v, g, beta, cu, h0, workspace=ws)
    assert gdn.gdn_query_device_status(ws) == gdn.GDN_ERR_INVALID_ARG
    assert gdn.gdn_query_device_status(ws) == gdn.GDN_OK
    # a valid call on the same workspace is clean
    gdn.gdn_chunk_fwd_varlen(q, k, v, g, beta, to_dev(inp["cu_seqlens"], dev), h0, workspace=ws)
    assert gdn.gdn_query_device_status(ws) == gdn.GDN_OK
