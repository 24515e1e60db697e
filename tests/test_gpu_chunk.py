"""GPU parity of gdn_chunk_fwd / gdn_chunk_bwd against the fp64 oracle, on
seeded inputs shaped like the layer's workloads, plus invariants that hold at
any size (chunk-size invariance, resume, Euler identities, determinism)."""
import numpy as np
import pytest
import torch

from gated_delta_rule_153_b200.inputs import KDA, L350M, LONG, TINY, make_chunk_inputs
from tests.parity import TOL, check_bwd, check_fwd, gpu_bwd, gpu_fwd, rel_err

pytestmark = pytest.mark.gpu


# ---- the small fp32 case (tolerance 1e-4) ---------------------------------
def test_tiny_fwd(dev):
    check_fwd(make_chunk_inputs(TINY), dev)


def test_tiny_fwd_bwd_with_states(dev):
    inp = make_chunk_inputs(TINY, h0_std=0.5, dhT_std=1.0)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


@pytest.mark.parametrize("dk,dv,T,C,gate", [
    (16, 16, 1, 16, "scalar"), (16, 32, 7, 16, "scalar"), (32, 16, 100, 32, "channel"),
    (64, 64, 130, 64, "scalar"), (128, 64, 77, 16, "channel"), (128, 128, 200, 64, "scalar"),
    (128, 128, 129, 64, "channel"), (64, 128, 65, 32, "scalar"),
])
def test_f32_shapes_ragged(dev, dk, dv, T, C, gate):
    inp = make_chunk_inputs(TINY, B=2, H=3, T=T, dk=dk, dv=dv, chunk=C, gate=gate,
                            g_shift=-1.0, h0_std=0.3, dhT_std=0.5, seed=77 + T)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


# ---- bf16 at the layer's shapes (tolerance 2e-2) ---------------------------
@pytest.mark.parametrize("dk,dv,T,gate", [(64, 64, 300, "scalar"), (32, 128, 97, "channel")])
def test_bf16_small_dims(dev, dk, dv, T, gate):
    inp = make_chunk_inputs(L350M, B=2, H=2, T=T, dk=dk, dv=dv, gate=gate, h0_std=0.1,
                            dhT_std=0.3, seed=5 + T)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


def test_350m_fwd_bwd(dev):
    inp = make_chunk_inputs(L350M)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


def test_long_context_fwd_bwd(dev):
    inp = make_chunk_inputs(LONG)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


def test_kda_fwd_bwd(dev):
    inp = make_chunk_inputs(KDA, B=1, H=8)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


@pytest.mark.parametrize("cfg,over", [
    (L350M, dict(B=2, g_shift=-6.0, h0_std=0.1, dhT_std=0.5)),
    (LONG, dict(H=4, g_shift=-6.0)),
    (KDA, dict(B=1, H=4, T=1024, g_shift=-6.0, h0_std=0.1)),
])
def test_slow_gate_keeps_state_path_alive(dev, cfg, over):
    """Gates near 1 so the inter-chunk state (and h0) matter for o."""
    inp = make_chunk_inputs(cfg, **over)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


def test_strong_gate_ragged_tail(dev):
    """g near -10 per token: the 8-token tail's gradients are tiny and must not
    be swamped by rounding of the undecayed (i, i) pairs."""
    inp = make_chunk_inputs(L350M, B=2, H=2, T=200, g_shift=10.0, h0_std=0.1, dhT_std=0.3)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


def test_zero_gate_small_beta(dev):
    inp = make_chunk_inputs(L350M, B=1, H=4, T=512, h0_std=0.1)
    inp["g"] = torch.zeros_like(inp["g"])
    inp["beta"] = inp["beta"] * 0.05
    check_fwd(inp, dev)
    check_bwd(inp, dev)


@pytest.mark.parametrize("cfg,over", [
    (L350M, dict(B=3, H=16, T=200, h0_std=0.1, dhT_std=0.3)),             # ragged tail, h0
    (L350M, dict(B=3, H=16, T=72, g_shift=10.0, h0_std=0.1)),             # strong gate, 8-token tails
    (KDA, dict(B=3, H=16, T=200, h0_std=0.1)),
    (KDA, dict(B=3, H=16, T=130, g_shift=10.0, h0_std=0.1)),
    (KDA, dict(B=3, H=16, T=64, g_shift=-6.0, h0_std=0.2)),               # slow gate: the state dominates
])
def test_whole_head_walk(dev, cfg, over):
    """Enough heads for the forward, and the backward's state recompute, to
    carry one whole head per CTA on the fifth-generation tensor cores (state
    in registers, operands in TMEM)."""
    inp = make_chunk_inputs(cfg, **over)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


@pytest.mark.parametrize("cfg,over", [
    (TINY, dict(B=2, H=3, T=77, dk=64, dv=32, chunk=16, h0_std=0.3, dhT_std=0.5)),       # SIMT fp32
    (L350M, dict(B=2, H=2, T=200, h0_std=0.1, dhT_std=0.3)),                           # 16-row walks
    (L350M, dict(B=3, H=16, T=130, h0_std=0.1, dhT_std=0.3)),                          # whole-head walks
    (KDA, dict(B=1, H=4, T=200, h0_std=0.1, dhT_std=0.3)),
    (KDA, dict(B=3, H=16, T=100, h0_std=0.1)),
])
def test_negative_eigenvalue(dev, cfg, over):
    """beta in (0, 2) (negative-eigenvalue transitions): the same kernels, a
    wider input range."""
    inp = make_chunk_inputs(cfg, beta_max=2.0, **over)
    assert float(inp["beta"].max()) > 1.0
    check_fwd(inp, dev)
    check_bwd(inp, dev)


# ---- invariants -----------------------------------------------------------
def test_chunk_size_invariance(dev):
    inp = make_chunk_inputs(L350M, B=1, H=4, T=1000, dtype="f32", g_shift=-2.0, h0_std=0.2)
    outs = [gpu_fwd(inp, dev, chunk=c) for c in (16, 32, 64)]
    for o, hT in outs[1:]:
        assert rel_err(o, outs[0][0].double().cpu().numpy()) < 1e-5
        assert rel_err(hT, outs[0][1].double().cpu().numpy()) < 1e-5


def test_resume_from_final_state(dev):
    inp = make_chunk_inputs(L350M, B=2, H=4, T=768, g_shift=-3.0, h0_std=0.2)
    o_full, h_full = gpu_fwd(inp, dev)
    a = {n: (inp[n][:, :320] if n in ("q", "k", "v", "g", "beta") else inp[n]) for n in inp}
    b = {n: (inp[n][:, 320:] if n in ("q", "k", "v", "g", "beta") else inp[n]) for n in inp}
    a = {n: (x.contiguous() if torch.is_tensor(x) else x) for n, x in a.items()}
    b = {n: (x.contiguous() if torch.is_tensor(x) else x) for n, x in b.items()}
    oa, ha = gpu_fwd(a, dev)
    b["h0"] = ha.cpu()
    ob, hb = gpu_fwd(b, dev)
    o_cat = torch.cat([oa, ob], 1)
    assert rel_err(o_cat, o_full.double().cpu().numpy()) < 2e-2
    assert rel_err(hb, h_full.double().cpu().numpy()) < 2e-2


def test_euler_identities_full_size(dev):
    """o, hT linear in (v, h0) and o linear in q:
    <dv,v> + <dh0,h0> = <dO,o> + <dhT,hT>,  <dq,q> = <dO,o>."""
    inp = make_chunk_inputs(LONG)
    o, hT = gpu_fwd(inp, dev)
    r = gpu_bwd(inp, dev)
    f = lambda x: x.double().cpu()
    dOo = float((f(inp["dO"]) * f(o)).sum())
    rhs = dOo + float((f(inp["dhT"]) * f(hT)).sum())
    lhs = float((f(r["dv"]) * f(inp["v"])).sum() + (f(r["dh0"]) * f(inp["h0"])).sum())
    scale = float(f(inp["dO"]).abs().sum() * f(o).abs().max())
    assert abs(lhs - rhs) <= 2e-2 * scale, (lhs, rhs)
    lq = float((f(r["dq"]) * f(inp["q"])).sum())
    assert abs(lq - dOo) <= 2e-2 * scale, (lq, dOo)


def test_deterministic(dev):
    inp = make_chunk_inputs(L350M, B=2, H=2, T=512)
    o1, h1 = gpu_fwd(inp, dev)
    o2, h2 = gpu_fwd(inp, dev)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    r1, r2 = gpu_bwd(inp, dev), gpu_bwd(inp, dev)
    for n in ("dq", "dk", "dv", "dg", "dbeta"):
        assert torch.equal(r1[n], r2[n]), n


@pytest.mark.parametrize("over", [
    dict(B=2, H=3, T=100, h0_std=0.1, dhT_std=0.3),             # ragged tail, MMA diagonal blocks
    dict(B=1, H=4, T=200, g_shift=10.0, h0_std=0.1),            # spans > 80: exact diagonal blocks
    dict(B=1, H=2, T=64, g_shift=-6.0, h0_std=0.2),             # slow gate, one chunk
    dict(B=3, H=2, T=72, g_shift=4.0, h0_std=0.1),              # 8-token tails next to another sequence
    dict(B=2, H=2, T=200, g_shift=10.0, dhT_std=0.3),           # strong gate: tiny dg in the short tail
])
def test_kda_tensor_core(dev, over):
    """Channel-gate forward and backward through the tensor-core path against the oracle."""
    inp = make_chunk_inputs(KDA, **over)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


def test_status_word_reports_and_clears(dev):
    """A bounded wait that runs out sets the workspace's status word; the
    query reports it once and clears it (the word is preset here: no kernel
    is made to time out)."""
    import gated_delta_rule_153_b200 as gdn
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    assert gdn.gdn_query_device_status(ws) == gdn.GDN_OK
    ws[0] = 1
    assert gdn.gdn_query_device_status(ws) == gdn.GDN_ERR_DEVICE_TIMEOUT
    assert gdn.gdn_query_device_status(ws) == gdn.GDN_OK


@pytest.mark.parametrize("T", [1, 63, 65, 129])
@pytest.mark.parametrize("cfg,over", [
    (L350M, dict(B=1, H=3)),          # 16-row walks
    (L350M, dict(B=3, H=16)),         # whole-head walks
    (KDA, dict(B=1, H=3)),
    (KDA, dict(B=3, H=16)),
])
def test_tensor_core_edge_lengths(dev, T, cfg, over):
    """A single token, one token short of / past a chunk, and past two chunks,
    on both walks and both gates (the tail chunk's padding rows and the
    one-step chains)."""
    inp = make_chunk_inputs(cfg, T=T, h0_std=0.2, dhT_std=0.3, seed=900 + T, **over)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


def test_many_chunks_one_head(dev):
    """256 chunks in one chain (T = 16384, one head, 16-row walks)."""
    inp = make_chunk_inputs(L350M, B=1, H=1, T=16384, g_shift=-3.0, h0_std=0.1, dhT_std=0.2)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


def test_kda_full_size_fwd_bwd(dev):
    """The channel-gate workload at its own size (B=2, H=32, T=4096): 64
    heads take the whole-head tcgen05 walks with the channel gate over
    64-chunk chains, forward, state recompute and reverse walk."""
    inp = make_chunk_inputs(KDA, dhT_std=0.3)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


def test_kda_slow_gate_whole_head_long_chain(dev):
    """Channel gate near 1 (g shift -6) on the whole-head walks over
    16-chunk chains, with h0 and dhT: the inter-chunk path carries the
    signal, so a wrong per-key decay of the state would show."""
    inp = make_chunk_inputs(KDA, T=1024, g_shift=-6.0, h0_std=0.1, dhT_std=0.3)
    check_fwd(inp, dev)
    check_bwd(inp, dev)


def test_walk_wait_runs_out_and_context_survives(dev):
    """A bounded device wait that actually runs out: the tcgen05 forward walk
    is run with the loads of chain step 3 never issued, so the waits on that
    stage (which no copy, MMA or thread completes) give up after 200 us.  The
    call returns, the status word reports the timeout once, and a normal call
    on the same stream afterwards still matches the oracle."""
    import ctypes
    import gated_delta_rule_153_b200 as gdn
    inp = make_chunk_inputs(L350M, B=1, H=40, T=512, h0_std=0.1, seed=31)
    q, k, v, g, beta, h0 = (inp[n].to(dev) for n in ("q", "k", "v", "g", "beta", "h0"))
    dims = gdn.make_dims(q, v, g)
    ws = torch.zeros(gdn.gdn_chunk_fwd_workspace(dims), dtype=torch.uint8, device=dev)
    o = torch.empty_like(v)
    hT = torch.empty(1, 40, 128, 128, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = gdn.lib().gdn_test_stalled_fwd(ctypes.byref(dims), q.data_ptr(), k.data_ptr(),
                                        v.data_ptr(), g.data_ptr(), beta.data_ptr(),
                                        h0.data_ptr(), o.data_ptr(), hT.data_ptr(),
                                        ws.data_ptr(), ws.numel(), 3, 200_000, stream)
    assert st == gdn.GDN_OK, gdn.status_string(st)
    assert gdn.gdn_query_device_status(ws) == gdn.GDN_ERR_DEVICE_TIMEOUT
    assert gdn.gdn_query_device_status(ws) == gdn.GDN_OK
    check_fwd(inp, dev)


@pytest.mark.parametrize("cfg,over", [
    # 6 chains of 43 chunks (runs of 4, the last one shorter); ragged tail, slow gate
    (L350M, dict(B=2, H=3, T=64 * 43 - 17, g_shift=-6.0, h0_std=0.1, dhT_std=0.3)),
    # no initial state: run 0 starts from zero
    (L350M, dict(B=1, H=4, T=64 * 40, g_shift=-4.0, dhT_std=0.3)),
    # one chain cut into the most runs (16), fast and slow gates
    (LONG, dict(H=1, T=64 * 130, g_shift=-6.0)),
    (LONG, dict(H=2, T=64 * 96)),
    # channel gate
    (KDA, dict(B=1, H=4, T=4096, g_shift=-6.0, h0_std=0.1, dhT_std=0.3)),
])
def test_segmented_chains(dev, cfg, over):
    """Few chains: each chain is cut into runs whose affine maps (walked from
    the identity and from zero) are scanned into the runs' entry states, then
    every run is walked from its entry state in parallel.  Slow gates keep the
    state, and so every map and every scan step, in the outputs."""
    inp = make_chunk_inputs(cfg, **over)
    check_fwd(inp, dev)
    check_bwd(inp, dev)
