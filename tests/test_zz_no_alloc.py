"""gdn_chunk_fwd_noalloc: the forward for callers that cannot call cudaMalloc.

Such callers (a fixed device-memory budget the allocator must not touch, a
runtime without device allocation, host code that must not allocate between
steps) get the same tensor-core forward with its workspace taken from a
64 MiB array built into the library.  These tests call it through the C ABI
and check it against gdn_chunk_fwd, which runs the same kernels on a
caller-provided workspace: the results must be identical bit for bit, so a
wrong offset into the shared array or stale contents left by an earlier call
cannot hide under a tolerance.  One case is also held to the fp64 oracle.
This file is collected last on purpose."""
import ctypes

import pytest
import torch

import gated_delta_rule_153_b200 as gdn
from gated_delta_rule_153_b200.inputs import L350M, make_chunk_inputs
from tests.parity import TOL, oracle_fwd, rel_err

SCRATCH_BYTES = 64 << 20  # the array's documented size


def _dims(B, T, H):
    return gdn.gdn_dims(B, T, H, 128, 128, 64, gdn.GDN_BF16, gdn.GDN_GATE_SCALAR, 1.0)


def _max_chunks(H):
    """Largest ceil(T/64) whose forward workspace fits the array, for B=1 and
    H heads (host-side sizing query only)."""
    L = gdn.lib()
    n = 1
    while L.gdn_chunk_fwd_workspace(ctypes.byref(_dims(1, 64 * (n + 1), H))) <= SCRATCH_BYTES:
        n += 1
    return n


def test_noalloc_rejects_oversize_on_host():
    """One chunk past what fits, the call fails before touching the device."""
    L = gdn.lib()
    p = ctypes.c_void_p(256)
    for H in (1, 4):
        big = _dims(1, 64 * (_max_chunks(H) + 1), H)
        assert L.gdn_chunk_fwd_noalloc(ctypes.byref(big), p, p, p, p, p, None, p, None,
                                       None) == gdn.GDN_ERR_WORKSPACE
    f32 = gdn.gdn_dims(1, 64, 1, 128, 128, 64, gdn.GDN_F32, gdn.GDN_GATE_SCALAR, 1.0)
    assert L.gdn_chunk_fwd_noalloc(ctypes.byref(f32), p, p, p, p, p, None, p, None,
                                   None) == gdn.GDN_ERR_UNSUPPORTED
    bad = _dims(0, 64, 1)
    assert L.gdn_chunk_fwd_noalloc(ctypes.byref(bad), p, p, p, p, p, None, p, None,
                                   None) == gdn.GDN_ERR_INVALID_ARG


def _run_pair(dev, B, T, H, seed, with_h0=True):
    """gdn_chunk_fwd_noalloc and gdn_chunk_fwd on the same inputs."""
    L = gdn.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    inp = make_chunk_inputs(L350M, B=B, T=T, H=H, h0_std=0.05, g_shift=-1.0, seed=seed)
    q, k, v, g, beta, h0 = (inp[n].to(dev) for n in ("q", "k", "v", "g", "beta", "h0"))
    if not with_h0:
        h0 = None
    o = torch.full_like(v, float("nan"))
    hT = torch.full((B, H, 128, 128), float("nan"), device=dev)
    d = _dims(B, T, H)
    st = L.gdn_chunk_fwd_noalloc(ctypes.byref(d), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                 g.data_ptr(), beta.data_ptr(),
                                 h0.data_ptr() if h0 is not None else None, o.data_ptr(),
                                 hT.data_ptr(), stream)
    assert st == gdn.GDN_OK, gdn.status_string(st)
    assert L.gdn_noalloc_device_status(stream) == gdn.GDN_OK
    o_ref, hT_ref = gdn.gdn_chunk_fwd(q, k, v, g, beta, h0, chunk=64)
    torch.cuda.synchronize()
    return inp, o, hT, o_ref, hT_ref


@pytest.mark.gpu
def test_noalloc_matches_chunk_fwd_twice(dev):
    # 8 and 6 heads take the 16-row walk, 48 heads the whole-head tcgen05 walk;
    # two calls in a row on each path
    for i, (seed, (B, T, H)) in enumerate(((11, (2, 1000, 4)), (12, (1, 2048, 6)),
                                           (13, (3, 300, 16)), (14, (3, 500, 16)))):
        inp, o, hT, o_ref, hT_ref = _run_pair(dev, B, T, H, seed)
        assert torch.equal(o, o_ref) and torch.equal(hT, hT_ref), (B, T, H)
        if i == 0:  # tied to the oracle, not only to the other entry point
            o_or, hT_or = oracle_fwd(inp)
            assert rel_err(o, o_or) <= TOL["bf16"]
            assert rel_err(hT, hT_or) <= TOL["bf16"]


@pytest.mark.gpu
def test_noalloc_largest_then_smaller_without_h0(dev):
    """The largest problem that fits the array, then a smaller call with no
    initial state that runs over what the large call left behind."""
    H = 4
    n = _max_chunks(H)
    _, o, hT, o_ref, hT_ref = _run_pair(dev, 1, 64 * n, H, seed=21)
    assert torch.equal(o, o_ref) and torch.equal(hT, hT_ref)
    _, o, hT, o_ref, hT_ref = _run_pair(dev, 2, 700, 3, seed=22, with_h0=False)
    assert torch.equal(o, o_ref) and torch.equal(hT, hT_ref)
