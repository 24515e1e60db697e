"""gdn_chunk_fwd_noalloc: the forward for callers that cannot call cudaMalloc.

Such callers (a fixed device-memory budget the allocator must not touch, a
runtime without device allocation, host code that must not allocate between
steps) get the same tensor-core forward with its workspace taken from a
64 MiB array built into the library.  These tests call it through the C ABI
and check it against gdn_chunk_fwd, which takes a caller-provided workspace.
This file is collected last on purpose."""
import ctypes

import pytest
import torch

import gated_delta_rule_153_b200 as gdn
from gated_delta_rule_153_b200.inputs import L350M, make_chunk_inputs
from tests.parity import rel_err


def _dims(B, T, H):
    return gdn.gdn_dims(B, T, H, 128, 128, 64, gdn.GDN_BF16, gdn.GDN_GATE_SCALAR, 1.0)


def test_noalloc_rejects_oversize_on_host():
    """Beyond 1628 chunk-heads the call fails before touching the device."""
    L = gdn.lib()
    p = ctypes.c_void_p(256)
    big = _dims(1, 64 * 1629, 1)      # 1629 chunk-heads
    assert L.gdn_chunk_fwd_noalloc(ctypes.byref(big), p, p, p, p, p, None, p, None,
                                   None) == gdn.GDN_ERR_WORKSPACE
    f32 = gdn.gdn_dims(1, 64, 1, 128, 128, 64, gdn.GDN_F32, gdn.GDN_GATE_SCALAR, 1.0)
    assert L.gdn_chunk_fwd_noalloc(ctypes.byref(f32), p, p, p, p, p, None, p, None,
                                   None) == gdn.GDN_ERR_UNSUPPORTED
    bad = _dims(0, 64, 1)
    assert L.gdn_chunk_fwd_noalloc(ctypes.byref(bad), p, p, p, p, p, None, p, None,
                                   None) == gdn.GDN_ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_matches_chunk_fwd_twice(dev):
    L = gdn.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # 8 and 6 heads take the 16-row walk, 48 heads the whole-head tcgen05 walk
    for seed, (B, T, H) in ((11, (2, 1000, 4)), (12, (1, 2048, 6)), (13, (3, 300, 16))):
        inp = make_chunk_inputs(L350M, B=B, T=T, H=H, h0_std=0.05, g_shift=-1.0, seed=seed)
        q, k, v, g, beta, h0 = (inp[n].to(dev) for n in ("q", "k", "v", "g", "beta", "h0"))
        o_ref, hT_ref = gdn.gdn_chunk_fwd(q, k, v, g, beta, h0, chunk=64)
        o = torch.full_like(o_ref, float("nan"))
        hT = torch.full_like(hT_ref, float("nan"))
        d = _dims(B, T, H)
        st = L.gdn_chunk_fwd_noalloc(ctypes.byref(d), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                     g.data_ptr(), beta.data_ptr(), h0.data_ptr(), o.data_ptr(),
                                     hT.data_ptr(), stream)
        assert st == gdn.GDN_OK, gdn.status_string(st)
        torch.cuda.synchronize()
        assert rel_err(o, o_ref.double().cpu().numpy()) <= 2e-2
        assert rel_err(hT, hT_ref.double().cpu().numpy()) <= 2e-2
