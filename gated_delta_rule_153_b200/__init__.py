"""Python binding of libgdn.so, the sm_100a gated delta-rule library.

Argument marshalling only: every function below checks tensor shapes, dtypes
and devices, allocates outputs with torch (device memory is torch's job),
and calls the C entry point of the same name through ctypes on the current
CUDA stream.  No arithmetic of the layer happens in Python, and there is no
CPU fallback: if the compiled library is missing, the first call raises.

Layouts follow the C ABI (include/gdn.h): q, k [B,T,H,dk]; v, o [B,T,H,dv];
g [B,T,H] (scalar gate) or [B,T,H,dk] (channel gate) fp32; beta [B,T,H] fp32;
states [B,H,dv,dk] fp32.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE, GDN_ERR_CUDA, \
    GDN_ERR_DEVICE_TIMEOUT = range(6)
GDN_BF16, GDN_F32 = 0, 1
GDN_GATE_SCALAR, GDN_GATE_CHANNEL = 0, 1

# Every symbol include/gdn.h declares.
EXPORTS = ("gdn_chunk_fwd_workspace", "gdn_chunk_fwd", "gdn_chunk_bwd_workspace",
           "gdn_chunk_bwd", "gdn_chunk_fwd_save", "gdn_chunk_bwd_saved",
           "gdn_chunk_conv_saved_workspace", "gdn_chunk_fwd_save_conv", "gdn_chunk_bwd_saved_conv", "gdn_recurrent_step", "gdn_query_device_status",
           "gdn_status_string", "gdn_profile_begin", "gdn_profile_end",
           "gdn_chunk_fwd_noalloc", "gdn_noalloc_device_status", "gdn_test_stalled_fwd", "gdn_product_fwd_workspace", "gdn_product_fwd",
           "gdn_product_bwd_workspace", "gdn_product_bwd", "gdn_chunk_fwd_varlen_workspace",
           "gdn_chunk_fwd_varlen", "gdn_chunk_bwd_varlen_workspace", "gdn_chunk_bwd_varlen",
           "gdn_tree_verify", "gdn_tree_commit", "gdn_short_conv_fwd",
           "gdn_short_conv_bwd_workspace", "gdn_short_conv_bwd")


class gdn_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("chunk", ctypes.c_int),
                ("dtype", ctypes.c_int), ("gate", ctypes.c_int), ("scale", ctypes.c_float)]


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libgdn.so with argument types set.  Raises if it is absent."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m gated_delta_rule_153_b200.build` (nvcc, sm_100a)")
            L = ctypes.CDLL(LIB_PATH)
            vp, fp, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
            dp = ctypes.POINTER(gdn_dims)
            i, f = ctypes.c_int, ctypes.c_float
            L.gdn_chunk_fwd_workspace.argtypes = [dp]
            L.gdn_chunk_fwd_workspace.restype = sz
            L.gdn_chunk_bwd_workspace.argtypes = [dp]
            L.gdn_chunk_bwd_workspace.restype = sz
            L.gdn_chunk_fwd.argtypes = [dp, vp, vp, vp, fp, fp, fp, vp, fp, vp, sz, vp]
            L.gdn_chunk_fwd.restype = i
            L.gdn_chunk_bwd.argtypes = [dp, vp, vp, vp, fp, fp, fp, vp, fp, vp, vp, vp,
                                        fp, fp, fp, vp, sz, vp]
            L.gdn_chunk_bwd.restype = i
            L.gdn_chunk_fwd_save.argtypes = L.gdn_chunk_fwd.argtypes
            L.gdn_chunk_fwd_save.restype = i
            L.gdn_chunk_bwd_saved.argtypes = L.gdn_chunk_bwd.argtypes
            L.gdn_chunk_bwd_saved.restype = i
            L.gdn_chunk_conv_saved_workspace.argtypes = [dp, i]
            L.gdn_chunk_conv_saved_workspace.restype = sz
            L.gdn_chunk_fwd_save_conv.argtypes = [dp, i, vp, vp, vp, fp, fp, fp, fp, fp, fp, vp, fp,
                                                  vp, sz, vp]
            L.gdn_chunk_fwd_save_conv.restype = i
            L.gdn_chunk_bwd_saved_conv.argtypes = [dp, i, vp, vp, vp, fp, fp, fp, fp, fp, fp, vp, fp,
                                                   vp, vp, vp, fp, fp, fp, fp, fp, fp, vp, sz, vp]
            L.gdn_chunk_bwd_saved_conv.restype = i
            L.gdn_recurrent_step.argtypes = [i, i, i, i, i, i, f, vp, vp, vp, fp, fp, fp,
                                             vp, vp]
            L.gdn_recurrent_step.restype = i
            L.gdn_query_device_status.argtypes = [vp, vp]
            L.gdn_query_device_status.restype = i
            L.gdn_chunk_fwd_noalloc.argtypes = [dp, vp, vp, vp, fp, fp, fp, vp, fp, vp]
            L.gdn_chunk_fwd_noalloc.restype = i
            L.gdn_test_stalled_fwd.argtypes = [dp, vp, vp, vp, fp, fp, fp, vp, fp, vp, sz, i,
                                               ctypes.c_ulonglong, vp]
            L.gdn_test_stalled_fwd.restype = i
            L.gdn_noalloc_device_status.argtypes = [vp]
            L.gdn_noalloc_device_status.restype = i
            L.gdn_product_fwd_workspace.argtypes = [dp, i]
            L.gdn_product_fwd_workspace.restype = sz
            L.gdn_product_bwd_workspace.argtypes = [dp, i]
            L.gdn_product_bwd_workspace.restype = sz
            L.gdn_product_fwd.argtypes = [dp, i, vp, vp, vp, fp, fp, fp, vp, fp, vp, sz, vp]
            L.gdn_product_fwd.restype = i
            L.gdn_product_bwd.argtypes = [dp, i, vp, vp, vp, fp, fp, fp, vp, fp, vp, vp, vp,
                                          fp, fp, fp, vp, sz, vp]
            L.gdn_product_bwd.restype = i
            L.gdn_chunk_fwd_varlen_workspace.argtypes = [dp, i]
            L.gdn_chunk_fwd_varlen_workspace.restype = sz
            L.gdn_chunk_bwd_varlen_workspace.argtypes = [dp, i]
            L.gdn_chunk_bwd_varlen_workspace.restype = sz
            L.gdn_chunk_fwd_varlen.argtypes = [dp, vp, i, vp, vp, vp, fp, fp, fp, vp, fp, vp,
                                               sz, vp]
            L.gdn_chunk_fwd_varlen.restype = i
            L.gdn_chunk_bwd_varlen.argtypes = [dp, vp, i, vp, vp, vp, fp, fp, fp, vp, fp, vp,
                                               vp, vp, fp, fp, fp, vp, sz, vp]
            L.gdn_chunk_bwd_varlen.restype = i
            L.gdn_tree_verify.argtypes = [i, i, i, i, i, i, i, f, vp, vp, vp, vp, fp, fp, fp,
                                          vp, vp, vp]
            L.gdn_tree_verify.restype = i
            L.gdn_tree_commit.argtypes = [i, i, i, i, i, i, i, vp, vp, vp, vp, fp, fp, fp, vp,
                                          vp]
            L.gdn_tree_commit.restype = i
            L.gdn_short_conv_fwd.argtypes = [i, i, i, i, i, i, i, vp, fp, vp, vp]
            L.gdn_short_conv_fwd.restype = i
            L.gdn_short_conv_bwd_workspace.argtypes = [i, i, i, i, i]
            L.gdn_short_conv_bwd_workspace.restype = sz
            L.gdn_short_conv_bwd.argtypes = [i, i, i, i, i, i, i, vp, fp, vp, vp, fp, vp, sz, vp]
            L.gdn_short_conv_bwd.restype = i
            L.gdn_profile_begin.argtypes = [i]
            L.gdn_profile_begin.restype = i
            L.gdn_profile_end.argtypes = [ctypes.POINTER(ctypes.c_float),
                                          ctypes.POINTER(ctypes.c_char_p), i]
            L.gdn_profile_end.restype = i
            L.gdn_status_string.argtypes = [i]
            L.gdn_status_string.restype = ctypes.c_char_p
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdn_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != GDN_OK:
        raise GdnError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _need(t, name, dtype=None, shape=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def make_dims(q, v, g, chunk=64, scale=1.0) -> gdn_dims:
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gate = GDN_GATE_CHANNEL if g.dim() == 4 else GDN_GATE_SCALAR
    return gdn_dims(B, T, H, dk, dv, int(chunk), _dtype_code(q), gate, float(scale))


def gdn_chunk_fwd_workspace(dims: gdn_dims) -> int:
    return int(lib().gdn_chunk_fwd_workspace(ctypes.byref(dims)))


def gdn_chunk_bwd_workspace(dims: gdn_dims) -> int:
    return int(lib().gdn_chunk_bwd_workspace(ctypes.byref(dims)))


def _validate_chunk_inputs(q, k, v, g, beta, h0):
    import torch
    _need(q, "q")
    B, T, H, dk = q.shape
    _need(k, "k", q.dtype, (B, T, H, dk))
    _need(v, "v", q.dtype)
    if v.shape[:3] != (B, T, H):
        raise ValueError("v must be [B,T,H,dv] matching q")
    dv = v.shape[3]
    _need(g, "g", torch.float32)
    if tuple(g.shape) not in ((B, T, H), (B, T, H, dk)):
        raise ValueError("g must be [B,T,H] or [B,T,H,dk]")
    _need(beta, "beta", torch.float32, (B, T, H))
    if h0 is not None:
        _need(h0, "h0", torch.float32, (B, H, dv, dk))
    return B, T, H, dk, dv


def _workspace(nbytes, device, workspace):
    import torch
    if nbytes == 0:
        return None
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def gdn_chunk_fwd(q, k, v, g, beta, h0=None, *, chunk=64, scale=1.0,
                  output_final_state=True, o=None, hT=None, workspace=None, stream=None):
    """Chunkwise forward.  Returns (o, hT); hT is None unless requested."""
    import torch
    B, T, H, dk, dv = _validate_chunk_inputs(q, k, v, g, beta, h0)
    dims = make_dims(q, v, g, chunk, scale)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
    if output_final_state and hT is None:
        hT = torch.empty(B, H, dv, dk, dtype=torch.float32, device=q.device)
    nbytes = gdn_chunk_fwd_workspace(dims)
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().gdn_chunk_fwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                             _ptr(beta), _ptr(h0), _ptr(o), _ptr(hT), _ptr(ws),
                             nbytes if ws is None else ws.numel() * ws.element_size(),
                             _stream(stream))
    _check(st, "gdn_chunk_fwd")
    return o, hT


def gdn_chunk_bwd(q, k, v, g, beta, dO, h0=None, dhT=None, *, chunk=64, scale=1.0,
                  workspace=None, stream=None):
    """Chunkwise backward of <dO,o> + <dhT,hT>.  Returns a dict with dq, dk,
    dv (dtype of q), dg (shape of g), dbeta, dh0 (None when h0 is None)."""
    import torch
    B, T, H, dk, dv = _validate_chunk_inputs(q, k, v, g, beta, h0)
    _need(dO, "dO", q.dtype, (B, T, H, dv))
    if dhT is not None:
        _need(dhT, "dhT", torch.float32, (B, H, dv, dk))
    dims = make_dims(q, v, g, chunk, scale)
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dg=torch.empty_like(g), dbeta=torch.empty_like(beta),
               dh0=None if h0 is None else torch.empty_like(h0))
    nbytes = gdn_chunk_bwd_workspace(dims)
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().gdn_chunk_bwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                             _ptr(beta), _ptr(h0), _ptr(dO), _ptr(dhT), _ptr(out["dq"]),
                             _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                             _ptr(out["dbeta"]), _ptr(out["dh0"]), _ptr(ws),
                             nbytes if ws is None else ws.numel() * ws.element_size(),
                             _stream(stream))
    _check(st, "gdn_chunk_bwd")
    return out


def gdn_chunk_saved_workspace(dims: gdn_dims) -> int:
    """Bytes of the workspace gdn_chunk_fwd_save fills and gdn_chunk_bwd_saved reads."""
    return max(gdn_chunk_bwd_workspace(dims), gdn_chunk_fwd_workspace(dims))


def gdn_chunk_fwd_save(q, k, v, g, beta, h0=None, *, chunk=64, scale=1.0,
                       output_final_state=True, o=None, hT=None, workspace=None, stream=None):
    """Forward of a training step.  Returns (o, hT, workspace): pass the
    workspace, and the same inputs, to gdn_chunk_bwd_saved."""
    import torch
    B, T, H, dk, dv = _validate_chunk_inputs(q, k, v, g, beta, h0)
    dims = make_dims(q, v, g, chunk, scale)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
    if output_final_state and hT is None:
        hT = torch.empty(B, H, dv, dk, dtype=torch.float32, device=q.device)
    nbytes = gdn_chunk_saved_workspace(dims)
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().gdn_chunk_fwd_save(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                  _ptr(beta), _ptr(h0), _ptr(o), _ptr(hT), _ptr(ws),
                                  nbytes if ws is None else ws.numel() * ws.element_size(),
                                  _stream(stream))
    _check(st, "gdn_chunk_fwd_save")
    return o, hT, ws


def gdn_chunk_bwd_saved(q, k, v, g, beta, dO, workspace, h0=None, dhT=None, *, chunk=64,
                        scale=1.0, out=None, stream=None):
    """Backward from gdn_chunk_fwd_save's workspace; results as gdn_chunk_bwd.
    ``out``: optional dict of preallocated result tensors (dq, dk, dv, dg,
    dbeta, dh0), filled in place."""
    import torch
    B, T, H, dk, dv = _validate_chunk_inputs(q, k, v, g, beta, h0)
    _need(dO, "dO", q.dtype, (B, T, H, dv))
    if dhT is not None:
        _need(dhT, "dhT", torch.float32, (B, H, dv, dk))
    dims = make_dims(q, v, g, chunk, scale)
    if out is None:
        out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                   dg=torch.empty_like(g), dbeta=torch.empty_like(beta),
                   dh0=None if h0 is None else torch.empty_like(h0))
    else:
        for n, ref in (("dq", q), ("dk", k), ("dv", v), ("dg", g), ("dbeta", beta)):
            _need(out[n], n, ref.dtype, tuple(ref.shape))
        if h0 is not None:
            _need(out["dh0"], "dh0", torch.float32, tuple(h0.shape))
    nbytes = gdn_chunk_saved_workspace(dims)
    if nbytes and (workspace is None or workspace.numel() * workspace.element_size() < nbytes):
        raise ValueError(f"workspace must be gdn_chunk_fwd_save's ({nbytes} bytes)")
    st = lib().gdn_chunk_bwd_saved(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                   _ptr(beta), _ptr(h0), _ptr(dO), _ptr(dhT), _ptr(out["dq"]),
                                   _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                                   _ptr(out["dbeta"]), _ptr(out["dh0"]), _ptr(workspace),
                                   0 if workspace is None else workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check(st, "gdn_chunk_bwd_saved")
    return out


def _validate_conv_chunk(xq, xk, xv, wq, wk, wv, g, beta, h0):
    import torch
    B, T, H, dk, dv = _validate_chunk_inputs(xq, xk, xv, g, beta, h0)
    K = wq.shape[-1] if wq.dim() == 3 else 0
    for w, name, d in ((wq, "wq", dk), (wk, "wk", dk), (wv, "wv", dv)):
        _need(w, name, torch.float32, (H, d, K))
    return B, T, H, dk, dv, K


def gdn_chunk_fwd_save_conv(xq, xk, xv, wq, wk, wv, g, beta, h0=None, *, chunk=64, scale=1.0,
                            output_final_state=True, o=None, hT=None, workspace=None, stream=None):
    """Forward of a training step from the raw projections: the short
    convolution, SiLU and (q, k) L2 norm, then the gated delta rule.  Returns
    (o, hT, workspace); pass the workspace to gdn_chunk_bwd_saved_conv."""
    import torch
    B, T, H, dk, dv, K = _validate_conv_chunk(xq, xk, xv, wq, wk, wv, g, beta, h0)
    dims = make_dims(xq, xv, g, chunk, scale)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=xq.dtype, device=xq.device)
    if output_final_state and hT is None:
        hT = torch.empty(B, H, dv, dk, dtype=torch.float32, device=xq.device)
    nbytes = int(lib().gdn_chunk_conv_saved_workspace(ctypes.byref(dims), K))
    ws = _workspace(nbytes, xq.device, workspace)
    st = lib().gdn_chunk_fwd_save_conv(ctypes.byref(dims), K, _ptr(xq), _ptr(xk), _ptr(xv),
                                       _ptr(wq), _ptr(wk), _ptr(wv), _ptr(g), _ptr(beta), _ptr(h0),
                                       _ptr(o), _ptr(hT), _ptr(ws),
                                       0 if ws is None else ws.numel() * ws.element_size(),
                                       _stream(stream))
    _check(st, "gdn_chunk_fwd_save_conv")
    return o, hT, ws


def gdn_chunk_bwd_saved_conv(xq, xk, xv, wq, wk, wv, g, beta, dO, workspace, h0=None, dhT=None,
                             *, chunk=64, scale=1.0, stream=None):
    """Backward from gdn_chunk_fwd_save_conv's workspace.  Returns a dict with
    dxq, dxk, dxv, dwq, dwk, dwv, dg, dbeta, dh0."""
    import torch
    B, T, H, dk, dv, K = _validate_conv_chunk(xq, xk, xv, wq, wk, wv, g, beta, h0)
    _need(dO, "dO", xq.dtype, (B, T, H, dv))
    if dhT is not None:
        _need(dhT, "dhT", torch.float32, (B, H, dv, dk))
    dims = make_dims(xq, xv, g, chunk, scale)
    out = dict(dxq=torch.empty_like(xq), dxk=torch.empty_like(xk), dxv=torch.empty_like(xv),
               dwq=torch.empty_like(wq), dwk=torch.empty_like(wk), dwv=torch.empty_like(wv),
               dg=torch.empty_like(g), dbeta=torch.empty_like(beta),
               dh0=None if h0 is None else torch.empty_like(h0))
    st = lib().gdn_chunk_bwd_saved_conv(
        ctypes.byref(dims), K, _ptr(xq), _ptr(xk), _ptr(xv), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(g),
        _ptr(beta), _ptr(h0), _ptr(dO), _ptr(dhT), _ptr(out["dxq"]), _ptr(out["dxk"]),
        _ptr(out["dxv"]), _ptr(out["dwq"]), _ptr(out["dwk"]), _ptr(out["dwv"]), _ptr(out["dg"]),
        _ptr(out["dbeta"]), _ptr(out["dh0"]), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "gdn_chunk_bwd_saved_conv")
    return out


def gdn_recurrent_step(q, k, v, g, beta, state, *, scale=1.0, o=None, stream=None):
    """One decode token, in place on ``state`` [N,H,dv,dk] fp32.  q,k [N,H,dk];
    v [N,H,dv]; g [N,H] or [N,H,dk]; beta [N,H].  Returns o [N,H,dv]."""
    import torch
    _need(q, "q")
    N, H, dk = q.shape
    _need(k, "k", q.dtype, (N, H, dk))
    _need(v, "v", q.dtype)
    dv = v.shape[-1]
    _need(g, "g", torch.float32)
    gate = GDN_GATE_CHANNEL if g.dim() == 3 else GDN_GATE_SCALAR
    _need(beta, "beta", torch.float32, (N, H))
    _need(state, "state", torch.float32, (N, H, dv, dk))
    if o is None:
        o = torch.empty(N, H, dv, dtype=q.dtype, device=q.device)
    st = lib().gdn_recurrent_step(N, H, dk, dv, _dtype_code(q), gate, float(scale), _ptr(q),
                                  _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
                                  _ptr(o), _stream(stream))
    _check(st, "gdn_recurrent_step")
    return o


def gdn_profile_begin(capacity: int) -> None:
    """Start bracketing this thread's next ``capacity`` library launches with
    CUDA events (a profiling aid)."""
    _check(lib().gdn_profile_begin(int(capacity)), "gdn_profile_begin")


def gdn_profile_end(capacity: int):
    """Stop recording; returns (launch count, [(kernel name, ms), ...])."""
    ms = (ctypes.c_float * capacity)()
    names = (ctypes.c_char_p * capacity)()
    n = lib().gdn_profile_end(ms, names, int(capacity))
    if n < 0:
        raise RuntimeError("gdn_profile_end: recording was not on or a CUDA call failed")
    return n, [(names[i].decode(), float(ms[i])) for i in range(min(n, capacity))]


def gdn_query_device_status(workspace, stream=None) -> int:
    """Status word of the most recent chunkwise call that used ``workspace``."""
    return int(lib().gdn_query_device_status(_ptr(workspace), _stream(stream)))


# ---- gated DeltaProduct (n delta-rule steps per token) ---------------------
def _validate_product_inputs(q, k, v, g, beta, h0):
    import torch
    _need(q, "q")
    B, T, H, dk = q.shape
    if k.dim() != 5:
        raise ValueError("k must be [B,T,n,H,dk]")
    n = k.shape[2]
    _need(k, "k", q.dtype, (B, T, n, H, dk))
    _need(v, "v", q.dtype)
    if v.dim() != 5 or v.shape[:4] != (B, T, n, H):
        raise ValueError("v must be [B,T,n,H,dv] matching k")
    dv = v.shape[4]
    _need(g, "g", torch.float32)
    if tuple(g.shape) not in ((B, T, H), (B, T, H, dk)):
        raise ValueError("g must be [B,T,H] or [B,T,H,dk]")
    _need(beta, "beta", torch.float32, (B, T, n, H))
    if h0 is not None:
        _need(h0, "h0", torch.float32, (B, H, dv, dk))
    return B, T, n, H, dk, dv


def gdn_product_fwd(q, k, v, g, beta, h0=None, *, chunk=64, scale=1.0,
                    output_final_state=True, workspace=None, stream=None):
    """Gated DeltaProduct forward: k [B,T,n,H,dk], v [B,T,n,H,dv],
    beta [B,T,n,H]; q, g, h0 as for gdn_chunk_fwd.  Returns (o, hT)."""
    import torch
    B, T, n, H, dk, dv = _validate_product_inputs(q, k, v, g, beta, h0)
    dims = make_dims(q, v, g, chunk, scale)
    o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
    hT = torch.empty(B, H, dv, dk, dtype=torch.float32, device=q.device) \
        if output_final_state else None
    nbytes = int(lib().gdn_product_fwd_workspace(ctypes.byref(dims), n))
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().gdn_product_fwd(ctypes.byref(dims), n, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                               _ptr(beta), _ptr(h0), _ptr(o), _ptr(hT), _ptr(ws),
                               nbytes if ws is None else ws.numel() * ws.element_size(),
                               _stream(stream))
    _check(st, "gdn_product_fwd")
    return o, hT


def gdn_product_bwd(q, k, v, g, beta, dO, h0=None, dhT=None, *, chunk=64, scale=1.0,
                    workspace=None, stream=None):
    """Gated DeltaProduct backward of <dO,o> + <dhT,hT>: gradients in the
    shapes of their primals (dh0 None when h0 is None)."""
    import torch
    B, T, n, H, dk, dv = _validate_product_inputs(q, k, v, g, beta, h0)
    _need(dO, "dO", q.dtype, (B, T, H, dv))
    if dhT is not None:
        _need(dhT, "dhT", torch.float32, (B, H, dv, dk))
    dims = make_dims(q, v, g, chunk, scale)
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dg=torch.empty_like(g), dbeta=torch.empty_like(beta),
               dh0=None if h0 is None else torch.empty_like(h0))
    nbytes = int(lib().gdn_product_bwd_workspace(ctypes.byref(dims), n))
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().gdn_product_bwd(ctypes.byref(dims), n, _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                               _ptr(beta), _ptr(h0), _ptr(dO), _ptr(dhT), _ptr(out["dq"]),
                               _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                               _ptr(out["dbeta"]), _ptr(out["dh0"]), _ptr(ws),
                               nbytes if ws is None else ws.numel() * ws.element_size(),
                               _stream(stream))
    _check(st, "gdn_product_bwd")
    return out


# ---- packed variable-length batches ----------------------------------------
def _validate_varlen(q, k, v, g, beta, cu_seqlens, h0):
    import torch
    B, T, H, dk, dv = _validate_chunk_inputs(q, k, v, g, beta, None)
    if B != 1:
        raise ValueError("packed sequences take q [1, total_tokens, H, dk]")
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be [nseq + 1] int32")
    nseq = cu_seqlens.numel() - 1
    if h0 is not None:
        _need(h0, "h0", torch.float32, (nseq, H, dv, dk))
    return nseq, T, H, dk, dv


def gdn_chunk_fwd_varlen(q, k, v, g, beta, cu_seqlens, h0=None, *, scale=1.0,
                         output_final_state=True, workspace=None, stream=None):
    """Chunkwise forward over packed sequences: q [1,T,H,dk] etc. hold nseq
    sequences back to back, sequence s at tokens cu_seqlens[s]..cu_seqlens[s+1]-1
    (cu_seqlens int32 on the device).  h0 / hT are [nseq,H,dv,dk].  Returns
    (o, hT)."""
    import torch
    nseq, T, H, dk, dv = _validate_varlen(q, k, v, g, beta, cu_seqlens, h0)
    dims = make_dims(q, v, g, 64, scale)
    o = torch.empty(1, T, H, dv, dtype=q.dtype, device=q.device)
    hT = torch.empty(nseq, H, dv, dk, dtype=torch.float32, device=q.device) \
        if output_final_state else None
    nbytes = int(lib().gdn_chunk_fwd_varlen_workspace(ctypes.byref(dims), nseq))
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().gdn_chunk_fwd_varlen(ctypes.byref(dims), _ptr(cu_seqlens), nseq, _ptr(q),
                                    _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(o),
                                    _ptr(hT), _ptr(ws),
                                    nbytes if ws is None else ws.numel() * ws.element_size(),
                                    _stream(stream))
    _check(st, "gdn_chunk_fwd_varlen")
    return o, hT


def gdn_chunk_bwd_varlen(q, k, v, g, beta, cu_seqlens, dO, h0=None, dhT=None, *, scale=1.0,
                         workspace=None, stream=None):
    """Backward of gdn_chunk_fwd_varlen: gradients in the shapes of their
    primals (dh0 None when h0 is None)."""
    import torch
    nseq, T, H, dk, dv = _validate_varlen(q, k, v, g, beta, cu_seqlens, h0)
    _need(dO, "dO", q.dtype, (1, T, H, dv))
    if dhT is not None:
        _need(dhT, "dhT", torch.float32, (nseq, H, dv, dk))
    dims = make_dims(q, v, g, 64, scale)
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dg=torch.empty_like(g), dbeta=torch.empty_like(beta),
               dh0=None if h0 is None else torch.empty_like(h0))
    nbytes = int(lib().gdn_chunk_bwd_varlen_workspace(ctypes.byref(dims), nseq))
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().gdn_chunk_bwd_varlen(ctypes.byref(dims), _ptr(cu_seqlens), nseq, _ptr(q),
                                    _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(dO),
                                    _ptr(dhT), _ptr(out["dq"]), _ptr(out["dk"]),
                                    _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
                                    _ptr(out["dh0"]), _ptr(ws),
                                    nbytes if ws is None else ws.numel() * ws.element_size(),
                                    _stream(stream))
    _check(st, "gdn_chunk_bwd_varlen")
    return out


# ---- draft-tree verification and commit ------------------------------------
def _validate_tree(parent, k, v, g, beta, state):
    import torch
    _need(parent, "parent", torch.int32)
    if parent.dim() != 2:
        raise ValueError("parent must be [N, M] int32")
    N, M = parent.shape
    _need(k, "k")
    if k.dim() != 4 or tuple(k.shape[:2]) != (N, M):
        raise ValueError("k must be [N, M, H, dk]")
    H, dk = k.shape[2], k.shape[3]
    _need(v, "v", k.dtype)
    if v.dim() != 4 or tuple(v.shape[:3]) != (N, M, H):
        raise ValueError("v must be [N, M, H, dv]")
    dv = v.shape[3]
    gate = GDN_GATE_CHANNEL if g.dim() == 4 else GDN_GATE_SCALAR
    _need(g, "g", torch.float32)
    if tuple(g.shape[:3]) != (N, M, H):
        raise ValueError("g must be [N, M, H]")
    _need(beta, "beta", torch.float32, (N, M, H))
    _need(state, "state", torch.float32, (N, H, dv, dk))
    return N, M, H, dk, dv, gate


def gdn_tree_verify(parent, q, k, v, g, beta, state, *, scale=1.0, o=None, status=None,
                    stream=None):
    """Outputs of every draft-tree node: o [N,M,H,dv], node i read out after
    the tokens of its root path, from ``state`` [N,H,dv,dk] (not modified)."""
    import torch
    N, M, H, dk, dv, gate = _validate_tree(parent, k, v, g, beta, state)
    _need(q, "q", k.dtype, tuple(k.shape))
    if o is None:
        o = torch.empty(N, M, H, dv, dtype=q.dtype, device=q.device)
    st = lib().gdn_tree_verify(N, M, H, dk, dv, _dtype_code(q), gate, float(scale),
                               _ptr(parent), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                               _ptr(state), _ptr(o), _ptr(status), _stream(stream))
    _check(st, "gdn_tree_verify")
    return o


def gdn_tree_commit(parent, accepted, k, v, g, beta, state, *, status=None, stream=None):
    """In place on ``state``: the state after the root path of node
    accepted[n] (int32 [N]; -1 leaves state[n] as it is)."""
    import torch
    N, M, H, dk, dv, gate = _validate_tree(parent, k, v, g, beta, state)
    _need(accepted, "accepted", torch.int32, (N,))
    st = lib().gdn_tree_commit(N, M, H, dk, dv, _dtype_code(k), gate, _ptr(parent),
                               _ptr(accepted), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                               _ptr(state), _ptr(status), _stream(stream))
    _check(st, "gdn_tree_commit")
    return state


# ---- q/k/v prologue: short causal convolution, SiLU, L2 norm ---------------
def _validate_conv(x, w):
    import torch
    _need(x, "x")
    if x.dim() != 4:
        raise ValueError("x must be [B, T, H, d]")
    B, T, H, d = x.shape
    _need(w, "w", torch.float32)
    if w.dim() != 3 or tuple(w.shape[:2]) != (H, d):
        raise ValueError("w must be [H, d, K] fp32")
    return B, T, H, d, w.shape[2]


def gdn_short_conv_fwd(x, w, *, l2norm=True, y=None, stream=None):
    """y = (L2-normalised) SiLU(causal depthwise conv of x with w): x
    [B,T,H,d] bf16/fp32, w [H,d,K] fp32.  Returns y (shape and dtype of x)."""
    import torch
    B, T, H, d, K = _validate_conv(x, w)
    if y is None:
        y = torch.empty_like(x)
    st = lib().gdn_short_conv_fwd(B, T, H, d, K, _dtype_code(x), int(bool(l2norm)), _ptr(x),
                                  _ptr(w), _ptr(y), _stream(stream))
    _check(st, "gdn_short_conv_fwd")
    return y


def gdn_short_conv_bwd(x, w, dy, *, l2norm=True, workspace=None, stream=None):
    """Gradients of <dy, y> for gdn_short_conv_fwd: returns (dx, dw)."""
    import torch
    B, T, H, d, K = _validate_conv(x, w)
    _need(dy, "dy", x.dtype, tuple(x.shape))
    dx = torch.empty_like(x)
    dw = torch.empty_like(w)
    nbytes = int(lib().gdn_short_conv_bwd_workspace(B, T, H, d, K))
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().gdn_short_conv_bwd(B, T, H, d, K, _dtype_code(x), int(bool(l2norm)), _ptr(x),
                                  _ptr(w), _ptr(dy), _ptr(dx), _ptr(dw), _ptr(ws),
                                  nbytes if ws is None else ws.numel() * ws.element_size(),
                                  _stream(stream))
    _check(st, "gdn_short_conv_bwd")
    return dx, dw
