"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The CUDA library never links,
loads or calls it, and it shares no code with the CUDA path.

The arithmetic lives in ``gdn_oracle.c`` (a plain token-by-token loop in
double precision, OpenMP over independent (sequence, head) pairs).  This module
compiles it on first use with the system C compiler and exposes numpy wrappers.

Source of the computation: "Gated Delta Networks: Improving Mamba2 with Delta
Rule" (paper review), section "Method" -- the gated delta rule
S_t = S_{t-1} a_t (I - b_t k_t k_t^T) + b_t v_t k_t^T, read out as
o_t = S_t q_t; the channel-gate variant (Kimi Delta Attention, named in the
same review's linked reviews and in the "Linear Attention Architectures"
abstract) replaces a_t by Diag(a_t) on the key index.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i, d = ctypes.c_int, ctypes.c_double
    lib.gdn_oracle_fwd.argtypes = [i, i, i, i, i, i, d] + [dp] * 8
    lib.gdn_oracle_fwd.restype = None
    lib.gdn_oracle_step.argtypes = [i, i, i, i, i, d] + [dp] * 7
    lib.gdn_oracle_step.restype = None
    lib.gdn_oracle_bwd.argtypes = [i, i, i, i, i, i, d] + [dp] * 14 + [i]
    lib.gdn_oracle_bwd.restype = None
    lib.gdn_oracle_threads.argtypes = []
    lib.gdn_oracle_threads.restype = ctypes.c_int
    return lib


def load_library(path):
    """Bind an oracle shared library built from (a variant of) gdn_oracle.c;
    the result can be passed as ``lib=`` to fwd/step/bwd.  Used by the tests
    that plant mistakes in the oracle to show that the pins catch them."""
    return _bind(path)


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB_PATH)
    return _lib


def threads() -> int:
    """Number of OpenMP threads the oracle uses."""
    return int(_load().gdn_oracle_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def fwd(q, k, v, g, beta, h0=None, scale=1.0, channel_gate=None, want_state=True,
        lib=None):
    """Token-loop forward.  q,k [B,T,H,dk], v [B,T,H,dv], g [B,T,H] or
    [B,T,H,dk], beta [B,T,H], h0 [B,H,dv,dk] or None.
    Returns (o [B,T,H,dv], hT [B,H,dv,dk]) as float64 arrays."""
    q, k, v, g, beta, h0 = map(_f64, (q, k, v, g, beta, h0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if channel_gate is None:
        channel_gate = g.ndim == 4
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dv, dk)) if want_state else None
    (lib or _load()).gdn_oracle_fwd(B, T, H, dk, dv, int(channel_gate), float(scale),
                           _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                           _ptr(h0), _ptr(o), _ptr(hT))
    return o, hT


def step(q, k, v, g, beta, state, scale=1.0, channel_gate=None, lib=None):
    """One decode step on N*H independent states.  q,k [N,H,dk], v [N,H,dv],
    g [N,H] or [N,H,dk], beta [N,H], state [N,H,dv,dk].
    Returns (o [N,H,dv], new_state) as float64 arrays (inputs untouched)."""
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    st = _f64(state).copy()
    N, H, dk = q.shape
    dv = v.shape[-1]
    if channel_gate is None:
        channel_gate = g.ndim == 3
    o = np.zeros((N, H, dv))
    (lib or _load()).gdn_oracle_step(N, H, dk, dv, int(channel_gate), float(scale),
                            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                            _ptr(st), _ptr(o))
    return o, st


def bwd(q, k, v, g, beta, dO, h0=None, dhT=None, scale=1.0, channel_gate=None,
        ckpt=64, lib=None):
    """Reverse-mode gradients of L = <dO, o> + <dhT, hT> through the token
    loop.  Returns dict(dq, dk, dv, dg, dbeta, dh0) of float64 arrays
    (dh0 is the gradient w.r.t. the initial state, zero-state included)."""
    q, k, v, g, beta, dO, h0, dhT = map(_f64, (q, k, v, g, beta, dO, h0, dhT))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if channel_gate is None:
        channel_gate = g.ndim == 4
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dg=np.zeros_like(g), dbeta=np.zeros_like(beta),
               dh0=np.zeros((B, H, dv, dk)))
    (lib or _load()).gdn_oracle_bwd(B, T, H, dk, dv, int(channel_gate), float(scale),
                           _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                           _ptr(h0), _ptr(dO), _ptr(dhT),
                           _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                           _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dh0"]),
                           int(ckpt))
    return out
