"""The C-ABI library loads, exports every symbol include/gdn.h declares, and
rejects bad arguments on the host before touching the device (CPU only)."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_153_b200 as gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(gdn_[a-z_0-9]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol():
    L = gdn.lib()
    declared = _declared()
    assert declared, "no declarations found"
    assert declared == set(gdn.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name


def _dims(**kw):
    d = dict(B=1, T=64, H=2, dk=128, dv=128, chunk=64, dtype=gdn.GDN_BF16,
             gate=gdn.GDN_GATE_SCALAR, scale=1.0)
    d.update(kw)
    return gdn.gdn_dims(**d)


def test_status_strings():
    assert gdn.status_string(gdn.GDN_OK) == "GDN_OK"
    assert gdn.status_string(gdn.GDN_ERR_DEVICE_TIMEOUT) == "GDN_ERR_DEVICE_TIMEOUT"


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), gdn.GDN_ERR_INVALID_ARG), (dict(T=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(H=-1), gdn.GDN_ERR_INVALID_ARG), (dict(chunk=48), gdn.GDN_ERR_INVALID_ARG),
    (dict(dtype=7), gdn.GDN_ERR_INVALID_ARG), (dict(gate=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=96), gdn.GDN_ERR_UNSUPPORTED), (dict(dv=256), gdn.GDN_ERR_UNSUPPORTED),
])
def test_dims_rejected_before_launch(kw, code):
    L = gdn.lib()
    d = _dims(**kw)
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    assert L.gdn_chunk_fwd_workspace(ctypes.byref(d)) == 0
    st = L.gdn_chunk_fwd(ctypes.byref(d), p, p, p, p, p, None, p, None, p, 1 << 40, None)
    assert st == code
    st = L.gdn_chunk_bwd(ctypes.byref(d), p, p, p, p, p, None, p, None, p, p, p, p, p, None,
                         p, 1 << 40, None)
    assert st == code


def test_pointer_checks():
    L = gdn.lib()
    d = _dims()
    p = ctypes.c_void_p(256)
    mis = ctypes.c_void_p(258)
    ws = ctypes.c_void_p(1 << 20)
    big = 1 << 40
    # null required pointer
    assert L.gdn_chunk_fwd(ctypes.byref(d), None, p, p, p, p, None, p, None, ws, big,
                           None) == gdn.GDN_ERR_INVALID_ARG
    # misaligned pointer
    assert L.gdn_chunk_fwd(ctypes.byref(d), p, mis, p, p, p, None, p, None, ws, big,
                           None) == gdn.GDN_ERR_INVALID_ARG
    # h0 aliasing hT
    assert L.gdn_chunk_fwd(ctypes.byref(d), p, p, p, p, p, p, p, p, ws, big,
                           None) == gdn.GDN_ERR_INVALID_ARG
    # workspace too small / missing / misaligned
    need = L.gdn_chunk_fwd_workspace(ctypes.byref(d))
    assert need > 0
    assert L.gdn_chunk_fwd(ctypes.byref(d), p, p, p, p, p, None, p, None, ws, need - 1,
                           None) == gdn.GDN_ERR_WORKSPACE
    assert L.gdn_chunk_fwd(ctypes.byref(d), p, p, p, p, p, None, p, None, None, big,
                           None) == gdn.GDN_ERR_WORKSPACE
    assert L.gdn_chunk_fwd(ctypes.byref(d), p, p, p, p, p, None, p, None,
                           ctypes.c_void_p((1 << 20) + 16), big, None) == gdn.GDN_ERR_WORKSPACE
    # dh0 given without h0 (and the reverse)
    assert L.gdn_chunk_bwd(ctypes.byref(d), p, p, p, p, p, None, p, None, p, p, p, p, p, p,
                           ws, big, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_chunk_bwd(ctypes.byref(d), p, p, p, p, p, p, p, None, p, p, p, p, p, None,
                           ws, big, None) == gdn.GDN_ERR_INVALID_ARG


def test_decode_checks():
    L = gdn.lib()
    p = ctypes.c_void_p(256)
    assert L.gdn_recurrent_step(0, 16, 128, 128, 0, 0, 1.0, p, p, p, p, p, p, p,
                                None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_recurrent_step(4, 16, 100, 128, 0, 0, 1.0, p, p, p, p, p, p, p,
                                None) == gdn.GDN_ERR_UNSUPPORTED
    assert L.gdn_recurrent_step(4, 16, 128, 128, 0, 0, 1.0, p, p, p, p, p, None, p,
                                None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_recurrent_step(4, 16, 128, 128, 0, 5, 1.0, p, p, p, p, p, p, p,
                                None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_query_device_status(None, None) == gdn.GDN_ERR_INVALID_ARG


def test_workspace_sizes_grow_with_problem():
    L = gdn.lib()
    a = L.gdn_chunk_bwd_workspace(ctypes.byref(_dims(T=64)))
    b = L.gdn_chunk_bwd_workspace(ctypes.byref(_dims(T=4096)))
    assert 0 < a < b
    assert L.gdn_chunk_fwd_workspace(ctypes.byref(_dims(T=64))) % 4 == 0


def test_product_checks():
    """gdn_product_*: n out of range is rejected on the host (no launch)."""
    L = gdn.lib()
    d = gdn.gdn_dims(1, 64, 2, 128, 128, 64, gdn.GDN_BF16, gdn.GDN_GATE_SCALAR, 1.0)
    assert L.gdn_product_fwd_workspace(ctypes.byref(d), 0) == 0
    assert L.gdn_product_fwd_workspace(ctypes.byref(d), 65) == 0
    assert L.gdn_product_fwd_workspace(ctypes.byref(d), 2) > L.gdn_chunk_fwd_workspace(ctypes.byref(d))
    assert L.gdn_product_bwd_workspace(ctypes.byref(d), 3) > 0
    p = ctypes.c_void_p(256)
    for n in (0, 65):
        assert L.gdn_product_fwd(ctypes.byref(d), n, p, p, p, p, p, None, p, None, p, 1 << 30,
                                 None) == gdn.GDN_ERR_INVALID_ARG


def test_varlen_checks():
    """gdn_chunk_*_varlen: B != 1, nseq < 1 and a null or misaligned offset
    array are rejected on the host, non-tensor-core shapes are unsupported;
    the workspace grows with the number of sequences."""
    L = gdn.lib()
    d = gdn.gdn_dims(1, 1000, 4, 128, 128, 64, gdn.GDN_BF16, gdn.GDN_GATE_SCALAR, 1.0)
    w1 = L.gdn_chunk_fwd_varlen_workspace(ctypes.byref(d), 1)
    w9 = L.gdn_chunk_fwd_varlen_workspace(ctypes.byref(d), 9)
    assert 0 < w1 < w9
    assert L.gdn_chunk_bwd_varlen_workspace(ctypes.byref(d), 9) > w9
    assert L.gdn_chunk_fwd_varlen_workspace(ctypes.byref(d), 0) == 0
    d2 = gdn.gdn_dims(2, 1000, 4, 128, 128, 64, gdn.GDN_BF16, gdn.GDN_GATE_SCALAR, 1.0)
    assert L.gdn_chunk_fwd_varlen_workspace(ctypes.byref(d2), 3) == 0
    f32 = gdn.gdn_dims(1, 1000, 4, 128, 128, 64, gdn.GDN_F32, gdn.GDN_GATE_SCALAR, 1.0)
    assert L.gdn_chunk_bwd_varlen_workspace(ctypes.byref(f32), 3) == 0
    p = ctypes.c_void_p(256)
    ws = 1 << 40
    fwd = L.gdn_chunk_fwd_varlen
    assert fwd(ctypes.byref(d), p, 0, p, p, p, p, p, None, p, None, p, ws, None) == \
        gdn.GDN_ERR_INVALID_ARG
    assert fwd(ctypes.byref(d2), p, 3, p, p, p, p, p, None, p, None, p, ws, None) == \
        gdn.GDN_ERR_INVALID_ARG
    assert fwd(ctypes.byref(d), None, 3, p, p, p, p, p, None, p, None, p, ws, None) == \
        gdn.GDN_ERR_INVALID_ARG
    assert fwd(ctypes.byref(d), ctypes.c_void_p(258), 3, p, p, p, p, p, None, p, None, p, ws,
               None) == gdn.GDN_ERR_INVALID_ARG
    assert fwd(ctypes.byref(f32), p, 3, p, p, p, p, p, None, p, None, p, ws, None) == \
        gdn.GDN_ERR_UNSUPPORTED
    assert fwd(ctypes.byref(d), p, 3, p, p, p, p, p, None, p, None, p, 16, None) == \
        gdn.GDN_ERR_WORKSPACE
    bwd = L.gdn_chunk_bwd_varlen
    assert bwd(ctypes.byref(d), p, 3, p, p, p, p, p, p, p, None, p, p, p, p, p, None, p, ws,
               None) == gdn.GDN_ERR_INVALID_ARG  # dh0 without h0


def test_tree_checks():
    """gdn_tree_*: host-side rejection before any launch."""
    L = gdn.lib()
    p = ctypes.c_void_p(256)
    bf, sc, ch = gdn.GDN_BF16, gdn.GDN_GATE_SCALAR, gdn.GDN_GATE_CHANNEL
    v = L.gdn_tree_verify
    args = (p, p, p, p, p, p, p, p, None, None)
    assert v(2, 0, 4, 128, 128, bf, sc, 1.0, *args) == gdn.GDN_ERR_INVALID_ARG
    assert v(2, 65, 4, 128, 128, bf, sc, 1.0, *args) == gdn.GDN_ERR_UNSUPPORTED
    assert v(2, 8, 4, 64, 128, bf, sc, 1.0, *args) == gdn.GDN_ERR_UNSUPPORTED
    assert v(2, 8, 4, 128, 128, gdn.GDN_F32, sc, 1.0, *args) == gdn.GDN_ERR_UNSUPPORTED
    # the channel gate is supported, with its g rows 16-byte aligned
    assert v(2, 8, 4, 128, 128, bf, ch, 1.0, p, p, p, p, ctypes.c_void_p(260), p, p, p, None,
             None) == gdn.GDN_ERR_INVALID_ARG
    assert v(2, 8, 4, 128, 128, bf, sc, float("nan"), *args) == gdn.GDN_ERR_INVALID_ARG
    assert v(2, 8, 4, 128, 128, bf, sc, 1.0, None, *args[1:]) == gdn.GDN_ERR_INVALID_ARG
    assert v(2, 8, 4, 128, 128, bf, sc, 1.0, p, ctypes.c_void_p(264), *args[2:]) == \
        gdn.GDN_ERR_INVALID_ARG
    c = L.gdn_tree_commit
    assert c(0, 8, 4, 128, 128, bf, sc, p, p, p, p, p, p, p, None, None) == \
        gdn.GDN_ERR_INVALID_ARG
    assert c(2, 8, 4, 128, 128, bf, sc, p, None, p, p, p, p, p, None, None) == \
        gdn.GDN_ERR_INVALID_ARG
    assert c(2, 8, 4, 128, 128, bf, sc, p, ctypes.c_void_p(258), p, p, p, p, p, None,
             None) == gdn.GDN_ERR_INVALID_ARG


def test_short_conv_checks():
    L = gdn.lib()
    p = ctypes.c_void_p(256)
    bf = gdn.GDN_BF16
    f = L.gdn_short_conv_fwd
    assert f(0, 8, 2, 128, 4, bf, 1, p, p, ctypes.c_void_p(512), None) == gdn.GDN_ERR_INVALID_ARG
    assert f(1, 8, 2, 96, 4, bf, 1, p, p, ctypes.c_void_p(512), None) == gdn.GDN_ERR_UNSUPPORTED
    assert f(1, 8, 2, 128, 5, bf, 1, p, p, ctypes.c_void_p(512), None) == gdn.GDN_ERR_UNSUPPORTED
    assert f(1, 8, 2, 128, 0, bf, 1, p, p, ctypes.c_void_p(512), None) == gdn.GDN_ERR_INVALID_ARG
    assert f(1, 8, 2, 128, 4, bf, 1, p, p, p, None) == gdn.GDN_ERR_INVALID_ARG  # y aliases x
    assert f(1, 8, 2, 128, 4, bf, 1, ctypes.c_void_p(264), p, ctypes.c_void_p(512),
             None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_short_conv_bwd_workspace(2, 100, 3, 128, 4) == 2 * 4 * 3 * 128 * 4 * 4
    b = L.gdn_short_conv_bwd
    q = ctypes.c_void_p(1024)
    assert b(2, 100, 3, 128, 4, bf, 1, p, p, ctypes.c_void_p(512), q, p, p, 16, None) == \
        gdn.GDN_ERR_WORKSPACE
    assert b(2, 100, 3, 128, 4, bf, 1, p, p, ctypes.c_void_p(512), p, p, p, 1 << 30, None) == \
        gdn.GDN_ERR_INVALID_ARG  # dx aliases x


def test_header_is_plain_c(tmp_path):
    """include/gdn.h compiles as C11 on its own, and every entry point it
    declares can be named from C (taking each one's address)."""
    import subprocess
    names = sorted(_declared())
    src = tmp_path / "use.c"
    src.write_text('#include "gdn.h"\ntypedef void (*entry)(void);\n' +
                   "entry gdn_entry_points[] = {\n" +
                   "".join(f"    (entry)&{n},\n" for n in names) + "};\n")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-pedantic", "-c",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(tmp_path / "use.o")],
                   check=True)


def test_stalled_fwd_hook_checks():
    """The wait-timeout test hook rejects bad hook arguments and shapes that
    do not take the tcgen05 whole-head walk, on the host."""
    L = gdn.lib()
    p = ctypes.c_void_p(256)
    ws = ctypes.c_void_p(1 << 20)
    big = 1 << 40
    wide = gdn.gdn_dims(1, 512, 40, 128, 128, 64, gdn.GDN_BF16, gdn.GDN_GATE_SCALAR, 1.0)
    narrow = gdn.gdn_dims(1, 512, 1, 128, 128, 64, gdn.GDN_BF16, gdn.GDN_GATE_SCALAR, 1.0)
    f32 = gdn.gdn_dims(1, 512, 40, 128, 128, 64, gdn.GDN_F32, gdn.GDN_GATE_SCALAR, 1.0)
    call = lambda d, stall, ns: L.gdn_test_stalled_fwd(ctypes.byref(d), p, p, p, p, p, None, p,
                                                       None, ws, big, stall, ns, None)
    assert call(wide, -1, 1000) == gdn.GDN_ERR_INVALID_ARG
    assert call(wide, 2, 0) == gdn.GDN_ERR_INVALID_ARG
    assert call(wide, 2, 2_000_000_000) == gdn.GDN_ERR_INVALID_ARG
    assert call(narrow, 2, 1000) == gdn.GDN_ERR_UNSUPPORTED
    assert call(f32, 2, 1000) == gdn.GDN_ERR_UNSUPPORTED


def test_training_pair_bindings_reject_host_tensors():
    """The training-pair bindings run their argument checks before any device
    work: host tensors are refused with TypeError."""
    import torch
    import gated_delta_rule_153_b200 as gdn
    B, T, H, d, K = 1, 8, 2, 128, 4
    x = torch.zeros(B, T, H, d, dtype=torch.bfloat16)
    w = torch.zeros(H, d, K)
    g, beta = torch.zeros(B, T, H), torch.zeros(B, T, H)
    with pytest.raises(TypeError):
        gdn.gdn_chunk_fwd_save(x, x, x, g, beta)
    with pytest.raises(TypeError):
        gdn.gdn_chunk_bwd_saved(x, x, x, g, beta, x, None)
    with pytest.raises(TypeError):
        gdn.gdn_chunk_fwd_save_conv(x, x, x, w, w, w, g, beta)
    with pytest.raises(TypeError):
        gdn.gdn_chunk_bwd_saved_conv(x, x, x, w, w, w, g, beta, x, None)
