"""The seeded input generators (CPU): shapes, determinism, and the structure
the kernels rely on -- parents before children in draft trees, offsets that
run from 0 to T in packed batches."""
import torch

from gated_delta_rule_153_b200.inputs import (L350M, make_chunk_inputs, make_prologue_inputs,
                                              make_tree_inputs, make_varlen_inputs, tree_parents)


def test_tree_parents_are_topological():
    for shape in ("random", "chain", "star", "kary4"):
        p = tree_parents(5, 40, shape, seed=3)
        assert p.dtype == torch.int32 and tuple(p.shape) == (5, 40)
        idx = torch.arange(40)
        assert bool(((p >= -1) & (p < idx)).all()), shape
    k = tree_parents(1, 21, "kary4")[0].tolist()
    assert k[0] == -1 and k[1:5] == [0] * 4 and k[5:9] == [1] * 4
    assert tree_parents(1, 6, "chain")[0].tolist() == [-1, 0, 1, 2, 3, 4]


def test_tree_inputs_shapes_and_determinism():
    a = make_tree_inputs(3, 17, 2, seed=9)
    b = make_tree_inputs(3, 17, 2, seed=9)
    assert tuple(a["q"].shape) == (3, 17, 2, 128) and a["q"].dtype == torch.bfloat16
    assert tuple(a["state"].shape) == (3, 2, 128, 128)
    assert bool(((a["accepted"] >= -1) & (a["accepted"] < 17)).all())
    for n in ("q", "k", "v", "g", "beta", "state", "parent", "accepted"):
        assert torch.equal(a[n], b[n]), n
    assert bool((a["g"] <= 0).all()) and bool(((a["beta"] > 0) & (a["beta"] < 1)).all())


def test_varlen_offsets_run_from_zero_to_t():
    lens = [0, 5, 64, 0, 130]
    v = make_varlen_inputs(L350M, lens, H=2, h0_std=0.1, dhT_std=0.1)
    cu = v["cu_seqlens"].tolist()
    assert cu == [0, 0, 5, 69, 69, 199]
    assert v["q"].shape[:2] == (1, 199) and tuple(v["h0"].shape) == (5, 2, 128, 128)
    assert tuple(v["dhT"].shape) == (5, 2, 128, 128)


def test_prologue_inputs():
    p = make_prologue_inputs(2, 33, 3, d=64, K=3, dtype="f32", seed=4)
    assert tuple(p["x"].shape) == (2, 33, 3, 64) and p["x"].dtype == torch.float32
    assert tuple(p["w"].shape) == (3, 64, 3) and p["w"].dtype == torch.float32
    assert torch.equal(p["x"], make_prologue_inputs(2, 33, 3, d=64, K=3, dtype="f32", seed=4)["x"])


def test_chunk_inputs_are_seeded():
    a = make_chunk_inputs(L350M, B=1, T=70, H=2, seed=5)
    b = make_chunk_inputs(L350M, B=1, T=70, H=2, seed=5)
    c = make_chunk_inputs(L350M, B=1, T=70, H=2, seed=6)
    assert torch.equal(a["k"], b["k"]) and not torch.equal(a["k"], c["k"])
    n = a["k"].float().pow(2).sum(-1)
    assert float((n - 1).abs().max()) < 2e-2  # L2-normalised before the bf16 cast
