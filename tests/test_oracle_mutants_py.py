"""Plant plausible mistakes in copies of the Python oracles (draft trees, the
q/k/v prologue, DeltaProduct) and check that their pins catch every one.  The
real sources are never modified: each mutant is a textual edit executed as a
separate module, swapped in for the oracle only inside the pin module under
test."""
import os
import types

import pytest

import oracle
import tests.test_oracle_product as product_pins
import tests.test_oracle_prologue as prologue_pins
import tests.test_oracle_tree as tree_pins

TREE = [
    ("root path taken leaf first", "    return path[::-1]", "    return path"),
    ("no decay along the path", "        S = S * np.exp(g[t])", "        S = S"),
    ("read-out before the node's own token",
     "S = _run_path(state[n, h], root_path(parent[n], i), k[n, :, h], v[n, :, h],",
     "S = _run_path(state[n, h], root_path(parent[n], i)[:-1], k[n, :, h], v[n, :, h],"),
    ("commit stops at the accepted node's parent",
     "        path = root_path(parent[n], a)", "        path = root_path(parent[n], a)[:-1]"),
    ("scale dropped from the read-out",
     "o[n, i, h] = scale * (S @ q[n, i, h])", "o[n, i, h] = S @ q[n, i, h]"),
    ("every earlier node treated as an ancestor", "        j = int(parent[j])", "        j = j - 1"),
    ("wrong sign of the prediction",
     "u = beta[t] * (v[t] - S @ k[t])", "u = beta[t] * (v[t] + S @ k[t])"),
]

PROLOGUE = [
    ("taps reversed", "w[:, :, j] * x[:, :T - j]", "w[:, :, K - 1 - j] * x[:, :T - j]"),
    ("filter looks ahead",
     "z[:, j:] = z[:, j:] + w[:, :, j] * x[:, :T - j]",
     "z[:, :T - j] = z[:, :T - j] + w[:, :, j] * x[:, j:]"),
    ("sigmoid in place of SiLU", "s = z * torch.sigmoid(z)", "s = torch.sigmoid(z)"),
    ("norm over the tokens", "(s * s).sum(-1, keepdim=True)", "(s * s).sum(1, keepdim=True)"),
    ("eps outside the square root",
     "torch.sqrt((s * s).sum(-1, keepdim=True) + EPS)",
     "(torch.sqrt((s * s).sum(-1, keepdim=True)) + EPS)"),
]

PRODUCT = [
    ("gate applied at every delta step",
     "        S = S * (a[:, :, None, :] if channel else a[:, :, None, None])\n        for j in range(n):\n",
     "        for j in range(n):\n            S = S * (a[:, :, None, :] if channel else a[:, :, None, None])\n"),
    ("beta of the first step reused", "bb = k[:, t, j], v[:, t, j], beta[:, t, j]",
     "bb = k[:, t, j], v[:, t, j], beta[:, t, 0]"),
    ("read-out after the first delta step only",
     "        outs.append(scale * torch.einsum(\"bhac,bhc->bha\", S, q[:, t]))",
     "        outs.append(scale * torch.einsum(\"bhac,bhc->bha\", S - torch.einsum(\"bha,bhc->bhac\", u, kk) if n > 1 else S, q[:, t]))"),
]


def _mutant(modname, old, new):
    path = os.path.join(os.path.dirname(oracle.__file__), f"{modname}.py")
    src = open(path).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    mod = types.ModuleType(f"oracle.{modname}_mutant")
    mod.__file__ = path
    exec(compile(src.replace(old, new), f"{path} (mutant)", "exec"), mod.__dict__)
    return mod


def _caught(pin_module, attr, mod, monkeypatch):
    monkeypatch.setattr(pin_module, attr, mod)
    caught = []
    for name in sorted(n for n in dir(pin_module) if n.startswith("test_")):
        try:
            getattr(pin_module, name)()
        except Exception:  # an assertion or a crash: the mistake did not pass
            caught.append(name)
    return caught


@pytest.mark.parametrize("name,old,new", TREE, ids=[m[0] for m in TREE])
def test_tree_pins_catch(monkeypatch, name, old, new):
    assert _caught(tree_pins, "tree", _mutant("tree", old, new), monkeypatch), name


@pytest.mark.parametrize("name,old,new", PROLOGUE, ids=[m[0] for m in PROLOGUE])
def test_prologue_pins_catch(monkeypatch, name, old, new):
    assert _caught(prologue_pins, "prologue", _mutant("prologue", old, new), monkeypatch), name


@pytest.mark.parametrize("name,old,new", PRODUCT, ids=[m[0] for m in PRODUCT])
def test_product_pins_catch(monkeypatch, name, old, new):
    assert _caught(product_pins, "product", _mutant("product", old, new), monkeypatch), name


@pytest.mark.parametrize("pins,attr,anchor", [
    (tree_pins, "tree", "    return path[::-1]"),
    (prologue_pins, "prologue", "s = z * torch.sigmoid(z)"),
    (product_pins, "product", "bb = k[:, t, j], v[:, t, j], beta[:, t, j]"),
], ids=["tree", "prologue", "product"])
def test_unmutated_copy_passes_every_pin(monkeypatch, pins, attr, anchor):
    """Control: the same machinery with no edit catches nothing."""
    assert _caught(pins, attr, _mutant(attr, anchor, anchor), monkeypatch) == []
