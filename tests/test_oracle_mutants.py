"""The oracle's pins catch plausible mistakes: each test plants one mistake in
a private copy of the oracle's source (CPU only; the oracle file itself is
never changed), runs the pins of tests/test_oracle_pins.py against the copy,
and requires at least one pin to fail.  An unchanged copy must pass them all.
"""
import os
import types

import pytest

import tests.test_oracle_pins as pins

SRC_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "oracle", "pisa_oracle.py")
with open(SRC_PATH) as f:
    SRC = f.read()

# (mistake, text in the oracle, planted text); each text occurs exactly once
MUTANTS = [
    ("dropped n_j in the denominator",
     "D = p_exact.sum(axis=1) + alpha @ counts[U].astype(np.float64)",
     "D = p_exact.sum(axis=1) + alpha.sum(axis=1)"),
    ("transposed Hbar in the first-order term",
     "Nt = Nt + (scale * (qi @ hbar))", "Nt = Nt + (scale * (qi @ hbar.T))"),
    ("sign of the first-order term",
     "Nt = Nt + (scale * (qi @ hbar))", "Nt = Nt - (scale * (qi @ hbar))"),
    ("first-order term without the softmax scale",
     "Nt = Nt + (scale * (qi @ hbar))", "Nt = Nt + (qi @ hbar)"),
    ("Hbar divided by L instead of N",
     "hbar = H.sum(axis=0) / N", "hbar = H.sum(axis=0) / L"),
    ("ties to the higher block index",
     "order = np.lexsort((j, -scores[r]))", "order = np.lexsort((-j, -scores[r]))"),
    ("mean instead of sum of the values",
     "vsum[j] = v[sl].sum(axis=0)", "vsum[j] = v[sl].sum(axis=0) / counts[j]"),
    ("centroid logits without the softmax scale",
     "lg_tail = scale * (qi @ kbar[U].T)", "lg_tail = qi @ kbar[U].T"),
    ("H_j without centring the keys",
     "delta = k[sl] - kbar[j]", "delta = k[sl]"),
    ("sink not forced",
     "chosen = np.concatenate([[sink], others])", "chosen = order[:k_sel]"),
    ("k_sel rounded up",
     "math.floor(density * N + 1e-6)", "math.ceil(density * N - 1e-6)"),
    ("covariance norm squared",
     "M[j] = math.sqrt(float(((Hj - hbar) ** 2).sum()))", "M[j] = float(((Hj - hbar) ** 2).sum())"),
    ("covariance norm of H_j, not of H_j - Hbar",
     "M[j] = math.sqrt(float(((Hj - hbar) ** 2).sum()))", "M[j] = math.sqrt(float((Hj ** 2).sum()))"),
    ("covariance weight ignored",
     "sc = sc + cov_weight * cov[None, :]", "sc = sc + 0.0 * cov[None, :]"),
    ("histogram: a value equal to hi kept in the last bin",
     "h[-1] += int((vals >= hi).sum())", "h[-1] += int((vals > hi).sum())"),
    ("histogram: deviations not centred",
     "y = scale * (qi @ (kb - kb.mean(axis=0)).T)", "y = scale * (qi @ kb.T)"),
    ("first block of the exact phase dropped",
     "ex = np.concatenate([np.arange(starts[j], starts[j] + counts[j]) for j in S])",
     "ex = np.concatenate([np.arange(starts[j], starts[j] + counts[j]) for j in S[1:]]"
     " + [np.zeros(0, dtype=np.int64)])"),
]


def _module(src, name):
    mod = types.ModuleType(name)
    exec(compile(src, name, "exec"), mod.__dict__)
    return mod


def _cases(fn):
    """Every argument combination of a pin's parametrize marks."""
    combos = [{}]
    for m in getattr(fn, "pytestmark", []):
        if m.name != "parametrize":
            continue
        names = m.args[0]
        names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
        new = []
        for c in combos:
            for val in m.args[1]:
                val = tuple(val) if len(names) > 1 else (val,)
                new.append({**c, **dict(zip(names, val))})
        combos = new
    return combos


def _pins():
    return [(n, getattr(pins, n)) for n in sorted(dir(pins))
            if n.startswith("test_") and callable(getattr(pins, n))]


def _first_failure(mod, monkeypatch, stop_at_first=True):
    monkeypatch.setattr(pins, "O", mod)
    failed = []
    for name, fn in _pins():
        for case in _cases(fn):
            try:
                fn(**case)
            except Exception:   # an assertion, or the mistake breaking a shape
                failed.append(name)
                if stop_at_first:
                    return failed
                break
    return failed


def test_unchanged_copy_passes_every_pin(monkeypatch):
    assert _first_failure(_module(SRC, "oracle_copy"), monkeypatch, False) == []


@pytest.mark.parametrize("what,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(monkeypatch, what, old, new):
    assert SRC.count(old) == 1, f"mutation site not unique: {old}"
    mod = _module(SRC.replace(old, new), "oracle_mutant")
    assert _first_failure(mod, monkeypatch), f"no pin catches: {what}"


# ---- the gradient oracle (oracle/pisa_backward.py) and its pins ----------------

import oracle as _O  # noqa: E402
import tests.test_oracle_backward_pins as bpins  # noqa: E402

BWD_PATH = os.path.join(os.path.dirname(SRC_PATH), "pisa_backward.py")
with open(BWD_PATH) as f:
    BWD_SRC = f.read().replace("from .pisa_oracle import", "from oracle.pisa_oracle import")

BWD_MUTANTS = [
    ("centroid as the key sum",
     "k[starts[j]:starts[j] + counts[j]].mean(dim=0)", "k[starts[j]:starts[j] + counts[j]].sum(dim=0)"),
    ("value mean instead of value sum",
     "v[starts[j]:starts[j] + counts[j]].sum(dim=0)", "v[starts[j]:starts[j] + counts[j]].mean(dim=0)"),
    ("dropped n_j in the denominator",
     "D = p_exact.sum(dim=1) + alpha @ n_j[U]", "D = p_exact.sum(dim=1) + alpha.sum(dim=1)"),
    ("lse without the factored maximum",
     "lses.append(m + torch.log(D))", "lses.append(torch.log(D))"),
    ("centroid logits without the softmax scale",
     "lg_tail = scale * (qi @ kbar[U].T)", "lg_tail = qi @ kbar[U].T"),
    ("statistics not differentiated",
     "for j in range(N)])\n    vsum", "for j in range(N)]).detach()\n    vsum"),
    ("dout rows paired in reverse",
     "(out * g[torch.as_tensor(rows)]).sum().backward()",
     "(out * g[torch.as_tensor(rows)].flip(0)).sum().backward()"),
]


def _bwd_namespace(src):
    mod = _module(src, "oracle_backward_copy")
    ns = types.SimpleNamespace(**{n: getattr(_O, n) for n in dir(_O) if not n.startswith("_")})
    ns.zeroth_order_backward = mod.zeroth_order_backward
    ns.zeroth_order_forward = mod.zeroth_order_forward
    return ns


def _bwd_failures(ns, monkeypatch, stop_at_first=True):
    monkeypatch.setattr(bpins, "O", ns)
    failed = []
    for name in sorted(dir(bpins)):
        fn = getattr(bpins, name)
        if not (name.startswith("test_") and callable(fn)):
            continue
        for case in _cases(fn):
            try:
                fn(**case)
            except Exception:
                failed.append(name)
                if stop_at_first:
                    return failed
                break
    return failed


def test_unchanged_gradient_oracle_copy_passes_every_pin(monkeypatch):
    assert _bwd_failures(_bwd_namespace(BWD_SRC), monkeypatch, False) == []


@pytest.mark.parametrize("what,old,new", BWD_MUTANTS, ids=[m[0] for m in BWD_MUTANTS])
def test_planted_gradient_mistake_fails_a_pin(monkeypatch, what, old, new):
    assert BWD_SRC.count(old) == 1, f"mutation site not unique: {old}"
    assert _bwd_failures(_bwd_namespace(BWD_SRC.replace(old, new)), monkeypatch), \
        f"no pin catches: {what}"
