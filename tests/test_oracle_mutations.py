"""The oracle's pins reject planted mistakes (CPU only).

Each case writes one plausible slip into a copy of an oracle source file -- a
dropped term, a wrong sign, a swapped index or operand, a wrong tie rule --
and runs every pin of that file against the copy; at least one pin must fail
with an assertion.  The copy is executed as a separate module and replaces the
oracle only inside the pin module's namespace for one case, so the oracle
itself is never modified.  A case whose mutation site no longer occurs exactly
once in the source fails, so an edit of the oracle that moves a site is
noticed here.
"""
import importlib
import os
import types
from dataclasses import dataclass

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle")


@dataclass(frozen=True)
class Slip:
    name: str
    src: str        # oracle file
    pins: str       # pin module under tests/
    handle: str     # the pin module's global that refers to the oracle
    old: str
    new: str


TILEQ = ("tileq.py", "test_oracle", "oracle")
SKETCH = ("sketch.py", "test_sketch_oracle", "sketch")
PLACE = ("placement.py", "test_placement_oracle", "P")

SLIPS = [
    # stored format
    Slip("bf16 widening shifted by one bit", *TILEQ,
         "<< np.uint32(16)", "<< np.uint32(15)"),
    Slip("code fields read from the top of the word", *TILEQ,
         "shifts = (2 * np.arange(16, dtype=np.uint32))",
         "shifts = (30 - 2 * np.arange(16, dtype=np.uint32))"),
    Slip("zero points read four bits apart", *TILEQ,
         "(4, 2, 3) if bits != 3", "(2, 4, 3) if bits != 3"),
    Slip("zero point added instead of subtracted", *TILEQ,
         "w = (q - z[:, :, None]) * s[:, :, None]", "w = (q + z[:, :, None]) * s[:, :, None]"),
    Slip("groups strided across the row instead of contiguous", *TILEQ,
         "q = q.reshape(proj.d_out, G, g)", "q = q.reshape(proj.d_out, g, G).transpose(0, 2, 1)"),
    Slip("3-bit high plane weighted 2 instead of 4", *TILEQ,
         "q = q + 4 * unpack_codes_hi", "q = q + 2 * unpack_codes_hi"),
    Slip("3-bit zero points masked to two bits", *TILEQ,
         "else (2, 4, 7)", "else (2, 4, 3)"),
    # routing and permutation
    Slip("ties go to the higher expert id", *TILEQ,
         "key=lambda e: (-float(lg[t, e]), e)", "key=lambda e: (-float(lg[t, e]), -e)"),
    Slip("NaN logits not ranked as -inf", *TILEQ,
         "lg = np.where(np.isnan(lg), -np.inf, lg)", "lg = lg"),
    Slip("default weights not renormalised over the chosen k", *TILEQ,
         "            w[t] = ex / ex.sum()",
         "            w[t] = ex / np.exp(lg[t] - vals.max()).sum()"),
    Slip("full-softmax variant renormalised over the chosen k", *TILEQ,
         "every = np.exp(lg[t] - vals.max())", "every = ex"),
    Slip("layer forward ignores the routing variant", *TILEQ,
         'idx, w = route(lg[toks], layer.top_k, getattr(layer, "route_mode", 0) == 1)',
         "idx, w = route(lg[toks], layer.top_k)"),
    Slip("batched forward ignores the routing variant", *TILEQ,
         'idx, w = route(lg, layer.top_k, getattr(layer, "route_mode", 0) == 1)',
         "idx, w = route(lg, layer.top_k)"),
    Slip("permutation not stable within an expert", *TILEQ,
         "for p, e in enumerate(flat):", "for p, e in reversed(list(enumerate(flat))):"),
    # the 2D-tiled low-rank term
    Slip("placement ignored: expert e taken at cell e", *TILEQ,
         "cell = int(proj.grid_assign[e])", "cell = int(e)"),
    Slip("Sigma dropped from the expert's low-rank block", *TILEQ,
         "return (Um * sig[None, :]) @ Vn.T", "return Um @ Vn.T"),
    Slip("Sigma applied on the wrong side (as Sigma^2 on U)", *TILEQ,
         "return (U * sig[None, :]) @ V.T", "return (U * (sig * sig)[None, :]) @ V.T"),
    Slip("low-rank term left out of the expert weight", *TILEQ,
         "return lowrank_block(proj, e, N) + dequant(proj, e)", "return dequant(proj, e)"),
    # the layer
    Slip("silu with the wrong sign in the exponent", *TILEQ,
         "return a / (1.0 + np.exp(-a))", "return a / (1.0 + np.exp(a))"),
    Slip("SwiGLU gates the up projection instead of the gate", *TILEQ,
         "h = silu(cache.get(0, e) @ xt) * (cache.get(1, e) @ xt)",
         "h = (cache.get(0, e) @ xt) * silu(cache.get(1, e) @ xt)"),
    Slip("routing weight not applied in the combine", *TILEQ,
         "out[i] += w[i, j] * y", "out[i] += y"),
    Slip("shared expert scaled by the first routing weight", *TILEQ,
         "out[i] += _shared_expert(layer, xt)", "out[i] += w[i, 0] * _shared_expert(layer, xt)"),
    Slip("shared expert's up and gate swapped", *TILEQ,
         "return Wd @ (silu(Wg @ xt) * (Wu @ xt))", "return Wd @ (silu(Wu @ xt) * (Wg @ xt))"),
    Slip("shared expert's down projection applied transposed", *TILEQ,
         'Wd = widen_bf16(sh["down"])\n', 'Wd = widen_bf16(sh["down"]).T\n'),
    Slip("batched form gates the up projection", *TILEQ,
         "H = silu(G) * Uu", "H = G * silu(Uu)"),
    # Gaussian-sketch decomposition
    Slip("sketch basis not orthonormalised", *SKETCH,
         "q, _ = np.linalg.qr(y)", "q = y"),
    Slip("sketch keeps the smallest singular triplets", *SKETCH,
         "return q @ ub[:, :r], s[:r], vbt[:r].T", "return q @ ub[:, -r:], s[-r:], vbt[-r:].T"),
    Slip("sketch V taken from columns of V^T", *SKETCH,
         "vbt[:r].T", "vbt[:, :r]"),
    Slip("W_big block row and column swapped", *SKETCH,
         "m, n = divmod(int(grid_assign[k]), N)", "n, m = divmod(int(grid_assign[k]), M)"),
    # placement
    Slip("sign convention reversed", *PLACE,
         "if f[i, j] < 0:", "if f[i, j] > 0:"),
    Slip("embedding flattened column-major", *PLACE,
         "e = canonical_signs(f).reshape(-1)", "e = canonical_signs(f).T.reshape(-1)"),
    Slip("embedding not normalised", *PLACE,
         "return e / n if n > 0 else e", "return e"),
    Slip("farthest-first takes the last of equal distances", *PLACE,
         "if mind[i] > mind[best]:", "if mind[i] >= mind[best]:"),
    Slip("K-Means assignment ties go to the highest centre", *PLACE,
         "lab[i] = int(np.argmin(d))", "lab[i] = C - 1 - int(np.argmin(d[::-1]))"),
    Slip("K-Means centres moved to the median", *PLACE,
         "centres[j] = members.mean(axis=0)", "centres[j] = np.median(members, axis=0)"),
    Slip("greedy allocation by L1 grid distance", *PLACE,
         "d = (m - int(ideal_m[k])) ** 2 + (n - int(ideal_n[k])) ** 2",
         "d = abs(m - int(ideal_m[k])) + abs(n - int(ideal_n[k]))"),
    Slip("greedy allocation lets two experts share a cell", *PLACE,
         "if grid[k] < 0 and free[cell]:", "if grid[k] < 0:"),
]


def _copy_of(src: str, old: str = "", new: str = ""):
    path = os.path.join(ORACLE, src)
    with open(path) as f:
        text = f.read()
    if old:
        assert text.count(old) == 1, f"mutation site not found exactly once in oracle/{src}: {old!r}"
        text = text.replace(old, new)
    mod = types.ModuleType("oracle._planted")
    mod.__file__ = path
    mod.__package__ = "oracle"
    exec(compile(text, path, "exec"), mod.__dict__)
    return mod


def _pins(module):
    """Every pin of a pin module as (id, function, kwargs), parametrized cases expanded."""
    for name, fn in sorted(vars(module).items()):
        if not name.startswith("test_") or not callable(fn):
            continue
        marks = getattr(fn, "pytestmark", [])
        par = [m for m in marks if m.name == "parametrize"]
        if not par:
            yield name, fn, {}
            continue
        assert len(par) == 1, name
        argnames, argvalues = par[0].args[0], par[0].args[1]
        names = [s.strip() for s in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
        for vals in argvalues:
            vals = getattr(vals, "values", vals)
            if len(names) == 1 and not isinstance(vals, tuple):
                vals = (vals,)
            yield f"{name}{list(vals)}", fn, dict(zip(names, vals))


def _run_pins(pin_module, handle, oracle_copy, monkeypatch):
    mod = importlib.import_module(pin_module)
    monkeypatch.setattr(mod, handle, oracle_copy)
    failed, errors = [], []
    for pid, fn, kwargs in _pins(mod):
        try:
            fn(**kwargs)
        except AssertionError:
            failed.append(pid)
        except Exception as e:          # noqa: BLE001 -- reported, not counted
            errors.append(f"{pid}: {type(e).__name__}")
    return failed, errors


@pytest.mark.parametrize("src,pins,handle", [TILEQ, SKETCH, PLACE], ids=["tileq", "sketch", "placement"])
def test_unchanged_copy_passes_every_pin(src, pins, handle, monkeypatch):
    failed, errors = _run_pins(pins, handle, _copy_of(src), monkeypatch)
    assert not failed and not errors, (failed, errors)


@pytest.mark.parametrize("slip", SLIPS, ids=[s.name for s in SLIPS])
def test_pins_reject_planted_mistake(slip, monkeypatch):
    failed, errors = _run_pins(slip.pins, slip.handle, _copy_of(slip.src, slip.old, slip.new), monkeypatch)
    assert failed, f"no pin in tests/{slip.pins}.py rejects: {slip.name} (errors: {errors})"
