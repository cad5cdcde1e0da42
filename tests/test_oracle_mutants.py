"""The pins have teeth: each plausible mistake, planted in a copy of oracle.c
(CPU only), must make at least one pin in test_oracle_pins.py fail."""
import os
import subprocess
import tempfile

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, text in oracle.c, replacement, occurrence index) -- each a one-token mistake
MUTANTS = [
    ("score sign", "double z = scale * dot_d(q + (size_t)h * d, k, d);",
     "double z = -scale * dot_d(q + (size_t)h * d, k, d);", 0),
    ("group max -> last head", "if (z > best) best = z;", "best = z;", 0),
    ("group head index", "decode_row(Q + ((size_t)b * Hq + (size_t)kvh * g + h) * d",
     "decode_row(Q + ((size_t)b * Hq + (size_t)kvh + h) * d", 0),
    ("block-score head index", "decode_row(Q + ((size_t)b * Hq + (size_t)kvh * g + h) * d",
     "decode_row(Q + ((size_t)b * Hq + (size_t)h) * d", 1),
    ("sort direction", "if (a->s > b->s) return -1;", "if (a->s > b->s) return 1;", 0),
    ("tie-break to higher index", "return (a->j > b->j) - (a->j < b->j);",
     "return (a->j < b->j) - (a->j > b->j);", 0),
    ("output not ascending", "qsort(out, (size_t)kb, sizeof(int32_t), by_int);", ";", 0),
    ("attention scale dropped", "z[t] = scale * dot_d(q, kv, d);", "z[t] = dot_d(q, kv, d);", 0),
    ("softmax denominator", "den += w;", "den += 1.0;", 0),
    ("V row index", "decode_row(Vb + (size_t)rows[t] * d, kv, d);",
     "decode_row(Vb + (size_t)t * d, kv, d);", 0),
    ("GQA head mapping", "const int h = kvh * g + hh;", "const int h = hh * Hkv + kvh;", 0),
    ("block mean divisor", "/ (double)(t1 - t0);", "/ (double)block;", 0),
    ("block expansion offset", "int t0 = e * block, t1 = e * block + block;",
     "int t0 = e, t1 = e + block;", 0),
    ("negative padding", "for (int t = kb; t < k_max; ++t) out[t] = -1;",
     "for (int t = kb; t < k_max; ++t) out[t] = 0;", 0),
]

PIN_TESTS = [(n, f) for n, f in vars(pins).items() if n.startswith("test_") and callable(f)]


def _call(f):
    import inspect

    params = inspect.signature(f).parameters
    if "seed" in params:
        for s in range(3):
            f(seed=s)
    elif "Hq" in params:
        for hq, hkv in [(8, 2), (4, 4), (8, 1)]:
            f(Hq=hq, Hkv=hkv)
    else:
        f()


def _replace_nth(text, old, new, n):
    pos = -1
    for _ in range(n + 1):
        pos = text.index(old, pos + 1)
    return text[:pos] + new + text[pos + len(old):]


@pytest.mark.parametrize("name,old,new,nth", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, nth, tmp_path):
    src = open(SRC).read()
    assert src.count(old) > nth, f"mutation site for {name!r} not found"
    bad = tmp_path / "mutant.c"
    bad.write_text(_replace_nth(src, old, new, nth))
    so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", str(bad), "-o",
                           str(so), "-lm"])
    caught = []
    with oracle.use_library(str(so)):
        for tname, f in PIN_TESTS:
            try:
                _call(f)
            except (AssertionError, ValueError):
                caught.append(tname)
    assert caught, f"no pin rejects the mutant {name!r}"


def test_unmutated_oracle_passes_every_pin():
    for _, f in PIN_TESTS:
        _call(f)


# The numpy parts of the oracle: (name, function, text in its source, replacement)
PY_MUTANTS = [
    ("overlap normalised by the source set", "index_overlap",
     "counts[i, j, u] / sets[j][u].size", "counts[i, j, u] / sets[i][u].size"),
    ("overlap keeps empty targets", "index_overlap",
     "for u in range(units) if sets[j][u].size > 0]", "for u in range(units) if True]"),
    ("overlap matrix transposed", "index_overlap", "M[j, i] = float(np.mean(ratios))",
     "M[i, j] = float(np.mean(ratios))"),
    ("overlap counts the -1 padding", "index_overlap", "a[l, u][a[l, u] >= 0]", "a[l, u]"),
    ("overlap of no units is 0", "index_overlap", "if ratios else 1.0", "if ratios else 0.0"),
    ("policy threshold not strict", "reuse_policy", "not M[j, cur] > theta", "not M[j, cur] >= theta"),
    ("policy ignores similarity", "reuse_policy", "key = (sum(full), -sim, src[::-1])",
     "key = (sum(full), src[::-1])"),
    ("policy minimises similarity", "reuse_policy", "key = (sum(full), -sim, src[::-1])",
     "key = (sum(full), sim, src[::-1])"),
    ("policy ties read forwards", "reuse_policy", "key = (sum(full), -sim, src[::-1])",
     "key = (sum(full), -sim, src)"),
    ("policy ignores forced layers", "reuse_policy",
     "forced = [j == 0 or (force_full is not None and bool(force_full[j])) for j in range(L)]",
     "forced = [j == 0 for j in range(L)]"),
    ("policy reads M transposed", "reuse_policy", "not M[j, cur] > theta", "not M[cur, j] > theta"),
]


@pytest.mark.parametrize("name,fn,old,new", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_python_mutant_is_caught(name, fn, old, new, monkeypatch):
    import inspect
    import warnings

    src = inspect.getsource(getattr(oracle, fn))
    assert src.count(old) == 1, f"mutation site for {name!r} not found once"
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    monkeypatch.setattr(oracle, fn, ns[fn])
    caught = []
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        for tname, f in PIN_TESTS:
            try:
                _call(f)
            except Exception:  # a failed pin, or a mutant that cannot even run
                caught.append(tname)
    assert caught, f"no pin rejects the mutant {name!r}"
