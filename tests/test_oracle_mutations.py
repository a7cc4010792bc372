"""The pins catch plausible mistakes: each case plants one mistake in a temporary
copy of the oracle's C source (on the CPU), rebuilds it, and requires that at
least one pin of tests/test_oracle_pins.py fails against the planted copy."""
import importlib.util
import inspect
import itertools
import os
import shutil
import sys

import pytest

import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "bias sign": ("        g -= c[i];", "        g += c[i];"),
    "predictor bias sign": ("        z[i] = acc - c[i];", "        z[i] = acc + c[i];"),
    "strict threshold": ("mask[i] = z[i] > threshold ? 1 : 0;", "mask[i] = z[i] >= threshold ? 1 : 0;"),
    "reglu drops relu": ("    if (act == OR_REGLU) return gp * u;", "    if (act == OR_REGLU) return g * u;"),
    "drelu keeps negative up": ("    double up = u > 0.0 ? u : 0.0;", "    double up = u;"),
    "transposed down": ("acc += h[i] * or_elem(wdtype, Wd, (long)j * F + i);",
                        "acc += h[i] * or_elem(wdtype, Wd, (long)i * d + j);"),
    "nibble order": ("int nib = (k % 2 == 0) ? (byte & 0xf) : (byte >> 4);",
                     "int nib = (k % 2 == 0) ? (byte >> 4) : (byte & 0xf);"),
    "nibble offset": ("* (double)(nib - 8);", "* (double)(nib - 7);"),
    "group size": ("or_half_to_double(scales[k / 32])", "or_half_to_double(scales[k / 16])"),
    "half exponent bias": ("ldexp(1.0 + (double)frac / 1024.0, expo - 15)",
                           "ldexp(1.0 + (double)frac / 1024.0, expo - 16)"),
    "rmsnorm eps outside": ("double inv = 1.0 / sqrt(ss / (double)d + eps);",
                            "double inv = 1.0 / (sqrt(ss / (double)d) + eps);"),
    "rmsnorm sum not mean": ("double inv = 1.0 / sqrt(ss / (double)d + eps);",
                             "double inv = 1.0 / sqrt(ss + eps);"),
    "tie to higher id": ("    return (a > b) - (a < b);", "    return (a < b) - (a > b);"),
    "no snake dealing": ("int b = (round % 2 == 0) ? k : S - 1 - k;", "int b = k;"),
    "router tie to higher": ("        if (p[e] > p[a]) a = e;", "        if (p[e] >= p[a]) a = e;"),
    "router no renorm": ("    weights[0] = p[lo] / (p[lo] + p[hi]);", "    weights[0] = p[lo];"),
    "predictor drops V": ("            acc += row[j] * x[j];\n        t[k] = acc;",
                          "            acc += x[j];\n        t[k] = acc;"),
    "int8 read unsigned": ("const int8_t *q = (const int8_t *)base + row * (long)n;",
                           "const uint8_t *q = (const uint8_t *)base + row * (long)n;"),
    "int8 scale of the wrong row": ("double s = (double)((const float *)scales)[row];",
                                    "double s = (double)((const float *)scales)[0];"),
    "down skips last neuron": ("        for (int i = 0; i < F; ++i) {\n                if (h[i] == 0.0)",
                               "        for (int i = 0; i < F - 1; ++i) {\n                if (h[i] == 0.0)"),
}

PIN_TESTS = [(n, f) for n, f in inspect.getmembers(pins, inspect.isfunction)
             if n.startswith("test_") and "oracle_mod" in inspect.signature(f).parameters]


def _planted(tmp_path, name, old, new):
    src = os.path.join(ROOT, "oracle")
    dst = tmp_path / "oracle_planted"
    shutil.copytree(src, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    c = (dst / "oracle.c").read_text()
    assert c.count(old) == 1, f"mutation '{name}' does not match the source exactly once"
    (dst / "oracle.c").write_text(c.replace(old, new))
    modname = "oracle_planted_" + "".join(ch if ch.isalnum() else "_" for ch in name)
    spec = importlib.util.spec_from_file_location(modname, dst / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    sys.modules[modname] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _params(f):
    grids = []
    for mk in getattr(f, "pytestmark", []):
        if mk.name == "parametrize":
            names = [n.strip() for n in mk.args[0].split(",")]
            grids.append([dict(zip(names, v if isinstance(v, tuple) else (v,))) for v in mk.args[1]])
    for combo in itertools.product(*grids):
        kw = {}
        for part in combo:
            kw.update(part)
        yield kw


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(tmp_path, name):
    old, new = MUTATIONS[name]
    mod = _planted(tmp_path, name, old, new)
    failed = []
    for tname, f in PIN_TESTS:
        for kw in _params(f):
            try:
                f(mod, **kw)
            except AssertionError:
                failed.append(tname)
                break
        if failed:
            break
    assert failed, f"no pin caught the planted mistake '{name}'"
