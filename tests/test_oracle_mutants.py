"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of oracle/moe_oracle.c, builds it, and
runs tests/test_oracle_pins.py against the broken build (ORACLE_LIB); the pins
must fail.  The mistakes are the kind a re-implementation makes: a sign, an
operand swap, a transposed index, a dropped term, a wrong constant, a wrong
order."""
import concurrent.futures
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "silu sign": ("double a = g[i] / (1.0 + exp(-g[i]));", "double a = g[i] / (1.0 + exp(g[i]));"),
    "W1/W3 swapped": ("g[i] += xj * w1[i]; u[i] += xj * w3[i];", "g[i] += xj * w3[i]; u[i] += xj * w1[i];"),
    "W2 transposed": ("for (int64_t c = 0; c < d; ++c) o[c] += hi * w2[c];",
                      "for (int64_t c = 0; c < d; ++c) o[c] += hi * W2[c * I + i];"),
    "gate transposed": ("acc += x[t * d + j] * Wg[e * d + j];", "acc += x[t * d + j] * Wg[j * E + e];"),
    "shared expert dropped": ("    if (Is > 0)\n        for (int64_t t = 0; t < T; ++t) {",
                              "    if (0)\n        for (int64_t t = 0; t < T; ++t) {"),
    "routing weight dropped": ("for (int64_t c = 0; c < d; ++c) y[t * d + c] += w[t * k + j] * o[c];",
                               "for (int64_t c = 0; c < d; ++c) y[t * d + c] += o[c];"),
    "ties to highest index": ("return (va > vb) || (va == vb && ia < ib);", "return (va > vb) || (va == vb && ia > ib);"),
    "e4m3 bias 8": ("v = ldexp(1.0 + (double)mant / 8.0, expo - 7);", "v = ldexp(1.0 + (double)mant / 8.0, expo - 8);"),
    "dispatch in slot order": ("    for (int e = 0; e < E; ++e)\n        for (int64_t t = 0; t < T; ++t)\n            for (int j = 0; j < k; ++j)",
                               "    for (int e = 0; e < E; ++e)\n        for (int j = 0; j < k; ++j)\n            for (int64_t t = 0; t < T; ++t)"),
    "group weights unnormalised": ("w[t * k + j] = route_scale * s[top[j]] / den;", "w[t * k + j] = route_scale * s[top[j]];"),
    "group score top-1": ("for (int i = 0; i < group_topn; ++i) acc += sel[inner[i]];",
                          "for (int i = 0; i < group_topn; ++i) acc = sel[inner[i]];"),
    "softmax not shifted by max": ("den += exp(l[top[j]] - l[top[0]]);", "den += exp(l[top[j]] - l[top[1 % k]]);"),
    "expert-parallel rank skips its first expert": ("if (e < e_lo || e >= e_lo + El) continue;",
                                                    "if (e <= e_lo || e >= e_lo + El) continue;"),
    "expert-parallel rank drops its shared slice": ("    if (Isl > 0)\n", "    if (0)\n"),
    "top-k gap taken against slot j+2": ("gaps[t * k + j] = (j + 1 < m) ? l[top[j]] - l[top[j + 1]] : INFINITY;",
                                         "gaps[t * k + j] = (j + 2 < m) ? l[top[j]] - l[top[j + 2]] : INFINITY;"),
    "group slot gap on unbiased scores": ("gaps[t * k + j] = (j + 1 < m) ? sel[top[j]] - sel[top[j + 1]] : INFINITY;",
                                          "gaps[t * k + j] = (j + 1 < m) ? s[top[j]] - s[top[j + 1]] : INFINITY;"),
    "group-boundary gap against the wrong group": (
        "gscore_gap[t] = (topk_group < n_group) ? gscore[gtop[topk_group - 1]] - gscore[gtop[topk_group]]",
        "gscore_gap[t] = (topk_group < n_group) ? gscore[gtop[topk_group - 2]] - gscore[gtop[topk_group]]"),
    "group weight rule without the scale": (
        "for (int j = 0; j < k; ++j) w[t * k + j] = route_scale * (1.0 / (1.0 + exp(-l[idx[t * k + j]]))) / den;",
        "for (int j = 0; j < k; ++j) w[t * k + j] = (1.0 / (1.0 + exp(-l[idx[t * k + j]]))) / den;"),
    "combine drops shared": ("        if (Ys)\n            for (int64_t c = 0; c < d; ++c) yt[c] += Ys[t * d + c];",
                             "        if (0)\n            for (int64_t c = 0; c < d; ++c) yt[c] += Ys[t * d + c];"),
}


def _build_and_run(name, tmpdir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    tag = "".join(ch if ch.isalnum() else "_" for ch in name)
    c_path = os.path.join(tmpdir, f"mut_{tag}.c")
    so_path = os.path.join(tmpdir, f"libmut_{tag}.so")
    with open(c_path, "w") as f:
        f.write(src.replace(old, new))
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-o", so_path, c_path, "-lm"],
                   check=True)
    env = dict(os.environ, ORACLE_LIB=so_path, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-q", "-x",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode, r.stdout[-400:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with concurrent.futures.ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(lambda n: _build_and_run(n, str(tmp_path)), MUTANTS))
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
    for n, rc, out in results:
        assert rc == 1, (n, rc, out)   # 1 = tests failed (not a crash or collection error)
