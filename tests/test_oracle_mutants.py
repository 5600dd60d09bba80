"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of the oracle's C source (never in the
oracle itself), builds it into a temporary library, and runs the pin tests
against that library: at least one pin must fail. This checks that the pins
constrain every step of the oracle -- a dropped term, a wrong index or sign,
a transposed tie rule or an off-by-one would not pass unnoticed.
"""
import os
import subprocess
import sys

import pytest

from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

MUTANTS = [
    ("bf16 rounding: ties away from zero", "double r = nearbyint(scaled);", "double r = round(scaled);"),
    ("seeding: stride off by one", "const float *k = keys + (size_t)c * stride * d;",
     "const float *k = keys + (size_t)(c * stride + 1) * d;"),
    ("assignment: ties to the highest index", "            if (s > best) {", "            if (s >= best) {"),
    ("assignment: last channel dropped", "for (int t = 0; t < d; ++t) s += (double)a[t] * b[t];",
     "for (int t = 0; t < d - 1; ++t) s += (double)a[t] * b[t];"),
    ("update: mean over n+1",
     "for (int t = 0; t < d; ++t) mu[(size_t)c * d + t] = sum[(size_t)c * d + t] / (double)cnt[c];",
     "for (int t = 0; t < d; ++t) mu[(size_t)c * d + t] = sum[(size_t)c * d + t] / (double)(cnt[c] + 1);"),
    ("update: empty cluster not kept", "        if (cnt[c] == 0) continue;",
     "        if (cnt[c] == 0) { for (int t = 0; t < d; ++t) mu[(size_t)c * d + t] = 0.0; continue; }"),
    ("update: unit copy not normalised", "muhat[t] = nrm > 0.0 ? round_to(mu[t] / nrm, mode) : 0.0;",
     "muhat[t] = round_to(mu[t], mode);"),
    ("index: descending positions inside a cluster",
     "for (int i = 0; i < n; ++i) perm[next[labels[i]]++] = tok_begin + i;",
     "for (int i = n - 1; i >= 0; --i) perm[next[labels[i]]++] = tok_begin + i;"),
    ("index: offsets start at 1", "    offsets[0] = perm_base;", "    offsets[0] = perm_base + 1;"),
    ("score: last butterfly step dropped", "for (int o = 16; o >= 1; o >>= 1) {",
     "for (int o = 16; o >= 2; o >>= 1) {"),
    ("score: only the first query head", "tot = (g == 0) ? h : tot + h;", "tot = (g == 0) ? h : tot;"),
    ("selection: no trimming of the last cluster",
     "int take = n_c <= budget - taken ? n_c : budget - taken;", "int take = n_c;"),
    ("selection: ties to the higher cluster id", "return (x->c > y->c) - (x->c < y->c);",
     "return (x->c < y->c) - (x->c > y->c);"),
    ("attention: scale applied twice", "logit[j] = scale * s;", "logit[j] = scale * scale * s;"),
    ("L2: distance with a plus sign", "double e = (double)k[t] - m[t];",
     "double e = (double)k[t] + m[t];"),
    ("L2: inner product used instead", "    if (metric != CKVO_METRIC_L2) return dot_d(k, m, d);",
     "    return dot_d(k, m, d);"),
    ("variants: assignment copy not rounded",
     "for (int t = 0; t < d; ++t) out[t] = round_to(mu[t], mode);",
     "for (int t = 0; t < d; ++t) out[t] = mu[t];"),
    ("variants: zero mean kept under every similarity",
     "if (metric == CKVO_METRIC_COSINE && ss == 0.0) continue;", "if (ss == 0.0) continue;"),
    ("cache: one step too long a window", "int cached = R > 0 && last[c] < step && last[c] >= step - R;",
     "int cached = R > 0 && last[c] < step && last[c] >= step - R - 1;"),
    ("cache: selection not recorded", "    for (int j = 0; j < n; ++j) last[clusters[j]] = step;",
     "    for (int j = 0; j + 1 < n; ++j) last[clusters[j]] = step;"),
    ("selected clusters: empty clusters listed", "        if (n_c == 0) continue;\n        int take",
     "        int take"),
    ("attended set: recent window one token short", "for (int j = tail_begin; j < tail_end; ++j) rows[n++] = j;",
     "for (int j = tail_begin; j < tail_end - 1; ++j) rows[n++] = j;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = open(oracle_build.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old}"
    mutated = tmp_path / "ckv_oracle_mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = oracle_build.build(force=True, out=str(tmp_path / "libmutant.so"), src=str(mutated))
    env = dict(os.environ, CKV_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, "test_oracle_pins.py"),
                        "-x", "-q", "-p", "no:cacheprovider"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"the pins did not catch: {name}\n{r.stdout[-2000:]}"
