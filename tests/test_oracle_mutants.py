"""Planted mistakes in the oracle are caught by its pins.

Each case copies oracle.c, replaces one ordering detail with a plausible
mistake (another summation order, another leaf size, eps outside the square
root, ...), compiles the copy with the oracle's flags and checks that the
matching ordering probe (tests/ordering_probes.py, expected values derived by
hand in tests/golden/ordering_probes.json) rejects it.  The unmodified oracle
passes every probe (tests/test_oracle_pins.py).  CPU only.
"""
import os
import shutil

import pytest

import oracle
from tests import ordering_probes as probes

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")

# (name, original text, planted mistake, probe that must fail)
MUTANTS = [
    ("baseline combine by the tree",
     "C[(size_t)i * N + n] = seq_f32(Q, 0, T);",
     "C[(size_t)i * N + n] = tree_f32(Q, 0, T);",
     "baseline_shard_sum"),
    ("baseline combine right to left",
     "float acc = P[lo];\n    for (int i = 1; i < n; ++i) acc = acc + P[lo + i];",
     "float acc = P[lo + n - 1];\n    for (int i = n - 2; i >= 0; --i) acc = acc + P[lo + i];",
     "baseline_shard_sum"),
    ("logprob baseline logits summed right to left",
     "for (int t = 0; t < T; ++t) {\n                    float acc = 0.0f;\n"
     "                    for (int k = t * Hs; k < (t + 1) * Hs; ++k) acc = fmaf(bf(h[k]), bf(w[k]), acc);\n"
     "                    sum = t ? sum + acc : acc;",
     "for (int t = T - 1; t >= 0; --t) {\n                    float acc = 0.0f;\n"
     "                    for (int k = t * Hs; k < (t + 1) * Hs; ++k) acc = fmaf(bf(h[k]), bf(w[k]), acc);\n"
     "                    sum = (t == T - 1) ? acc : sum + acc;",
     "logprob_baseline_logit_sum"),
    ("rmsnorm eps outside the square root",
     "float inv = 1.0f / sqrtf(ms + eps);",
     "float inv = 1.0f / (sqrtf(ms) + eps);",
     "rmsnorm_cancellation"),
    ("rmsnorm mean over H - 1",
     "float ms = ss / (float)H;",
     "float ms = ss / (float)(H - 1);",
     "rmsnorm_cancellation"),
    ("rmsnorm leaves of 4 elements",
     "int nl = H / 8;\n    float* r",
     "int nl = H / 4;\n    float* r",
     "rmsnorm_cancellation"),
    ("rmsnorm leaves of 16 elements",
     "int nl = H / 8;\n    float* r",
     "int nl = H / 16;\n    float* r",
     "rmsnorm_cancellation"),
    ("rmsnorm leaves summed left to right",
     "for (int s = 0; s < T; ++s) Q[s] = tree_f32(P, s * (nl / T), nl / T);",
     "for (int s = 0; s < T; ++s) Q[s] = seq_f32(P, s * (nl / T), nl / T);",
     "rmsnorm_cancellation"),
    ("rmsnorm residual input dropped",
     "for (int h = 0; h < H; ++h) r[h] = bf(xr[h]) + bf(rr[h]);",
     "for (int h = 0; h < H; ++h) r[h] = bf(xr[h]) + 0.0f * bf(rr[h]);",
     "rmsnorm_cancellation"),
    ("vocab leaf summed in descending column order",
     "for (int c = c0; c < c1; ++c) s = s + exp_spec(z[c] - m);",
     "for (int c = c1 - 1; c >= c0; --c) s = s + exp_spec(z[c] - m);",
     "vocab_leaf_ascending_sum"),
    ("vocab leaf as two interleaved partial sums",
     "for (int c = c0; c < c1; ++c) s = s + exp_spec(z[c] - m);",
     "float s1 = 0.0f;\n            for (int c = c0; c < c1; ++c) {\n"
     "                if ((c - c0) & 1) s1 = s1 + exp_spec(z[c] - m); else s = s + exp_spec(z[c] - m);\n"
     "            }\n            s = s + s1;",
     "vocab_leaf_ascending_sum"),
]


def _leaf_edit(src, width):
    """The leaf-size mutants also change the element loop of a leaf."""
    old = "for (int e = 0; e < 8; ++e) acc = fmaf(r[8 * j + e], r[8 * j + e], acc);"
    assert src.count(old) == 1
    return src.replace(old, f"for (int e = 0; e < {width}; ++e) acc = fmaf(r[{width} * j + e], r[{width} * j + e], acc);")


@pytest.mark.parametrize("name,old,new,probe", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new, probe):
    src = oracle.source()
    assert src.count(old) == 1, f"mutation site not found once: {name}"
    mutated = src.replace(old, new)
    if "leaves of 4" in name:
        mutated = _leaf_edit(mutated, 4)
    elif "leaves of 16" in name:
        mutated = _leaf_edit(mutated, 16)
    so = oracle.compile_variant(mutated, os.path.join(str(tmp_path), "liboracle_mutant.so"))
    with oracle.library(so):
        with pytest.raises(AssertionError):
            probes.ALL[probe]()
    # the wrappers are back on the real oracle, which passes
    probes.ALL[probe]()
