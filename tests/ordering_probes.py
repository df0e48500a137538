"""Ordering probes of the oracle: inputs whose expected outputs are derived by
hand in exact binary32 arithmetic (tests/golden/ordering_probes.json holds the
derivations) and on which a different reduction order, leaf size or operand
placement moves the output far outside rounding.

Each probe raises AssertionError when the oracle disagrees.  They are shared by
the pin tests (the real oracle must pass) and the mutation tests (a copy of
oracle.c with one planted mistake must fail the matching probe).
"""
import json
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ordering_probes.json")


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def bf16_exact(x) -> np.ndarray:
    """bf16 bit patterns of values that bf16 represents exactly (no rounding:
    asserts the low 16 bits of the binary32 pattern are zero)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    assert not np.any(u & 0xFFFF), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


# ------------------------------------------------- baseline shard sum (GEMM)

def check_baseline_shard_sum():
    g = golden()["baseline_shard_sum"]
    for key, T in (("T4", 4), ("T8", 8)):
        a = bf16_exact(np.array([g[key]["A"]], dtype=np.float32))
        b = bf16_exact(np.ones((T, 1), dtype=np.float32))
        c, q = oracle.gemm_noninv(a, b, b_nk=False, T=T, shards=True)
        assert np.array_equal(q[:, 0, 0], np.array(g[key]["A"], dtype=np.float32)), key
        assert c[0, 0] == np.float32(g[key]["expected"]), (key, float(c[0, 0]))


# ---------------------------------------- logprob baseline (logit shard sum)

def check_logprob_baseline_logit_sum():
    g = golden()["logprob_baseline_logit_sum"]
    h = bf16_exact(np.array([[2.0 ** 27, 1.0, -(2.0 ** 27), 1.0]], dtype=np.float32))
    w = bf16_exact(np.array([[1, 1, 1, 1], [0, 0, 0, 0]], dtype=np.float32))
    t = np.array([0], dtype=np.int32)
    out = oracle.logprob(h, w, t, T=4, leaf=4, noninv=True)
    expect = 1.0 - math.log1p(math.e)
    assert abs(expect - g["expected_value"]) < 1e-15
    assert abs(float(out[0]) - expect) <= g["tolerance"], float(out[0])


# --------------------------------------------------------------- RMSNorm

RMS_H = 256


def rmsnorm_probe_inputs():
    r = np.ones(RMS_H, dtype=np.float32)
    r[0::16] = 2.0 ** 12  # first element of every even leaf of 8
    gamma = (1.0 + (np.arange(RMS_H) % 128) / 128.0).astype(np.float32)
    return r, gamma


def check_rmsnorm_cancellation():
    g = golden()["rmsnorm_cancellation"]
    r, gamma = rmsnorm_probe_inputs()
    rb, gb = bf16_exact(r[None, :]), bf16_exact(gamma)
    zero = bf16_exact(np.zeros((1, RMS_H), dtype=np.float32))
    expect = bf16_exact(2.0 * r * gamma)
    for T in (1, 2, 4, 8):
        # the residual stream in x, in res, or no residual input at all
        for x, res in ((rb, zero), (zero, rb), (rb, None)):
            y, ro = oracle.rmsnorm_residual(x, res, gb, eps=g["eps"], T=T)
            assert np.array_equal(y[0], expect), (T, res is None)
            assert np.array_equal(ro[0], rb[0])


# ---------------------------------------------------------- vocab leaf

def _vocab_probe(z, target):
    H = 16
    h = np.zeros((1, H), dtype=np.float32)
    h[0, 0] = 1.0
    w = np.zeros((len(z), H), dtype=np.float32)
    w[:, 0] = z
    return bf16_exact(h), bf16_exact(w), np.array([target], dtype=np.int32)


def check_vocab_leaf_ascending_sum():
    g = golden()["vocab_leaf_ascending_sum"]
    z = np.full(64, -18.0, dtype=np.float32)
    z[0] = 0.0
    h, w, t = _vocab_probe(z, 0)
    for T in (1, 2, 4, 8):
        out = oracle.logprob(h, w, t, T=T, leaf=16)
        assert out[0] == np.float32(g["max_first"]["expected"]), (T, float(out[0]))
    z = np.full(64, -18.0, dtype=np.float32)
    z[63] = 0.0
    h, w, t = _vocab_probe(z, 63)
    lo, hi = g["max_last"]["expected_range"]
    out = oracle.logprob(h, w, t, T=1, leaf=16)
    assert lo <= float(out[0]) <= hi, float(out[0])


ALL = {
    "baseline_shard_sum": check_baseline_shard_sum,
    "logprob_baseline_logit_sum": check_logprob_baseline_logit_sum,
    "rmsnorm_cancellation": check_rmsnorm_cancellation,
    "vocab_leaf_ascending_sum": check_vocab_leaf_ascending_sum,
}
