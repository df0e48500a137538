"""The oracle's ordering probes (tests/golden/ordering_probes.json) run through
the CUDA kernels in exact-order mode: the baseline's left-to-right shard sum,
the RMSNorm leaf size, mean and eps placement, and the ascending vocabulary
leaf sum give the hand-derived outputs bit for bit, equal to the oracle's."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests import ordering_probes as probes  # noqa: E402
from tests.gpu_util import dev_bf16, dev_i32, host_bits16, host_f32, u32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402


def test_baseline_shard_sum_left_to_right_on_gpu():
    g = probes.golden()["baseline_shard_sum"]
    for key, T in (("T4", 4), ("T8", 8)):
        a = probes.bf16_exact(np.array([g[key]["A"]], dtype=np.float32))
        b = probes.bf16_exact(np.ones((T, 1), dtype=np.float32))
        c = host_f32(tbik.gemm(dev_bf16(a), dev_bf16(b), T=T, leaf=1, tc=False, noninv=True))
        assert tbik.get_error() == tbik.TBIK_OK
        assert c[0, 0] == np.float32(g[key]["expected"]), key


def test_rmsnorm_cancellation_probe_on_gpu():
    g = probes.golden()["rmsnorm_cancellation"]
    r, gamma = probes.rmsnorm_probe_inputs()
    rb, gb = probes.bf16_exact(r[None, :]), probes.bf16_exact(gamma)
    zero = probes.bf16_exact(np.zeros_like(r)[None, :])
    expect = probes.bf16_exact(2.0 * r * gamma)
    for T in (1, 2, 4, 8):
        for x, res in ((rb, zero), (zero, rb), (rb, None)):
            y, _ = tbik.rmsnorm_residual(dev_bf16(x), None if res is None else dev_bf16(res), dev_bf16(gb),
                                         eps=g["eps"], T=T)
            assert tbik.get_error() == tbik.TBIK_OK
            assert np.array_equal(host_bits16(y)[0], expect), (T, res is None)


def test_vocab_leaf_ascending_sum_on_gpu():
    H = 16
    for first in (True, False):
        z = np.full(64, -18.0, dtype=np.float32)
        tgt = 0 if first else 63
        z[tgt] = 0.0
        h = np.zeros((1, H), dtype=np.float32)
        h[0, 0] = 1.0
        w = np.zeros((64, H), dtype=np.float32)
        w[:, 0] = z
        hb, wb = probes.bf16_exact(h), probes.bf16_exact(w)
        t = np.array([tgt], dtype=np.int32)
        ref = oracle.logprob(hb, wb, t, T=1, leaf=H)
        for T in (1, 2, 4, 8):
            got = host_f32(tbik.logprob(dev_bf16(hb), dev_bf16(wb), dev_i32(t), T=T, leaf=H, tc=False))
            assert tbik.get_error() == tbik.TBIK_OK
            assert np.array_equal(u32(got), u32(ref)), (first, T)
        if first:
            assert float(ref[0]) == 0.0


def test_logprob_baseline_logit_sum_on_gpu():
    """H = 16 split into T = 8 chains of 2: the shard partials are
    (2^27, 1, -2^27, 1, 0, 0, 0, 0), summed left to right to the logit 1."""
    h = np.zeros((1, 16), dtype=np.float32)
    h[0, [0, 2, 4, 6]] = [2.0 ** 27, 1.0, -(2.0 ** 27), 1.0]
    w = np.zeros((2, 16), dtype=np.float32)
    w[0] = 1.0
    hb, wb = probes.bf16_exact(h), probes.bf16_exact(w)
    t = np.array([0], dtype=np.int32)
    ref = oracle.logprob(hb, wb, t, T=8, leaf=16, noninv=True)
    got = host_f32(tbik.logprob(dev_bf16(hb), dev_bf16(wb), dev_i32(t), T=8, leaf=16, tc=False, noninv=True))
    assert tbik.get_error() == tbik.TBIK_OK
    assert np.array_equal(u32(got), u32(ref))
    assert abs(float(ref[0]) - probes.golden()["logprob_baseline_logit_sum"]["expected_value"]) <= 1e-6
