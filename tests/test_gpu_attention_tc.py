"""Tensor-core mode of the tree-ordered causal attention (tbik_attention_tc).

Not bit-exact to the oracle (the dot products run on the tensor cores, the
keys are reduced in 128-key leaves and the softmax weights are rounded to bf16
before P V), so it is checked against the binary64 definition with a bound
derived from that arithmetic:
  the weights of a row are p_j rounded to bf16 (relative error <= 2^-9) and
  the sum s uses the same rounded weights, so the output is an exact weighted
  average of the v_j with each normalised weight moved by at most about
  2 * 2^-9 of itself: |o/s - exact| <= 2^-8 * max_j |v_j - exact| <= 2^-7 * max|v|;
  the output rounding to bf16 adds 2^-9 |out| (2^-8 here, with margin); the
  fp32 score and combine arithmetic is orders of magnitude below these.
It must also be bitwise independent of the batch composition and of how the
heads are split, and agree with the exact mode to the same bound.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, host_bits16  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402


def qkv(seed, shape, std=1.0):
    return [synth.normal_bf16(seed + i, shape, std=std) for i in range(3)]


def f32(bits16):
    return (np.asarray(bits16).astype(np.uint32) << 16).view(np.float32)


def within_bound(got, ref, v):
    vmax = float(np.abs(f32(v)).max())
    return np.abs(got - ref) <= 2.0 ** -7 * vmax + 2.0 ** -8 * np.abs(ref)


@pytest.mark.parametrize("B,S,NH", [(1, 128, 1), (2, 256, 3), (1, 1024, 2), (1, 2048, 1), (1, 4096, 1)])
def test_tc_attention_vs_binary64(B, S, NH):
    # 1024, 2048 and 4096 positions: 8, 16 and 32 leaves; from 2048 on, pending
    # summaries of >= 5 leaves (8, then 16 and 8) use the L2 stack
    q, k, v = qkv(500 + S, (B, S, NH, 128))
    got = f32(host_bits16(tbik.attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), tc=True)))
    assert tbik.get_error() == tbik.TBIK_OK
    ref = oracle.attention_f64(q, k, v)
    assert np.all(np.isfinite(got))
    assert np.all(within_bound(got, ref, v))
    assert float(np.mean(np.abs(got - ref))) <= 1e-3
    exact = f32(oracle.attention(q, k, v, chunk=64))
    assert np.all(within_bound(got, exact, v))


def test_tc_attention_more_than_32_leaves():
    """4224 positions: the last query tile has 33 leaves, so the epilogue's lanes
    walk the leaf tree for a second block of 32 leaves; checked against binary64.
    The same positions inside an 8192-position sequence (64 leaves, deeper L2
    stack) give the same bits: a row's result depends only on its own keys."""
    B, S, NH = 1, 4224, 2
    q, k, v = qkv(4224, (B, S, NH, 128))
    got_bits = host_bits16(tbik.attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), tc=True))
    assert tbik.get_error() == tbik.TBIK_OK
    got = f32(got_bits)
    ref = oracle.attention_f64(q, k, v)
    assert np.all(np.isfinite(got))
    assert np.all(within_bound(got, ref, v))
    assert float(np.mean(np.abs(got - ref))) <= 1e-3
    L = 8192
    ext = qkv(8192, (B, L - S, NH, 128))
    q2, k2, v2 = (np.ascontiguousarray(np.concatenate([x, e], axis=1)) for x, e in zip((q, k, v), ext))
    long_bits = host_bits16(tbik.attention(dev_bf16(q2), dev_bf16(k2), dev_bf16(v2), tc=True))
    assert tbik.get_error() == tbik.TBIK_OK
    assert np.array_equal(long_bits[:, :S], got_bits)


def test_tc_attention_large_scores():
    # std-4 queries and keys: a wide score range, so the chunk maxima and the
    # exp(m - M) factors of the tree combine matter
    q, k, v = qkv(530, (2, 384, 2, 128), std=4.0)
    got = f32(host_bits16(tbik.attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), tc=True)))
    ref = oracle.attention_f64(q, k, v)
    assert np.all(np.isfinite(got)) and np.all(within_bound(got, ref, v))


def test_tc_attention_batch_and_head_split_invariance():
    B, S, NH = 3, 512, 4
    q, k, v = (dev_bf16(a) for a in qkv(540, (B, S, NH, 128)))
    full = host_bits16(tbik.attention(q, k, v, tc=True))
    one = host_bits16(tbik.attention(q[1:2].contiguous(), k[1:2].contiguous(), v[1:2].contiguous(), tc=True))
    assert np.array_equal(one[0], full[1])
    for T in (2, 4):
        w = NH // T
        for t in range(T):
            sl = slice(t * w, (t + 1) * w)
            part = host_bits16(tbik.attention(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                              v[:, :, sl].contiguous(), tc=True))
            assert np.array_equal(part, full[:, :, sl]), (T, t)
    perm = [2, 0, 1]
    shuf = host_bits16(tbik.attention(q[perm].contiguous(), k[perm].contiguous(), v[perm].contiguous(), tc=True))
    assert np.array_equal(shuf, full[perm])
    assert tbik.get_error() == tbik.TBIK_OK


def test_tc_attention_repeat_runs_and_batch_subset_at_2048():
    """Several 2048-position tiles per CTA (persistent grid) with leaf trees
    deep enough for the L2 stack: repeated calls give the same bits, and so
    does one sequence alone."""
    B, S, NH = 4, 2048, 16
    g = torch.Generator(device="cuda").manual_seed(5)
    q, k, v = [torch.randn(B, S, NH, 128, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3)]
    runs = [host_bits16(tbik.attention(q, k, v, tc=True)) for _ in range(3)]
    for r in runs[1:]:
        assert np.array_equal(r, runs[0])
    one = host_bits16(tbik.attention(q[2:3].contiguous(), k[2:3].contiguous(), v[2:3].contiguous(), tc=True))
    assert np.array_equal(one[0], runs[0][2])
    assert tbik.get_error() == tbik.TBIK_OK


def test_tc_attention_argument_errors():
    lib = tbik.load_library()
    s = torch.cuda.current_stream().cuda_stream
    x = torch.zeros((1, 256, 2, 128), dtype=torch.bfloat16, device="cuda")
    p = x.data_ptr()
    assert lib.tbik_attention_tc(p, p, p, p, 1, 200, 2, 128, 128, None, 0, s) == tbik.TBIK_ERR_SHAPE  # seq % 128
    assert lib.tbik_attention_tc(p, p, p, p, 1, 256, 2, 64, 128, None, 0, s) == tbik.TBIK_ERR_SHAPE   # head_dim
    assert lib.tbik_attention_tc(p, p, p, p, 1, 256, 2, 128, 64, None, 0, s) == tbik.TBIK_ERR_SHAPE   # leaf
    assert lib.tbik_attention_tc(p, p, p, p, 1, 256, 2, 128, 32, None, 0, s) == tbik.TBIK_ERR_SHAPE   # leaf
    assert lib.tbik_attention_tc(p + 2, p, p, p, 1, 256, 2, 128, 128, None, 0, s) == tbik.TBIK_ERR_ALIGN
    assert lib.tbik_attention_tc_workspace(1, 200, 2, 128, 128) == (1 << 64) - 1
    assert lib.tbik_attention_tc_workspace(1, 256, 2, 128, 128) == 0  # 2 leaves: nothing pending in L2
    need = lib.tbik_attention_tc_workspace(1, 2048, 2, 128, 128)
    assert need > 0  # 16 leaves: the tree has a pending value of 8 leaves
    big = torch.zeros((1, 2048, 2, 128), dtype=torch.bfloat16, device="cuda")
    b = big.data_ptr()
    assert lib.tbik_attention_tc(b, b, b, b, 1, 2048, 2, 128, 128, None, 0, s) == tbik.TBIK_ERR_WORKSPACE
    assert tbik.get_error() == tbik.TBIK_OK


@pytest.mark.parametrize("tc", [True, False])
def test_prefix_invariance_longer_sequence(tc):
    """Row i attends to keys <= i through its fixed leaf tree, so its bits do
    not depend on how long the sequence is: the first 1024 positions of a
    2048-position sequence equal the same 1024 positions computed alone (the
    consistency a serving loop needs between a prefill and a longer one)."""
    B, S, NH = 2, 2048, 4
    g = torch.Generator(device="cuda").manual_seed(11)
    q, k, v = [torch.randn(B, S, NH, 128, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3)]
    full = host_bits16(tbik.attention(q, k, v, tc=tc))
    for L in (1024, 384, 128):
        part = host_bits16(tbik.attention(q[:, :L].contiguous(), k[:, :L].contiguous(), v[:, :L].contiguous(), tc=tc))
        assert np.array_equal(part, full[:, :L]), L
    assert tbik.get_error() == tbik.TBIK_OK
