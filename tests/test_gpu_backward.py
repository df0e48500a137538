"""Backward GEMMs with the same tree (the pages' FSDP side): the input gradient
dX = dY W^T is the tree GEMM with W read as [N, K]; the weight gradient
dW = X^T dY reduces over tokens, so with token leaves and T data-parallel
shards of the tokens combined by the tree it is bitwise the same for every
shard count.  Exact mode is bit-exact to the oracle; tensor-core mode is
invariant over T and within 2e-5 relative Frobenius error of binary64."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, host_bits16, host_f32, rel_frob, u32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402


def test_transpose_exact():
    # (256, 128), (200, 136), (64, 8), (8, 640): the 16-byte vector path (both
    # sizes multiples of 8), full and ragged 64 x 64 tiles; the rest element-wise
    for rows, cols in ((1, 1), (33, 70), (256, 128), (1000, 37), (200, 136), (64, 8), (8, 640)):
        x = synth.normal_bf16(800 + rows, (rows, cols))
        got = host_bits16(tbik.transpose(dev_bf16(x)))
        assert np.array_equal(got, np.ascontiguousarray(x.T)), (rows, cols)


def test_input_gradient_is_the_tree_gemm_with_w_as_n_by_k():
    M, K, N = 200, 384, 512  # forward Y[M,N] = X[M,K] W[K,N]; dX[M,K] = dY[M,N] W^T
    dy = synth.normal_bf16(810, (M, N))
    w = synth.normal_bf16(811, (K, N), std=0.05)
    ref = oracle.gemm_tree(dy, w, b_nk=True, T=1, leaf=64)  # W [K, N] is the [N', K'] operand
    for T in (1, 2, 8):
        got = host_f32(tbik.gemm(dev_bf16(dy), dev_bf16(w), T=T, leaf=64, tc=False, b_nk=True))
        assert np.array_equal(u32(got), u32(ref)), T
    tcs = [host_f32(tbik.gemm(dev_bf16(dy), dev_bf16(w), T=T, leaf=64, tc=True, b_nk=True)) for T in (1, 2, 8)]
    for o in tcs[1:]:
        assert np.array_equal(u32(o), u32(tcs[0]))
    assert rel_frob(tcs[0], oracle.gemm_f64(dy, w, b_nk=True)) <= 2e-5


def test_weight_gradient_over_token_shards():
    M, K, N = 2048, 256, 384  # tokens, in, out; token leaves of 256, T data-parallel shards
    x = synth.normal_bf16(820, (M, K))
    dy = synth.normal_bf16(821, (M, N), std=0.1)
    xt_h = np.ascontiguousarray(x.T)
    ref = oracle.gemm_tree(xt_h, dy, b_nk=False, T=1, leaf=256)
    xt = tbik.transpose(dev_bf16(x))
    assert np.array_equal(host_bits16(xt), xt_h)
    dyd = dev_bf16(dy)
    for T in (1, 2, 4, 8):
        got = host_f32(tbik.gemm(xt, dyd, T=T, leaf=256, tc=False))
        assert np.array_equal(u32(got), u32(ref)), T
    tcs = [host_f32(tbik.gemm(xt, dyd, T=T, leaf=256, tc=True)) for T in (1, 2, 4, 8)]
    for o in tcs[1:]:
        assert np.array_equal(u32(o), u32(tcs[0]))
    assert rel_frob(tcs[0], oracle.gemm_f64(xt_h, dy, b_nk=False)) <= 2e-5
    # the non-invariant baseline (per-shard chain, shards summed in order) moves with T
    non = [host_f32(tbik.gemm(xt, dyd, T=T, leaf=256, tc=True, noninv=True)) for T in (1, 8)]
    assert not np.array_equal(u32(non[0]), u32(non[1]))
    assert tbik.get_error() == tbik.TBIK_OK
