"""GPU parity of the tree-ordered causal attention (tbik_attention) against the
CPU oracle: bit-exact, since both sides take the same fp32 operation sequence;
plus invariance to the batch composition and to splitting the heads, and the
embedding gather."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, dev_i32, host_bits16  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402


def qkv(seed, shape, std=1.0):
    return [synth.normal_bf16(seed + i, shape, std=std) for i in range(3)]


@pytest.mark.parametrize("B,S,NH,D", [(1, 1, 1, 128), (2, 64, 2, 128), (2, 65, 3, 128), (2, 200, 3, 128),
                                      (1, 300, 2, 64), (3, 129, 1, 64)])
def test_attention_bitwise_vs_oracle(B, S, NH, D):
    q, k, v = qkv(400 + S, (B, S, NH, D))
    got = tbik.attention(dev_bf16(q), dev_bf16(k), dev_bf16(v))
    assert np.array_equal(host_bits16(got), oracle.attention(q, k, v, chunk=64))
    assert tbik.get_error() == tbik.TBIK_OK


def test_attention_large_scores_and_cancelling_values():
    # wide score range (std 4 queries and keys) exercises the chunk max and
    # the exp(m - M) rescaling in the tree combine
    q, k, v = qkv(430, (2, 333, 2, 128), std=4.0)
    got = tbik.attention(dev_bf16(q), dev_bf16(k), dev_bf16(v))
    assert np.array_equal(host_bits16(got), oracle.attention(q, k, v, chunk=64))


def test_attention_batch_and_head_split_invariance():
    B, S, NH, D = 3, 257, 4, 128
    q, k, v = (dev_bf16(a) for a in qkv(440, (B, S, NH, D)))
    full = host_bits16(tbik.attention(q, k, v))
    # one sequence alone
    one = host_bits16(tbik.attention(q[1:2].contiguous(), k[1:2].contiguous(), v[1:2].contiguous()))
    assert np.array_equal(one[0], full[1])
    # heads split as over T = 2 and T = 4 devices
    for T in (2, 4):
        w = NH // T
        for t in range(T):
            part = host_bits16(tbik.attention(q[:, :, t * w:(t + 1) * w].contiguous(),
                                              k[:, :, t * w:(t + 1) * w].contiguous(),
                                              v[:, :, t * w:(t + 1) * w].contiguous()))
            assert np.array_equal(part, full[:, :, t * w:(t + 1) * w]), (T, t)
    # a shuffled batch gives each sequence the same bits
    perm = [2, 0, 1]
    shuf = host_bits16(tbik.attention(q[perm].contiguous(), k[perm].contiguous(), v[perm].contiguous()))
    assert np.array_equal(shuf, full[perm])


def test_attention_full_config_sampled():
    # the decoder configuration: batch 8 x seq 2048, 16 heads of 128
    B, S, NH, D = 8, 2048, 16, 128
    q, k, v = qkv(450, (B, S, NH, D))
    got = host_bits16(tbik.attention(dev_bf16(q), dev_bf16(k), dev_bf16(v)))
    b, h = 5, 11
    for i in (0, 63, 64, 1000, 2047):
        ref = oracle.attention(q[b:b + 1, :i + 1, h:h + 1].copy(), k[b:b + 1, :i + 1, h:h + 1].copy(),
                               v[b:b + 1, :i + 1, h:h + 1].copy(), chunk=64)
        assert np.array_equal(got[b, i, h], ref[0, i, 0]), i


def test_attention_argument_errors():
    lib = tbik.load_library()
    x = torch.zeros((1, 8, 1, 128), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    p = x.data_ptr()
    assert lib.tbik_attention(p, p, p, p, 1, 8, 1, 96, 64, s) == tbik.TBIK_ERR_SHAPE
    assert lib.tbik_attention(p, p, p, p, 1, 8, 1, 128, 32, s) == tbik.TBIK_ERR_SHAPE
    assert lib.tbik_attention(p + 2, p, p, p, 1, 8, 1, 128, 64, s) == tbik.TBIK_ERR_ALIGN
    assert lib.tbik_attention(None, p, p, p, 1, 8, 1, 128, 64, s) == tbik.TBIK_ERR_ARG
    assert lib.tbik_attention(p, p, p, p, 0, 8, 1, 128, 64, s) == tbik.TBIK_OK


def test_embedding_rows_and_bad_ids():
    V, d = 1000, 2048
    table = synth.normal_bf16(460, (V, d), std=0.02)
    ids = np.array([0, 999, 5, 5, 123], dtype=np.int32)
    got = host_bits16(tbik.embedding(dev_i32(ids), dev_bf16(table)))
    assert np.array_equal(got, table[ids])
    assert tbik.get_error() == tbik.TBIK_OK
    bad = host_bits16(tbik.embedding(dev_i32(np.array([1, V, -1], dtype=np.int32)), dev_bf16(table)))
    assert tbik.get_error() == tbik.TBIK_ERR_TARGET
    assert np.array_equal(bad[0], table[1]) and not bad[1].any() and not bad[2].any()
