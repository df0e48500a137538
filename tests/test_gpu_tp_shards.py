"""The cross-GPU shard level of the tree through the C ABI, on one GPU.

The T ranks of a tensor-parallel group are emulated in one process: each
shard's kernels run on its own slice (a K shard of the GEMM, a vocabulary shard
of the lm_head), the shard results are stacked in rank order (what the
all-gather delivers on every rank), and tbik_tree_combine /
tbik_logprob_combine apply the shard level.  The result must be bitwise the
one-GPU call's, in tensor-core and exact mode; exact mode also equals the
oracle.  The tp module's functions run once in a one-rank NCCL group.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, dev_i32, host_bits16, host_f32, u32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402


def _k_shards(a, b, T):
    K = a.shape[1]
    ks = K // T
    return [(a[:, t * ks:(t + 1) * ks].contiguous(), b[t * ks:(t + 1) * ks].contiguous()) for t in range(T)]


@pytest.mark.parametrize("tc", [True, False])
def test_row_parallel_gemm_shards_reproduce_one_gpu_bits(tc):
    M, N, K, leaf = 300, 264, 4096, 256  # 16 leaves; shards of 8, 4, 2 leaves
    a_h = synth.normal_bf16(700, (M, K))
    b_h = synth.normal_bf16(701, (K, N), std=0.02)
    r_h = synth.normal_bf16(702, (M, N))
    a, b, r = dev_bf16(a_h), dev_bf16(b_h), dev_bf16(r_h)
    one = host_f32(tbik.gemm(a, b, T=1, leaf=leaf, tc=tc))
    one_bf = host_bits16(tbik.gemm(a, b, T=1, leaf=leaf, tc=tc, out_bf16=True))
    one_res = host_bits16(tbik.gemm(a, b, T=1, leaf=leaf, tc=tc, residual=r))
    if not tc:
        assert np.array_equal(u32(one), u32(oracle.gemm_tree(a_h, b_h, b_nk=False, T=1, leaf=leaf)))
    for T in (2, 4, 8):
        parts = torch.stack([tbik.gemm(at, bt, T=1, leaf=leaf, tc=tc) for at, bt in _k_shards(a, b, T)])
        assert np.array_equal(u32(host_f32(tbik.tree_combine(parts))), u32(one)), T
        assert np.array_equal(host_bits16(tbik.tree_combine(parts, out_bf16=True)), one_bf), T
        assert np.array_equal(host_bits16(tbik.tree_combine(parts, residual=r)), one_res), T
        # the baseline: one chain per shard, shard results summed left to right
        nparts = torch.stack([tbik.gemm(at, bt, T=1, leaf=leaf, tc=tc, noninv=True) for at, bt in _k_shards(a, b, T)])
        base = host_f32(tbik.gemm(a, b, T=T, leaf=leaf, tc=tc, noninv=True))
        assert np.array_equal(u32(host_f32(tbik.tree_combine(nparts, noninv=True))), u32(base)), T
    assert tbik.get_error() == tbik.TBIK_OK


def _vocab_parallel(h, w, t, V, T, *, tc, leaf):
    parts = []
    for s in range(T):
        v0, vs, lvs = tbik.vocab_shard(V, T, s)
        parts.append(tbik.logprob_partial(h, w[v0:v0 + vs].contiguous(), t, v0=v0, Lvs=lvs, leaf=leaf, tc=tc))
    return tbik.logprob_combine(torch.stack(parts), t, V)


@pytest.mark.parametrize("tc", [True, False])
def test_vocab_parallel_logprob_reproduces_one_gpu_bits(tc):
    # V = 18900 pads to 18944 = 37 * 512 columns: at T = 8 the shards are 2368
    # columns wide, so odd shards start half way into a 128-column GEMM tile
    V, H, M, leaf = 18900, 1024, 70, 256
    h_h = synth.normal_bf16(710, (M, H))
    w_h = synth.normal_bf16(711, (V, H), std=0.05)
    tg = synth.uniform_int32(712, M, 0, V)
    # targets on both sides of every shard boundary (T = 2, 4, 8), in the ragged
    # last leaf [18880, 18900) and on the first and last columns
    tg[:16] = [2367, 2368, 4735, 4736, 7103, 7104, 9471, 9472, 11839, 11840, 14207, 14208, 18880, 18899, 0, 63]
    h, w, t = dev_bf16(h_h), dev_bf16(w_h), dev_i32(tg)
    one = host_f32(tbik.logprob(h, w, t, T=1, leaf=leaf, tc=tc))
    if not tc:
        assert np.array_equal(u32(one), u32(oracle.logprob(h_h, w_h, tg, T=1, leaf=leaf)))
    for T in (1, 2, 4, 8):
        got = host_f32(_vocab_parallel(h, w, t, V, T, tc=tc, leaf=leaf))
        assert np.array_equal(u32(got), u32(one)), T
    assert tbik.get_error() == tbik.TBIK_OK


def test_vocab_parallel_padding_only_shard_and_bad_target():
    """V = 100 with T = 8: shards 2..7 hold padding only (no W rows).  A target
    outside [0, V) gives NaN and TBIK_ERR_TARGET, as in tbik_logprob."""
    V, H, M = 100, 256, 5
    h_h = synth.normal_bf16(720, (M, H))
    w_h = synth.normal_bf16(721, (V, H), std=0.1)
    tg = np.array([0, 99, 64, 63, 5], dtype=np.int32)
    h, w, t = dev_bf16(h_h), dev_bf16(w_h), dev_i32(tg)
    ref = oracle.logprob(h_h, w_h, tg, T=1, leaf=256)
    got = host_f32(_vocab_parallel(h, w, t, V, 8, tc=False, leaf=256))
    assert np.array_equal(u32(got), u32(ref))
    assert tbik.get_error() == tbik.TBIK_OK
    bad = dev_i32(np.array([0, 100, 64, -1, 5], dtype=np.int32))
    out = host_f32(_vocab_parallel(h, w, bad, V, 8, tc=True, leaf=256))
    assert np.isnan(out[1]) and np.isnan(out[3]) and np.all(np.isfinite(out[[0, 2, 4]]))
    assert tbik.get_error() == tbik.TBIK_ERR_TARGET


def test_shard_level_argument_errors():
    lib = tbik.load_library()
    s = torch.cuda.current_stream().cuda_stream
    p = torch.zeros((4, 64), dtype=torch.float32, device="cuda")
    o = torch.zeros(64, dtype=torch.float32, device="cuda")
    assert lib.tbik_tree_combine(p.data_ptr(), o.data_ptr(), 64, 3, 0, None, s) == tbik.TBIK_ERR_SHAPE
    assert lib.tbik_tree_combine(p.data_ptr(), o.data_ptr(), 64, 4, 0x1, None, s) == tbik.TBIK_ERR_ARG
    assert lib.tbik_tree_combine(p.data_ptr(), o.data_ptr(), 64, 4, 0, p.data_ptr(), s) == tbik.TBIK_ERR_ARG
    assert lib.tbik_tree_combine(p.data_ptr() + 4, o.data_ptr(), 60, 4, 0, None, s) == tbik.TBIK_ERR_ALIGN
    assert lib.tbik_logprob_partial_workspace(4, 100, 1, 256, 256, tbik.TC) == (1 << 64) - 1  # 1 leaf < 100 cols
    assert lib.tbik_logprob_partial_workspace(4, 100, 2, 256, 256, tbik.TC | tbik.NONINV) == (1 << 64) - 1
    t = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert lib.tbik_logprob_combine(p.data_ptr(), t.data_ptr(), o.data_ptr(), 4, 10, 5, s) == tbik.TBIK_ERR_SHAPE
    assert tbik.get_error() == tbik.TBIK_OK


def test_tp_module_in_a_one_rank_group():
    import os
    import socket

    import torch.distributed as dist

    from invariant_tree_ordered_b200 import tp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        a = dev_bf16(synth.normal_bf16(730, (64, 512)))
        b = dev_bf16(synth.normal_bf16(731, (512, 128), std=0.05))
        c = tp.gemm_row_parallel(a, b, leaf=128)
        assert np.array_equal(u32(host_f32(c)), u32(host_f32(tbik.gemm(a, b, T=1, leaf=128))))
        h = dev_bf16(synth.normal_bf16(732, (16, 256)))
        w = dev_bf16(synth.normal_bf16(733, (3000, 256), std=0.1))
        t = dev_i32(synth.uniform_int32(734, 16, 0, 3000))
        lp = tp.logprob_vocab_parallel(h, w, t, 3000)
        assert np.array_equal(u32(host_f32(lp)), u32(host_f32(tbik.logprob(h, w, t, T=1))))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
