"""GPU parity of the fused lm_head -> log-softmax -> target logprob.

Exact-order mode: bit-exact to the oracle.  Tensor-core mode: bitwise
identical across T, batch size and batch order, and within 1e-4 of the oracle.
The non-invariant baseline diverges across T.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, dev_i32, host_f32, oracle_rows, sample_rows, u32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402

TS = (1, 2, 4, 8)


def lp(h, w, t, **kw):
    out = host_f32(tbik.logprob(h, w, t, **kw))
    assert tbik.get_error() == tbik.TBIK_OK
    return out


@pytest.mark.parametrize("M,V,H,leaf", [(5, 1000, 256, 128), (130, 2176, 512, 256), (1, 127, 256, 256),
                                        (33, 8192 + 72, 768, 256)])
def test_small_exact_bitwise_tc_close_and_invariant(M, V, H, leaf):
    h = synth.normal_bf16(300 + M, (M, H))
    w = synth.normal_bf16(301 + V, (V, H), std=0.05)
    t = synth.uniform_int32(302, M, 0, V)
    ref = oracle.logprob(h, w, t, T=1, leaf=leaf)
    hd, wd, td = dev_bf16(h), dev_bf16(w), dev_i32(t)
    tc_outs = []
    for T in TS:
        ex = lp(hd, wd, td, T=T, leaf=leaf, tc=False)
        assert np.array_equal(u32(ex), u32(ref)), ("exact", T)
        tc_outs.append(lp(hd, wd, td, T=T, leaf=leaf, tc=True))
    for o in tc_outs[1:]:
        assert np.array_equal(u32(o), u32(tc_outs[0]))
    assert np.max(np.abs(tc_outs[0] - ref)) <= 1e-4
    ref64 = oracle.logprob_f64(h, w, t)
    assert np.max(np.abs(tc_outs[0] - ref64)) <= 1e-4


def test_noninv_exact_matches_oracle_and_tc_diverges():
    M, V, H = 64, 8192, 512
    h = synth.normal_bf16(310, (M, H))
    w = synth.normal_bf16(311, (V, H), std=0.2)
    t = synth.uniform_int32(312, M, 0, V)
    hd, wd, td = dev_bf16(h), dev_bf16(w), dev_i32(t)
    for T in TS:
        ex = lp(hd, wd, td, T=T, leaf=256, tc=False, noninv=True)
        assert np.array_equal(u32(ex), u32(oracle.logprob(h, w, t, T=T, leaf=256, noninv=True))), T
    non = [lp(hd, wd, td, T=T, leaf=256, tc=True, noninv=True) for T in TS]
    assert any(not np.array_equal(u32(non[0]), u32(o)) for o in non[1:])


def test_target_out_of_range_is_nan_and_flagged():
    M, V, H = 4, 1000, 256
    h = dev_bf16(synth.normal_bf16(320, (M, H)))
    w = dev_bf16(synth.normal_bf16(321, (V, H), std=0.05))
    t = dev_i32(np.array([3, V, -1, 999], dtype=np.int32))
    out = host_f32(tbik.logprob(h, w, t, leaf=256))
    assert tbik.get_error() == tbik.TBIK_ERR_TARGET
    assert np.isnan(out[1]) and np.isnan(out[2]) and np.isfinite(out[0]) and np.isfinite(out[3])
    assert tbik.get_error() == tbik.TBIK_OK


@pytest.fixture(scope="module")
def lm_head():
    hidden, w, targets = synth.logprob_inputs(4096)
    return hidden, w, targets, dev_bf16(hidden), dev_bf16(w), dev_i32(targets)


def test_lm_head_full_size_invariance_over_T_M_and_order(lm_head):
    hidden, w, targets, hd, wd, td = lm_head
    base = {T: lp(hd, wd, td, T=T, tc=True) for T in TS}
    for T in TS[1:]:
        assert np.array_equal(u32(base[T]), u32(base[1])), T
    for M in (1, 256):
        part = lp(hd[:M].contiguous(), wd, td[:M].contiguous(), T=8 if M == 1 else 2, tc=True)
        assert np.array_equal(u32(part), u32(base[1][:M])), M
    perm = synth.permutation(33, 4096)
    pt = torch.from_numpy(perm.astype(np.int64)).cuda()
    shuf = lp(hd[pt].contiguous(), wd, td[pt].contiguous(), T=4, tc=True)
    assert np.array_equal(u32(shuf), u32(base[1][perm]))


def test_lm_head_full_size_vs_oracle_sampled_rows(lm_head):
    """64 seeded rows of the 4096-token launch, compared with the oracle row by
    row.  Their targets are set to the cases where an order or index mistake
    would show: the first and last vocabulary columns, both sides of vocab-leaf
    boundaries (64 columns), of the T = 8 shard boundaries (19008 columns) and
    of 128-column GEMM tiles, and every column of the last vocabulary leaf's
    edges [151872, 151936)."""
    hidden, w, targets, hd, wd, td = lm_head
    V = 151936
    rows = sample_rows(34, 4096, 64, must=(0, 1, 4095))
    edge = [0, V - 1, 63, 64, 127, 128, 19007, 19008, 38015, 38016, 133055, 133056, 151871, 151872, 151873,
            151935, 76031, 76032, 114047, 114048]
    tg = targets.copy()
    for i, r in enumerate(rows):
        if i < len(edge):
            tg[r] = edge[i]
    tdd = dev_i32(tg)
    tc = lp(hd, wd, tdd, T=8, tc=True)  # the full launch, T = 8
    ref = oracle_rows(lambda rs: oracle.logprob(hidden[rs], w, tg[rs], T=1, leaf=256), rows)
    assert np.max(np.abs(tc[rows] - ref)) <= 1e-4
    ex = lp(hd[rows].contiguous(), wd, tdd[rows].contiguous(), T=2, tc=False)
    assert np.array_equal(u32(ex), u32(ref))


def test_lm_head_argument_errors(lm_head):
    _, _, _, hd, wd, td = lm_head
    lib = tbik.load_library()
    s = torch.cuda.current_stream().cuda_stream
    out = torch.empty(4, dtype=torch.float32, device="cuda")
    args = (hd.data_ptr(), wd.data_ptr(), td.data_ptr(), out.data_ptr(), 4, 151936, 4096)
    assert lib.tbik_logprob(*args, 3, 256, tbik.TC, None, 0, s) == tbik.TBIK_ERR_SHAPE
    assert lib.tbik_logprob(*args, 1, 200, tbik.TC, None, 0, s) == tbik.TBIK_ERR_SHAPE
    assert lib.tbik_logprob(*args, 1, 256, tbik.TC, None, 0, s) == tbik.TBIK_ERR_WORKSPACE
    assert lib.tbik_logprob(*args, 1, 256, tbik.TC | tbik.EXACT, None, 0, s) == tbik.TBIK_ERR_ARG
