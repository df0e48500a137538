"""Failure detection without a GPU fault: the tensor-core GEMM's epilogue is
told (test hook) to withhold its "accumulator drained" arrive, so the MMA
issuer's bounded wait expires.  The kernel must record TBIK_ERR_TIMEOUT, drain
its own copies, free its TMEM and return; the context stays usable."""
import time

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, host_f32, u32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402


# the 128-column tile kernel (forced by its test hook) and the 192-column one
# with B as [K,N] and as [N,K]
@pytest.mark.parametrize("b_nk,tile128", [(False, True), (False, False), (True, False)])
def test_withheld_arrive_times_out_and_context_survives(b_nk, tile128):
    # 148 (99) output tiles, 16 leaves each: every CTA streams more than two
    # leaves, so the MMA issuer has to wait for a drained accumulator.
    M, N, K, leaf = 128, 128 * 148, 256, 16
    a = dev_bf16(synth.normal_bf16(400, (M, K)))
    bh = synth.normal_bf16(401, (K, N), std=0.05)
    b = dev_bf16(np.ascontiguousarray(bh.T) if b_nk else bh)
    tile = tbik.DEBUG_TILE128 if tile128 else 0
    try:
        tbik.debug_set(tile, 0)
        good = host_f32(tbik.gemm(a, b, T=1, leaf=leaf, tc=True, b_nk=b_nk))
        assert tbik.get_error() == tbik.TBIK_OK
        tbik.debug_set(tile | tbik.DEBUG_WITHHOLD_ACC_ARRIVE, 50_000_000)  # 50 ms per wait
        t0 = time.time()
        tbik.gemm(a, b, T=1, leaf=leaf, tc=True, b_nk=b_nk)
        status = tbik.get_error()
        elapsed = time.time() - t0
        tbik.debug_set(tile, 0)
        again = host_f32(tbik.gemm(a, b, T=1, leaf=leaf, tc=True, b_nk=b_nk))
    finally:
        tbik.debug_set(0, 0)
    assert status == tbik.TBIK_ERR_TIMEOUT
    assert elapsed < 10.0
    assert tbik.get_error() == tbik.TBIK_OK
    assert np.array_equal(u32(again), u32(good))
    assert torch.cuda.synchronize() is None


def test_attention_withheld_arrive_times_out_and_context_survives():
    """The tensor-core attention with its epilogue's "P written" arrive
    withheld: the MMA issuer's bounded wait expires, the producer and the
    epilogue warps leave through their own bounded waits (the pair barrier
    takes both warps of a quadrant out together), the copies in flight land
    and TMEM is freed; the next call gives the same bits as before."""
    B, S, NH = 2, 1024, 4
    g = torch.Generator(device="cuda").manual_seed(9)
    q, k, v = [torch.randn(B, S, NH, 128, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3)]
    try:
        tbik.debug_set(0, 0)
        good = tbik.attention(q, k, v, tc=True).view(torch.int16).cpu().numpy()
        assert tbik.get_error() == tbik.TBIK_OK
        tbik.debug_set(tbik.DEBUG_WITHHOLD_ACC_ARRIVE, 50_000_000)  # 50 ms per wait
        t0 = time.time()
        tbik.attention(q, k, v, tc=True)
        status = tbik.get_error()
        elapsed = time.time() - t0
        tbik.debug_set(0, 0)
        again = tbik.attention(q, k, v, tc=True).view(torch.int16).cpu().numpy()
    finally:
        tbik.debug_set(0, 0)
    assert status == tbik.TBIK_ERR_TIMEOUT
    assert elapsed < 10.0
    assert tbik.get_error() == tbik.TBIK_OK
    assert np.array_equal(again, good)
