"""tbik_logprob_noalloc, the entry point for callers that cannot allocate
device memory (for example code that must not call cudaMalloc while its stream
is being captured, or plain C callers without a device allocator).

It must give the same logprobs as the allocating entry point tbik_logprob on
consecutive calls (the scratch array it shares between calls keeps the previous
call's contents), and refuse, without launching anything, arguments whose
scratch would not fit its fixed array.  This file is collected last so a run
that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, dev_i32, host_f32, u32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402

SCRATCH_BYTES = 32 << 20


def _entry():
    lib = tbik.load_library()
    fn = lib.tbik_logprob_noalloc
    vp, i32, u32_ = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
    fn.restype = i32
    fn.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, u32_, vp]
    return lib, fn


def test_noalloc_logprob_matches_allocating_entry_point_on_two_calls():
    lib, noalloc = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    V, H, leaf = 20000, 2048, 256  # 8 K leaves: the kernels use the scratch's global stack
    w = dev_bf16(synth.normal_bf16(500, (V, H), std=0.05))
    for M, T, seed in ((300, 2, 501), (200, 8, 503)):
        h = dev_bf16(synth.normal_bf16(seed, (M, H)))
        t = dev_i32(synth.uniform_int32(seed + 1, M, 0, V))
        ref = host_f32(tbik.logprob(h, w, t, T=T, leaf=leaf, tc=True))
        assert tbik.get_error() == tbik.TBIK_OK
        out = torch.full((M,), float("nan"), dtype=torch.float32, device="cuda")
        status = noalloc(h.data_ptr(), w.data_ptr(), t.data_ptr(), out.data_ptr(), M, V, H, T, leaf, tbik.TC, stream)
        assert status == tbik.TBIK_OK
        assert tbik.get_error() == tbik.TBIK_OK
        got = host_f32(out)
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref)) <= 1e-4
        assert np.array_equal(u32(got), u32(ref))


def test_noalloc_noninv_baseline_matches_allocating_entry_point():
    """The non-invariant baseline (TBIK_TC | TBIK_NONINV: a different chain
    plan and scratch size) through the fixed array, bitwise equal to
    tbik_logprob(noninv=True), on two calls in a row."""
    lib, noalloc = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    V, H, leaf = 12000, 2048, 256
    w = dev_bf16(synth.normal_bf16(510, (V, H), std=0.05))
    for M, T, seed in ((260, 4, 511), (77, 8, 513)):
        h = dev_bf16(synth.normal_bf16(seed, (M, H)))
        t = dev_i32(synth.uniform_int32(seed + 1, M, 0, V))
        ref = host_f32(tbik.logprob(h, w, t, T=T, leaf=leaf, tc=True, noninv=True))
        assert tbik.get_error() == tbik.TBIK_OK
        out = torch.full((M,), float("nan"), dtype=torch.float32, device="cuda")
        status = noalloc(h.data_ptr(), w.data_ptr(), t.data_ptr(), out.data_ptr(), M, V, H, T, leaf,
                         tbik.TC | tbik.NONINV, stream)
        assert status == tbik.TBIK_OK
        assert tbik.get_error() == tbik.TBIK_OK
        assert np.array_equal(u32(host_f32(out)), u32(ref))


def _largest_fitting_rows(lib, V, H, T, leaf):
    lo, hi = 1, 1 << 20
    while lo < hi:  # largest M whose scratch fits the fixed array
        mid = (lo + hi + 1) // 2
        if lib.tbik_logprob_workspace(mid, V, H, T, leaf, tbik.TC) <= SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid - 1
    return lo


def test_noalloc_refuses_arguments_beyond_its_scratch():
    lib, noalloc = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    V, H, leaf, T = 151936, 4096, 256, 8
    m_max = _largest_fitting_rows(lib, V, H, T, leaf)
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert m_max == 997  # the limit stated in tbik.h for the 151936 x 4096 lm_head
    big = m_max + 1
    # The size check comes before any pointer is used: small stand-in buffers.
    dummy = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    tg = torch.zeros(big, dtype=torch.int32, device="cuda")
    out = torch.full((big,), float("nan"), dtype=torch.float32, device="cuda")
    status = noalloc(dummy.data_ptr(), dummy.data_ptr(), tg.data_ptr(), out.data_ptr(), big, V, H, T, leaf, tbik.TC,
                     stream)
    assert status == tbik.TBIK_ERR_WORKSPACE
    assert noalloc(dummy.data_ptr(), dummy.data_ptr(), tg.data_ptr(), out.data_ptr(), 4, V, H, T, leaf, tbik.EXACT,
                   stream) == tbik.TBIK_ERR_ARG
    # the statuses tbik_logprob gives: an unknown mode bit, a bad shard count
    assert noalloc(dummy.data_ptr(), dummy.data_ptr(), tg.data_ptr(), out.data_ptr(), 4, V, H, T, leaf,
                   tbik.TC | 0x80, stream) == tbik.TBIK_ERR_ARG
    assert noalloc(dummy.data_ptr(), dummy.data_ptr(), tg.data_ptr(), out.data_ptr(), 4, V, H, 3, leaf, tbik.TC,
                   stream) == tbik.TBIK_ERR_SHAPE
    torch.cuda.synchronize()
    assert torch.isnan(out).all()
    assert tbik.get_error() == tbik.TBIK_OK
